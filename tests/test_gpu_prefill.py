"""GPU parity of chunked-prefill attention (nf_prefill_attn) against the CPU
oracle.  The operation is the oracle's attention with n_q = the chunk: query j
of a sequence sits at position L - n_q + j and, causal, sees keys 0 .. its own
position.  Pool bytes must match the oracle's append bit for bit; outputs
within max-abs 2e-3 and relative-L2 1e-3 of the fp64 result, lse within 2e-3."""
import os

import numpy as np
import pytest
import torch

import long_context_quantized_b200 as nf
import oracle
import workloads
from nfcase import POISON, check_attention, compare_pool, gpu_layer, oracle_attention, oracle_pool, run_case

pytestmark = pytest.mark.gpu
K8 = nf.NF_KV_K8V4


@pytest.fixture(autouse=True)
def _clean_device_error():
    torch.cuda.synchronize()
    assert nf.nf_get_device_error() == 0
    yield
    torch.cuda.synchronize()


CASES = [
    # a whole prompt as one chunk (n_q = L): textbook causal self-attention
    ("whole_prompt_300", dict(cached=(0,), n_new=300, n_q=300, num_q_heads=8, num_kv_heads=1)),
    # a ragged chunk in the middle of a block, GQA 8
    ("chunk_257_at_1000", dict(cached=(1000,), n_new=257, n_q=257, num_q_heads=32, num_kv_heads=4)),
    # two sequences of different lengths, GQA 5 (tiles span fractional positions)
    ("gqa5_ragged_batch", dict(cached=(100, 700), n_new=64, n_q=64, num_q_heads=10, num_kv_heads=2)),
    # GQA 16: one tile holds 8 positions
    ("gqa16", dict(cached=(300,), n_new=40, n_q=40, num_q_heads=16, num_kv_heads=1)),
    # one query (the decode shape through the prefill kernel)
    ("n_q_1", dict(cached=(777,), n_new=1, n_q=1, num_q_heads=8, num_kv_heads=2)),
    # queries fewer than the appended tokens: the last n_q positions
    ("n_q_below_new", dict(cached=(500,), n_new=40, n_q=24, num_q_heads=4, num_kv_heads=2)),
    # a full 1024-token chunk spanning several blocks
    ("chunk_1024_at_2048", dict(cached=(2048,), n_new=1024, n_q=1024, num_q_heads=16, num_kv_heads=2)),
]


@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_prefill_small_shapes(case, causal):
    w = workloads.custom("pf_" + case[0], q_dtype=torch.bfloat16, kv_in_dtype=torch.bfloat16, causal=causal,
                         **case[1])
    run_case(w, 0, K8, attn="prefill")


def test_prefill_mha_fp32_kv_input():
    w = workloads.custom("pf_mha", cached=(500,), n_new=100, n_q=100, num_q_heads=3, num_kv_heads=3,
                         q_dtype=torch.bfloat16, kv_in_dtype=torch.float32, causal=True, dist="head_variance")
    run_case(w, 0, K8, attn="prefill")


def test_prefill_full_size_sampled_rows():
    # the last 1024-token chunk of a 180224-token prompt; kv-head 1, rows at the
    # chunk's ends and middle
    w = workloads.get("prefill_chunk")
    hs = [1]
    g = gpu_layer(w, 0, K8, attn="prefill")
    pool, _ = oracle_pool(w, K8, g["kvin"], g["bt"], hs)
    compare_pool(g["kv"], pool, hs)
    G = w.group
    positions = [0, 1, 2, 255, 511, 512, 777, 1021, 1022, 1023]
    rows = np.array([j * G + gh for j in positions for gh in range(G)], np.int64)
    qn = g["q"].float().cpu().numpy().astype(np.float64)[:, :, hs[0] * G:(hs[0] + 1) * G]
    ref_o, ref_l = oracle.decode_attn(pool, qn, g["bt"], np.array(w.seqlens, np.int32), w.softmax_scale,
                                      w.causal, rows=rows, nthreads=os.cpu_count())
    got = g["out"][0, :, hs[0] * G:(hs[0] + 1) * G].reshape(-1, 128)[torch.as_tensor(rows)]
    gl = g["lse"][0, :, hs[0] * G:(hs[0] + 1) * G].reshape(-1)[torch.as_tensor(rows)]
    check_attention(got[None, None], gl[None, None], ref_o[None, None], ref_l[None, None])


def test_prefill_short_sequence_is_reported():
    w = workloads.custom("pf_short", cached=(200,), n_new=16, n_q=16, num_q_heads=4, num_kv_heads=1,
                         q_dtype=torch.bfloat16, kv_in_dtype=torch.bfloat16, causal=True)
    g = gpu_layer(w, 0, K8, attn="prefill")
    out = torch.full_like(g["out"], 7.0)
    lse = torch.zeros_like(g["lse"])
    nf.nf_prefill_attn(g["kv"], g["q"], torch.as_tensor(g["bt"], device="cuda"),
                       torch.tensor([10], dtype=torch.int32, device="cuda"), 216, w.softmax_scale, True, out, lse)
    torch.cuda.synchronize()
    assert nf.nf_get_device_error() == 3  # NF_DEVERR_SEQLEN, and the word is cleared
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_prefill_rejects_other_formats_and_fp32_queries():
    w = workloads.custom("pf_rej", cached=(100,), n_new=8, n_q=8, num_q_heads=4, num_kv_heads=1,
                         q_dtype=torch.bfloat16, kv_in_dtype=torch.bfloat16, causal=True)
    g = gpu_layer(w, 0, K8, attn="prefill")
    bt = torch.as_tensor(g["bt"], device="cuda")
    sl = torch.tensor([108], dtype=torch.int32, device="cuda")
    with pytest.raises(nf.NfError) as e:
        nf.nf_prefill_attn(g["kv"], g["q"].float(), bt, sl, 108, w.softmax_scale, True, g["out"], None)
    assert e.value.status == nf.NF_ERR_UNSUPPORTED
    kv8 = nf.KVLayer.empty(nf.NF_KV_K8V8, w.pool_blocks, 1, fill=0)
    with pytest.raises(nf.NfError) as e:
        nf.nf_prefill_attn(kv8, g["q"], bt, sl, 108, w.softmax_scale, True, g["out"], None)
    assert e.value.status == nf.NF_ERR_UNSUPPORTED


def _pool_with_scaled_inputs(w, k_mul, v_mul):
    dev = "cuda"
    bt_np = workloads.block_table(w)
    bt = torch.as_tensor(bt_np, device=dev)
    kv = nf.KVLayer.empty(K8, w.pool_blocks, w.num_kv_heads, device=dev, fill=POISON)
    k, v = workloads.layer_kv(w, 0, 0, device=dev)
    k, v = (k.float() * k_mul).contiguous(), (v.float() * v_mul).contiguous()
    nf.nf_kv_append_quant(kv, k[None], v[None], bt, torch.zeros(1, dtype=torch.int32, device=dev))
    return kv, bt, bt_np, [(k, v)]


def test_prefill_reports_v_outside_fp16_range_where_decode_is_exact():
    # V inputs of magnitude ~8e4: V scales above 9352, so 7 x scale leaves fp16.
    # nf_prefill_attn records NF_DEVERR_RANGE; nf_decode_attn (weights x scale
    # <= 65504) still matches the oracle.
    mul = 2e4
    w = workloads.custom("pf_range_v", cached=(0,), n_new=600, n_q=4, num_q_heads=8, num_kv_heads=1,
                         q_dtype=torch.bfloat16, kv_in_dtype=torch.float32, causal=True)
    kv, bt, bt_np, kvin = _pool_with_scaled_inputs(w, 1.0, mul)
    q = workloads.layer_q(w, 0, device="cuda")
    sl = torch.as_tensor(w.seqlens, dtype=torch.int32, device="cuda")
    out = torch.empty((1, w.n_q, w.num_q_heads, 128), device="cuda")
    lse = torch.empty((1, w.n_q, w.num_q_heads), device="cuda")
    nf.nf_prefill_attn(kv, q, bt, sl, 600, w.softmax_scale, True, out, lse)
    torch.cuda.synchronize()
    assert nf.nf_get_device_error() == nf.NF_DEVERR_RANGE
    ws = torch.zeros(nf.nf_decode_attn_workspace_size(1, w.n_q, w.num_q_heads, 1, 600), dtype=torch.uint8,
                     device="cuda")
    nf.nf_decode_attn(kv, q, bt, sl, 600, w.softmax_scale, True, out, lse, ws)
    torch.cuda.synchronize()
    assert nf.nf_get_device_error() == 0
    pool, hs = oracle_pool(w, K8, kvin, bt_np)
    compare_pool(kv, pool, hs)
    ref_o, ref_l = oracle_attention(w, pool, hs, q, bt_np)
    # the tolerance is stated for unit-scale values: compare o / mul
    check_attention(out / mul, lse, ref_o / mul, ref_l)


def test_prefill_reports_k_outside_fp16_range():
    w = workloads.custom("pf_range_k", cached=(0,), n_new=300, n_q=8, num_q_heads=4, num_kv_heads=1,
                         q_dtype=torch.bfloat16, kv_in_dtype=torch.float32, causal=True)
    kv, bt, _, _ = _pool_with_scaled_inputs(w, 3e4, 1.0)
    q = workloads.layer_q(w, 0, device="cuda")
    out = torch.empty((1, w.n_q, w.num_q_heads, 128), device="cuda")
    nf.nf_prefill_attn(kv, q, bt, torch.as_tensor(w.seqlens, dtype=torch.int32, device="cuda"), 300,
                       w.softmax_scale, True, out, None)
    torch.cuda.synchronize()
    assert nf.nf_get_device_error() == nf.NF_DEVERR_RANGE
