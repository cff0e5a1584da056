"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Codes and scales must match bit for bit (every byte of the pool planes,
untouched slots included); attention outputs within max-abs 2e-3 and
relative-L2 1e-3 of the oracle's fp64 result, lse within 2e-3.
"""
import math

import numpy as np
import pytest
import torch

import long_context_quantized_b200 as nf
import oracle
import workloads
from nfcase import ATOL, REL_L2, run_case, gpu_layer, oracle_pool, compare_pool, oracle_attention, \
    select_heads, check_attention

pytestmark = pytest.mark.gpu

K8, BF, I8, F8, K4 = nf.NF_KV_K8V4, nf.NF_KV_BF16, nf.NF_KV_K8V8, nf.NF_KV_F8, nf.NF_KV_K4V4


@pytest.fixture(autouse=True)
def _clean_device_error():
    torch.cuda.synchronize()
    assert nf.nf_get_device_error() == 0
    yield
    torch.cuda.synchronize()


# ----------------------------------------------------------- edge-case shapes
SMALL = [
    # (id, kwargs for workloads.custom)
    ("len1", dict(cached=(1,))),
    ("len15", dict(cached=(15,))),
    ("len16", dict(cached=(16,))),
    ("len17", dict(cached=(17,))),
    ("len255", dict(cached=(255,))),
    ("len256", dict(cached=(256,))),
    ("len257", dict(cached=(257,))),
    ("len1000_gqa8", dict(cached=(1000,), num_q_heads=16, num_kv_heads=2)),
    ("len700_mha", dict(cached=(700,), num_q_heads=3, num_kv_heads=3)),
    ("len2049_gqa5", dict(cached=(2049,), num_q_heads=10, num_kv_heads=2)),
    ("ragged3", dict(cached=(1, 300, 1000), num_q_heads=8, num_kv_heads=2)),
    ("mtp4_causal", dict(cached=(500,), n_new=4, n_q=4, num_q_heads=32, num_kv_heads=4, causal=True)),
    ("mtp4_noncausal", dict(cached=(500,), n_new=4, n_q=4, num_q_heads=8, num_kv_heads=2, causal=False)),
    ("mtp3_gqa5", dict(cached=(300, 41), n_new=3, n_q=3, num_q_heads=10, num_kv_heads=2, causal=True)),
    ("mtp4_short", dict(cached=(0,), n_new=4, n_q=4, num_q_heads=8, num_kv_heads=1, causal=True)),
    ("append1", dict(cached=(767,), n_new=1, num_q_heads=8, num_kv_heads=1)),
    ("q_rows_64", dict(cached=(400,), n_new=4, n_q=4, num_q_heads=16, num_kv_heads=1, causal=True)),
]


@pytest.mark.parametrize("fmt", [K8, BF, I8, F8, K4], ids=["k8v4", "bf16", "k8v8", "f8", "k4v4"])
@pytest.mark.parametrize("qdt", [torch.float32, torch.bfloat16], ids=["qf32", "qbf16"])
@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_shapes(case, qdt, fmt):
    w = workloads.custom(case[0], q_dtype=qdt, kv_in_dtype=qdt, **case[1])
    run_case(w, 0, fmt)


def test_max_seqlen_above_actual_lengths():
    # the split plan is sized for 5000 keys; the sequences are shorter, so the
    # trailing splits see no key and must not disturb the result
    w = workloads.custom("slack", cached=(700, 33), num_q_heads=8, num_kv_heads=2)
    run_case(w, 0, K8, max_seqlen=5000)


def test_large_query_scale_and_outlier_keys():
    # peaked softmax: a large-norm query against outlier channels
    w = workloads.custom("peaked", cached=(3000,), num_q_heads=8, num_kv_heads=1,
                         q_dtype=torch.bfloat16, kv_in_dtype=torch.bfloat16, dist="k_outlier_channels")
    q = workloads.layer_q(w, 0, device="cuda").float() * 6.0
    run_case(w, 0, K8, q_override=q.to(torch.bfloat16))


# ------------------------------------------------------------- combine
def test_combine_matches_oracle():
    g = torch.Generator(device="cpu").manual_seed(5)
    S, rows = 37, 45
    po = torch.randn((S, rows, 128), generator=g)
    pl = torch.randn((S, rows), generator=g) * 4
    pl[3] = -math.inf
    pl[:, 7] = -math.inf          # a row no split saw
    out = torch.empty((rows, 128), device="cuda")
    lse = torch.empty(rows, device="cuda")
    nf.nf_attn_combine(po.cuda(), pl.cuda(), out, lse)
    ro, rl = oracle.combine(po.double().numpy(), pl.double().numpy())
    go = out.cpu().double().numpy()
    assert np.abs(go - ro).max() <= 1e-5
    gl = lse.cpu().double().numpy()
    assert gl[7] == -math.inf and np.all(go[7] == 0)
    fin = np.isfinite(rl)
    assert np.abs(gl[fin] - rl[fin]).max() <= 1e-5


# ------------------------------------------------ device checks, no faults
def test_bad_block_id_is_reported_not_faulted():
    w = workloads.custom("bad", cached=(600,), num_q_heads=4, num_kv_heads=1)
    bt = workloads.block_table(w).copy()
    g = gpu_layer(w, 0, K8)                     # a clean run first
    assert nf.nf_get_device_error() == 0
    bt_bad = torch.as_tensor(bt, dtype=torch.int32, device="cuda")
    bt_bad[0, 1] = w.pool_blocks + 7            # the block holding keys 256..511
    out = torch.empty_like(g["out"])
    sl = torch.tensor([600], dtype=torch.int32, device="cuda")
    ws = torch.zeros(nf.nf_decode_attn_workspace_size(1, 1, 4, 1, 600), dtype=torch.uint8, device="cuda")
    nf.nf_decode_attn(g["kv"], g["q"], bt_bad, sl, 600, w.softmax_scale, False, out, None, ws)
    assert nf.nf_get_device_error() == nf.NF_DEVERR_BLOCK_ID
    # the context is still usable and a correct call still gives the right answer
    nf.nf_decode_attn(g["kv"], g["q"], torch.as_tensor(bt, device="cuda"), sl, 600, w.softmax_scale,
                      False, out, None, ws)
    torch.cuda.synchronize()
    assert torch.equal(out, g["out"])
    assert nf.nf_get_device_error() == 0


def test_append_outside_table_is_reported():
    kv = nf.KVLayer.empty(K8, 2, 1, fill=0)
    bt = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    k = torch.randn((1, 1, 1, 128), device="cuda")
    nf.nf_kv_append_quant(kv, k, k, bt, torch.tensor([512], dtype=torch.int32, device="cuda"))
    assert nf.nf_get_device_error() == nf.NF_DEVERR_TABLE
    bt[0, 1] = 9
    nf.nf_kv_append_quant(kv, k, k, bt, torch.tensor([256], dtype=torch.int32, device="cuda"))
    assert nf.nf_get_device_error() == nf.NF_DEVERR_BLOCK_ID
    assert torch.all(kv.k_codes == 0)


def test_seqlen_above_bound_is_reported():
    w = workloads.custom("sl", cached=(300,), num_q_heads=4, num_kv_heads=1)
    g = gpu_layer(w, 0, K8)
    sl = torch.tensor([400], dtype=torch.int32, device="cuda")
    out = torch.empty_like(g["out"])
    lse = torch.empty_like(g["lse"])
    ws = torch.zeros(nf.nf_decode_attn_workspace_size(1, 1, 4, 1, 300), dtype=torch.uint8, device="cuda")
    nf.nf_decode_attn(g["kv"], g["q"], torch.as_tensor(g["bt"], device="cuda"), sl, 300,
                      w.softmax_scale, False, out, lse, ws)
    assert nf.nf_get_device_error() == nf.NF_DEVERR_SEQLEN
    assert torch.all(out == 0) and torch.all(torch.isinf(lse))


def test_bounded_wait_times_out_and_context_survives():
    # a wait that nothing ends gives up after its limit and reports, instead of
    # hanging the GPU; the context stays usable
    nf.nf_selftest_bounded_wait(20000)  # 20 ms
    torch.cuda.synchronize()
    assert nf.nf_get_device_error() == nf.NF_DEVERR_TIMEOUT
    w = workloads.custom("after_timeout", cached=(500,), num_q_heads=8, num_kv_heads=1)
    run_case(w, 0, K8)
    assert nf.nf_get_device_error() == 0


def test_workspace_too_small_is_refused():
    w = workloads.custom("ws", cached=(300,), num_q_heads=4, num_kv_heads=1)
    g = gpu_layer(w, 0, K8)
    need = nf.nf_decode_attn_workspace_size(1, 1, 4, 1, 300)
    ws = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(nf.NfError) as e:
        nf.nf_decode_attn(g["kv"], g["q"], torch.as_tensor(g["bt"], device="cuda"),
                          torch.tensor([300], dtype=torch.int32, device="cuda"), 300,
                          w.softmax_scale, False, torch.empty_like(g["out"]), None, ws)
    assert e.value.status == nf.NF_ERR_WORKSPACE


# ------------------------------------------------- the five workloads, full size
def _full_size(name, fmt, heads, layer=0):
    w = workloads.get(name)
    g = gpu_layer(w, layer, fmt)
    pool, hs = oracle_pool(w, fmt, g["kvin"], g["bt"], heads)
    compare_pool(g["kv"], pool, hs)
    ref_o, ref_l = oracle_attention(w, pool, hs, g["q"], g["bt"])
    return check_attention(select_heads(g["out"], w, hs), select_heads(g["lse"], w, hs), ref_o, ref_l)


# K8/V4 at full size: every layer's codes and every kv-head's attention of three
# layers per workload are in test_gpu_full_size.py.


def test_workload_longest_bf16_cache_sampled_head():
    _full_size("longest", BF, heads=[5])


@pytest.mark.parametrize("name,heads", [("ctx32k_append", [2]), ("mtp_verify", [1]), ("longest", [3])])
def test_workload_int8_cache_sampled_heads(name, heads):
    _full_size(name, I8, heads=heads)


@pytest.mark.parametrize("name,heads", [("ctx32k_append", [1]), ("mtp_verify", [3]), ("longest", [6])])
def test_workload_fp8_cache_sampled_heads(name, heads):
    _full_size(name, F8, heads=heads)


@pytest.mark.parametrize("name,heads", [("ctx32k_append", [3]), ("ragged_c2", [1]), ("mtp_verify", [0]),
                                        ("longest", [2])])
def test_workload_k4v4_cache_sampled_heads(name, heads):
    _full_size(name, K4, heads=heads)


def test_k4v4_groups_of_very_different_magnitudes():
    # V groups of one key 2^20 apart in magnitude and keys whose largest V
    # exponents differ widely: the per-key exponent shift and the per-group
    # factors keep every weight inside fp16
    w = workloads.custom("k4_mag", cached=(900,), n_new=4, n_q=4, num_q_heads=8, num_kv_heads=1,
                         q_dtype=torch.bfloat16, kv_in_dtype=torch.float32, causal=True)
    dev = "cuda"
    bt_np = workloads.block_table(w)
    bt = torch.as_tensor(bt_np, device=dev)
    k, v = workloads.layer_kv(w, 0, 0, device=dev)
    g = torch.Generator(device="cpu").manual_seed(9)
    vmul = (2.0 ** torch.randint(-12, 13, (904, 1, 4), generator=g).float()).repeat_interleave(32, dim=2).to(dev)
    v = (v * vmul).contiguous()
    kv = nf.KVLayer.empty(K4, w.pool_blocks, 1, device=dev, fill=0xA5)
    nf.nf_kv_append_quant(kv, k[None].contiguous(), v[None], bt, torch.zeros(1, dtype=torch.int32, device=dev))
    q = workloads.layer_q(w, 0, device=dev)
    sl = torch.as_tensor(w.seqlens, dtype=torch.int32, device=dev)
    out = torch.empty((1, 4, 8, 128), device=dev)
    lse = torch.empty((1, 4, 8), device=dev)
    ws = torch.zeros(nf.nf_decode_attn_workspace_size(1, 4, 8, 1, 904), dtype=torch.uint8, device=dev)
    nf.nf_decode_attn(kv, q, bt, sl, 904, w.softmax_scale, True, out, lse, ws)
    torch.cuda.synchronize()
    pool, hs = oracle_pool(w, K4, [(k, v)], bt_np)
    compare_pool(kv, pool, hs)
    ref_o, ref_l = oracle_attention(w, pool, hs, q, bt_np)
    # the values span 2^24: compare relative to the output norm per row
    go = out.cpu().double().numpy().reshape(ref_o.shape)
    rel = np.linalg.norm(go - ref_o) / np.linalg.norm(ref_o)
    assert np.all(np.isfinite(go)) and rel <= REL_L2, rel
    fin = np.isfinite(ref_l)
    assert np.abs(lse.cpu().double().numpy().reshape(ref_l.shape)[fin] - ref_l[fin]).max() <= 2e-3


# ------------------------------------------- early KV streaming (flag path)
@pytest.mark.parametrize("name,kw,fmt", [
    ("mtp", dict(cached=(700,), n_new=4, n_q=4, num_q_heads=32, num_kv_heads=4, causal=True), K8),
    ("ragged", dict(cached=(1500, 3000), n_new=1, num_q_heads=16, num_kv_heads=2), K8),
    ("mtp_int8", dict(cached=(700,), n_new=4, n_q=4, num_q_heads=32, num_kv_heads=4, causal=True), I8),
    ("ragged_fp8", dict(cached=(1500, 3000), n_new=1, num_q_heads=16, num_kv_heads=2), F8),
    ("mtp_k4v4", dict(cached=(700,), n_new=4, n_q=4, num_q_heads=32, num_kv_heads=4, causal=True), K4),
    ("ragged_k4v4", dict(cached=(1500, 3000), n_new=1, num_q_heads=16, num_kv_heads=2), K4),
])
def test_early_kv_back_to_back_layers(name, kw, fmt):
    # several layers of (append the step's tokens, decode) queued on one stream
    # without host syncs, so each decode kernel starts while the append before
    # it runs; with NF_DECODE_EARLY_KV the decode streams the older rows before
    # the append has finished.  Results must equal the plain call bit for bit
    # and match the oracle.
    w = workloads.custom("early_" + name, q_dtype=torch.bfloat16, kv_in_dtype=torch.bfloat16, layers=3, **kw)
    dev = "cuda"
    bt_np = workloads.block_table(w)
    bt = torch.as_tensor(bt_np, device=dev)
    before = torch.as_tensor(w.cached, dtype=torch.int32, device=dev)
    sl = torch.as_tensor(w.seqlens, dtype=torch.int32, device=dev)
    msl = max(w.seqlens)
    res = {}
    for flags in (0, nf.NF_DECODE_EARLY_KV):
        kvs, news, qs = [], [], []
        for layer in range(w.layers):
            kv = nf.KVLayer.empty(fmt, w.pool_blocks, w.num_kv_heads, device=dev, fill=0xA5)
            kn, vn = [], []
            for b in range(w.batch):
                k, v = workloads.layer_kv(w, layer, b, device=dev)
                c = w.cached[b]
                nf.nf_kv_append_quant(kv, k[None, :c].contiguous(), v[None, :c].contiguous(), bt[b:b + 1],
                                      torch.zeros(1, dtype=torch.int32, device=dev))
                kn.append(k[c:])
                vn.append(v[c:])
            kvs.append(kv)
            news.append((torch.stack(kn).contiguous(), torch.stack(vn).contiguous()))
            qs.append(workloads.layer_q(w, layer, device=dev))
        ws = torch.zeros(nf.nf_decode_attn_workspace_size(w.batch, w.n_q, w.num_q_heads, w.num_kv_heads, msl),
                         dtype=torch.uint8, device=dev)
        outs = [torch.empty((w.batch, w.n_q, w.num_q_heads, 128), device=dev) for _ in range(w.layers)]
        lses = [torch.empty((w.batch, w.n_q, w.num_q_heads), device=dev) for _ in range(w.layers)]
        torch.cuda.synchronize()
        for layer in range(w.layers):
            nf.nf_kv_append_quant(kvs[layer], news[layer][0], news[layer][1], bt, before)
            nf.nf_decode_attn_ex(kvs[layer], qs[layer], bt, sl, msl, w.softmax_scale, w.causal, flags,
                                 outs[layer], lses[layer], ws)
        torch.cuda.synchronize()
        assert nf.nf_get_device_error() == 0
        res[flags] = (outs, lses, kvs, qs)
    for layer in range(w.layers):
        assert torch.equal(res[0][0][layer], res[1][0][layer])
        assert torch.equal(res[0][1][layer], res[1][1][layer])
    # the last layer against the oracle
    layer = w.layers - 1
    kvin = [workloads.layer_kv(w, layer, b, device=dev) for b in range(w.batch)]
    pool, hs = oracle_pool(w, fmt, kvin, bt_np)
    compare_pool(res[1][2][layer], pool, hs)
    ref_o, ref_l = oracle_attention(w, pool, hs, res[1][3][layer], bt_np)
    check_attention(res[1][0][layer], res[1][1][layer], ref_o, ref_l)


def test_decode_flags_rejects_unknown_bits():
    w = workloads.custom("flags", cached=(300,), num_q_heads=4, num_kv_heads=1)
    g = gpu_layer(w, 0, K8)
    ws = torch.zeros(nf.nf_decode_attn_workspace_size(1, 1, 4, 1, 300), dtype=torch.uint8, device="cuda")
    with pytest.raises(nf.NfError) as e:
        nf.nf_decode_attn_ex(g["kv"], g["q"], torch.as_tensor(g["bt"], device="cuda"),
                             torch.tensor([300], dtype=torch.int32, device="cuda"), 300, w.softmax_scale, False,
                             0x2, torch.empty_like(g["out"]), None, ws)
    assert e.value.status == nf.NF_ERR_INVALID_ARG


@pytest.mark.parametrize("name,kw", [
    # 8 rows per kv-head, several segments per CTA and many pieces per segment
    ("rows8", dict(cached=(20000, 3000, 9000), num_q_heads=16, num_kv_heads=2)),
    # 32 rows per kv-head: partials larger than one ring round -> two-step merge
    ("rows32", dict(cached=(60000,), n_new=4, n_q=4, num_q_heads=32, num_kv_heads=4, causal=True)),
])
def test_repeated_calls_are_bitwise_identical(name, kw):
    # which CTA takes a segment's last ticket changes from run to run; the
    # merges must not depend on it
    w = workloads.custom("rep_" + name, q_dtype=torch.bfloat16, kv_in_dtype=torch.bfloat16, **kw)
    g = gpu_layer(w, 0, K8)
    bt = torch.as_tensor(g["bt"], device="cuda")
    sl = torch.as_tensor(w.seqlens, dtype=torch.int32, device="cuda")
    ws = torch.zeros(nf.nf_decode_attn_workspace_size(w.batch, w.n_q, w.num_q_heads, w.num_kv_heads,
                                                      max(w.seqlens)), dtype=torch.uint8, device="cuda")
    for _ in range(5):
        out = torch.empty_like(g["out"])
        lse = torch.empty_like(g["lse"])
        nf.nf_decode_attn(g["kv"], g["q"], bt, sl, max(w.seqlens), w.softmax_scale, w.causal, out, lse, ws)
        torch.cuda.synchronize()
        assert torch.equal(out, g["out"]) and torch.equal(lse, g["lse"])
    assert nf.nf_get_device_error() == 0
    hs = [0]
    pool, hs = oracle_pool(w, K8, g["kvin"], g["bt"], hs)
    ref_o, ref_l = oracle_attention(w, pool, hs, g["q"], g["bt"])
    check_attention(select_heads(g["out"], w, hs), select_heads(g["lse"], w, hs), ref_o, ref_l)
