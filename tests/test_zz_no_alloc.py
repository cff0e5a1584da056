"""nf_decode_attn_noalloc: the decode-attention entry point for callers that
cannot allocate device memory at call time (an engine that reserves its whole
budget at start-up and gives plug-ins no allocator, or a latency-critical loop
that cannot afford cudaMalloc's implicit synchronisation).  Its scratch is a
fixed array inside libnf's device image.

Checked through the C ABI against nf_decode_attn (caller-provided workspace)
on two calls in a row with different queries.  Both run the same deterministic
kernel with the same split plan, so the results must be identical bit for bit;
any leftover of the previous call in the shared scratch would show.  This
file is collected last on purpose."""
import pytest
import torch

import long_context_quantized_b200 as nf
import workloads
from nfcase import gpu_layer

pytestmark = pytest.mark.gpu


def _two_calls_match(w):
    g = gpu_layer(w, 0, nf.NF_KV_K8V4)
    bt = torch.as_tensor(g["bt"], device="cuda")
    sl = torch.as_tensor(w.seqlens, dtype=torch.int32, device="cuda")
    msl = max(w.seqlens)
    need = nf.nf_decode_attn_workspace_size(w.batch, w.n_q, w.num_q_heads, w.num_kv_heads, msl)
    assert need <= nf.NF_NOALLOC_SCRATCH_BYTES
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    queries = [g["q"], (g["q"].float() * -1.5).to(torch.bfloat16)]
    for q in queries:  # two calls in a row; the second must not see the first's scratch
        ref = torch.empty_like(g["out"])
        ref_lse = torch.empty_like(g["lse"])
        nf.nf_decode_attn(g["kv"], q, bt, sl, msl, w.softmax_scale, w.causal, ref, ref_lse, ws)
        out = torch.full_like(g["out"], float("nan"))
        lse = torch.full_like(g["lse"], float("nan"))
        nf.nf_decode_attn_noalloc(g["kv"], q, bt, sl, msl, w.softmax_scale, w.causal, out, lse)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert torch.equal(out, ref)
        assert torch.equal(lse, ref_lse)
    assert nf.nf_get_device_error() == 0


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    # ragged batch, causal MTP rows (32 per kv-head: the tcgen05 kernel):
    # segments split over a few CTAs, their final merges shared among them
    w = workloads.custom("noalloc", cached=(3000, 1200), n_new=4, n_q=4, num_q_heads=16, num_kv_heads=2,
                         q_dtype=torch.bfloat16, kv_in_dtype=torch.bfloat16, causal=True)
    _two_calls_match(w)


def test_noalloc_merge_from_the_ring_on_two_calls():
    # four segments of about 37 pieces each, 8 rows: the partial slots fit the
    # idle stage ring, so the last ticket's CTA merges them from its bulk copy
    w = workloads.custom("noalloc_ring", cached=(20000,), n_q=1, num_q_heads=32, num_kv_heads=4,
                         q_dtype=torch.bfloat16, kv_in_dtype=torch.bfloat16, causal=False)
    _two_calls_match(w)


def test_noalloc_merge_from_l2_on_two_calls():
    # one sequence and one kv-head: every CTA holds a piece of the single
    # segment, more partial slots than the stage ring holds, so the last
    # ticket's CTA merges them from L2 -- the ticket state reused across calls
    w = workloads.custom("noalloc_long", cached=(60000,), n_q=1, num_q_heads=8, num_kv_heads=1,
                         q_dtype=torch.bfloat16, kv_in_dtype=torch.bfloat16, causal=False)
    _two_calls_match(w)


def test_noalloc_refuses_shapes_above_its_scratch():
    # 64 sequences x 8 queries x 64 heads needs far more scratch than the fixed array
    kv = nf.KVLayer.empty(nf.NF_KV_K8V4, 4, 8, device="cuda", fill=0)
    B, n_q, H_q, msl = 64, 8, 64, 1 << 20
    need = nf.nf_decode_attn_workspace_size(B, n_q, H_q, 8, msl)
    assert need > nf.NF_NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, n_q, H_q, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((B, n_q, H_q, 128), dtype=torch.float32, device="cuda")
    bt = torch.zeros((B, msl // 256), dtype=torch.int32, device="cuda")
    sl = torch.full((B,), 16, dtype=torch.int32, device="cuda")
    with pytest.raises(nf.NfError) as e:
        nf.nf_decode_attn_noalloc(kv, q, bt, sl, msl, 0.1, False, out)
    assert e.value.status == nf.NF_ERR_WORKSPACE
