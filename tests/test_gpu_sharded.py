"""Context-sharded decode on one GPU: each shard's partial through the CUDA
decode kernel written into its packed slot (decode_partial_into), the slots
stacked as the all-gather would deliver them, and the CUDA packed log-sum-exp
combine -- against the oracle's
attention over the whole cache.  The shards run one after the other on the
same device; no rank waits on another."""
import numpy as np
import pytest
import torch

import long_context_quantized_b200 as nf
import workloads
from long_context_quantized_b200 import sharded
from nfcase import check_attention, gpu_layer, oracle_attention, oracle_pool

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,case", [
    (3, dict(cached=(1500, 600), n_new=4, n_q=4, num_q_heads=16, num_kv_heads=4, causal=True)),
    (4, dict(cached=(3000, 100), n_new=1, n_q=1, num_q_heads=8, num_kv_heads=1, causal=False)),
])
def test_sharded_partials_and_combine_match_whole_attention(world, case):
    w = workloads.custom("gshard", q_dtype=torch.bfloat16, kv_in_dtype=torch.bfloat16, **case)
    g = gpu_layer(w, 0, nf.NF_KV_K8V4)
    bt = torch.as_tensor(g["bt"], device="cuda")
    specs = sharded.shard_plan(list(w.seqlens), w.n_q, world, w.causal)
    rows = w.batch * w.n_q * w.num_q_heads
    # the slots as the all-gather would deliver them: [rank][packed slot]
    parts = torch.empty((world, nf.nf_attn_packed_slot_floats(rows, 128)), device="cuda")
    ws = torch.zeros(nf.nf_decode_attn_workspace_size(w.batch, w.n_q, w.num_q_heads, w.num_kv_heads,
                                                      max(w.seqlens)), dtype=torch.uint8, device="cuda")
    for s in specs:  # one workspace serves every shard, one after the other
        sharded.decode_partial_into(g["kv"], g["q"], s, sharded.local_block_table(s, bt), w.softmax_scale,
                                    parts[s.rank], ws)
    torch.cuda.synchronize()
    assert nf.nf_get_device_error() == 0
    out = torch.empty((rows, 128), device="cuda")
    lse = torch.empty(rows, device="cuda")
    nf.nf_attn_combine_packed(parts, rows, out, lse)
    torch.cuda.synchronize()
    # the two-array combine of the same partials gives the same numbers
    views = [sharded.packed_views(parts[r], w.batch, w.n_q, w.num_q_heads) for r in range(world)]
    out2 = torch.empty_like(out)
    nf.nf_attn_combine(torch.stack([v[0].reshape(rows, 128) for v in views]).contiguous(),
                       torch.stack([v[1].reshape(rows) for v in views]).contiguous(), out2, None)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
    pool, hs = oracle_pool(w, nf.NF_KV_K8V4, g["kvin"], g["bt"])
    ref_o, ref_l = oracle_attention(w, pool, hs, g["q"], g["bt"])
    check_attention(out.reshape(g["out"].shape), lse.reshape(g["lse"].shape), ref_o, ref_l)
    # and it agrees with the unsharded call
    assert float((out.reshape(g["out"].shape) - g["out"]).abs().max()) < 1e-3


def test_sharded_decoder_single_rank_equals_plain_call():
    w = workloads.custom("gshard1", cached=(5000,), n_new=4, n_q=4, num_q_heads=32, num_kv_heads=4, causal=True,
                         q_dtype=torch.bfloat16, kv_in_dtype=torch.bfloat16)
    g = gpu_layer(w, 0, nf.NF_KV_K8V4)
    bt = torch.as_tensor(g["bt"], device="cuda")
    spec = sharded.shard_plan(list(w.seqlens), w.n_q, 1, w.causal)[0]
    dec = sharded.ShardedDecoder(spec, w.batch, w.n_q, w.num_q_heads, w.num_kv_heads, "cuda")
    for _ in range(2):  # buffers and workspace reused
        o, lse = dec(g["kv"], g["q"], sharded.local_block_table(spec, bt), w.softmax_scale)
        torch.cuda.synchronize()
        assert torch.equal(o, g["out"]) and torch.equal(lse, g["lse"])


def test_bench_sharded_path_single_rank_matches_the_oracle():
    # the bench's shard-local pool (only this rank's blocks, local table) for
    # one rank holding everything, with the step's appended tokens: the
    # decoder's output per layer against the oracle
    import bench
    w = workloads.custom("bshard", cached=(3000,), n_new=4, n_q=4, num_q_heads=16, num_kv_heads=2, causal=True,
                         q_dtype=torch.bfloat16, kv_in_dtype=torch.bfloat16, layers=2)
    sw = bench.ShardedWorkload(w, "k8v4", torch.device("cuda", 0), 1, 0)
    assert sw.appends
    sw.step()
    torch.cuda.synchronize()
    assert nf.nf_get_device_error() == 0
    for layer in range(w.layers):
        kvin = [workloads.layer_kv(w, layer, b, device="cuda") for b in range(w.batch)]
        bt = sw.local_bt.cpu().numpy()
        pool, hs = oracle_pool(w, nf.NF_KV_K8V4, kvin, bt)
        ref_o, ref_l = oracle_attention(w, pool, hs, sw.q[layer], bt)
        check_attention(sw.out_all[layer], sw.lse_all[layer], ref_o, ref_l)
