"""Context-sharded decode on one GPU: each shard's partial through the CUDA
decode kernel (decode_partial), the partials stacked as the all-gather would
deliver them, and the CUDA log-sum-exp combine -- against the oracle's
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
    parts = [sharded.decode_partial(g["kv"], g["q"], s, sharded.local_block_table(s, bt), w.softmax_scale)
             for s in specs]
    torch.cuda.synchronize()
    assert nf.nf_get_device_error() == 0
    rows = w.batch * w.n_q * w.num_q_heads
    part_o = torch.stack([o.reshape(rows, 128) for o, _ in parts]).contiguous()
    part_l = torch.stack([l.reshape(rows) for _, l in parts]).contiguous()
    out = torch.empty((rows, 128), device="cuda")
    lse = torch.empty(rows, device="cuda")
    nf.nf_attn_combine(part_o, part_l, out, lse)
    torch.cuda.synchronize()
    pool, hs = oracle_pool(w, nf.NF_KV_K8V4, g["kvin"], g["bt"])
    ref_o, ref_l = oracle_attention(w, pool, hs, g["q"], g["bt"])
    check_attention(out.reshape(g["out"].shape), lse.reshape(g["lse"].shape), ref_o, ref_l)
    # and it agrees with the unsharded call
    assert float((out.reshape(g["out"].shape) - g["out"]).abs().max()) < 1e-3
