"""Context-sharded decode (long_context_quantized_b200.sharded) on CPU.

The shard plan is checked as index arithmetic, and the exchange as world_size
2 and 3 gloo process groups.  Each rank's partial stands in for its GPU decode
through the oracle (the test's own computation), the ranks all-gather the
partials with the package's gather_partials, and the oracle's log-sum-exp
merge of them must equal the oracle's attention over the whole cache.
"""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from long_context_quantized_b200 import sharded  # noqa: E402


@pytest.mark.parametrize("world", [1, 2, 3, 8])
@pytest.mark.parametrize("n_q", [1, 4])
def test_shard_plan_covers_every_key_once(world, n_q):
    seqlens = [5, 256, 257, 1000, 4096 + 3, 300]
    specs = sharded.shard_plan(seqlens, n_q, world, causal=True)
    assert len(specs) == world
    for b, L in enumerate(seqlens):
        nb = math.ceil(L / 256)
        first = [s.first_block[b] for s in specs]
        count = [s.n_blocks[b] for s in specs]
        # contiguous ranges that tile [0, nb)
        assert first[0] == 0 and sum(count) == nb
        for r in range(1, world):
            assert first[r] == first[r - 1] + count[r - 1]
        assert sum(s.lengths[b] for s in specs) == L
        # every shard but the last ends at or before the first query's position
        for s in specs[:-1]:
            if s.lengths[b]:
                assert 256 * (s.first_block[b] + s.n_blocks[b]) <= L - n_q
        assert specs[-1].lengths[b] >= n_q
    assert [s.causal for s in specs] == [False] * (world - 1) + [True]
    assert not any(s.causal for s in sharded.shard_plan(seqlens, n_q, world, causal=False))


def test_shard_plan_balances_long_sequences():
    specs = sharded.shard_plan([262144], 1, 8, causal=False)
    assert [s.lengths[0] for s in specs] == [32768] * 8


def test_local_block_table_slices_rows():
    bt = torch.arange(24, dtype=torch.int32).reshape(2, 12)
    specs = sharded.shard_plan([3000, 700], 1, 2, causal=False)
    t0 = sharded.local_block_table(specs[0], bt)
    t1 = sharded.local_block_table(specs[1], bt)
    assert t0[0, :6].tolist() == list(range(0, 6)) and t1[0, :6].tolist() == list(range(6, 12))
    assert t0[1, :1].tolist() == [12] and t1[1, :2].tolist() == [13, 14]
    assert (t0[1, 1:] == -1).all() and (t1[1, 2:] == -1).all()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, case, results):
    sys.path.insert(0, ROOT)
    import oracle
    import workloads
    from long_context_quantized_b200 import sharded as sh
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        w = workloads.custom("shard", q_dtype=torch.float32, kv_in_dtype=torch.float32, **case)
        bt = workloads.block_table(w)
        pool = oracle.Pool(oracle.FMT_K8V4, w.pool_blocks, w.num_kv_heads, 128)
        for b in range(w.batch):
            k, v = workloads.layer_kv(w, 0, b)
            assert oracle.append(pool, k.numpy()[None], v.numpy()[None], bt[b:b + 1], np.zeros(1, np.int32)) == 0
        q = workloads.layer_q(w, 0).numpy().astype(np.float64)
        spec = sh.shard_plan(list(w.seqlens), w.n_q, world, w.causal)[rank]
        local = sh.local_block_table(spec, torch.as_tensor(bt)).numpy()
        # this rank's partial (the oracle standing in for its GPU decode)
        rows = w.batch * w.n_q * w.num_q_heads
        o = np.zeros((w.batch, w.n_q, w.num_q_heads, 128))
        lse = np.full((w.batch, w.n_q, w.num_q_heads), -np.inf)
        for b in range(w.batch):
            if spec.lengths[b]:
                ob, lb = oracle.decode_attn(pool, q[b:b + 1], local[b:b + 1], [spec.lengths[b]], w.softmax_scale,
                                            spec.causal)
                o[b] = ob.reshape(w.n_q, w.num_q_heads, 128)
                lse[b] = lb.reshape(w.n_q, w.num_q_heads)
        # the rank's packed slot (o rows, then lse), exchanged in one all-gather
        import long_context_quantized_b200 as nf
        slot = torch.zeros(nf.nf_attn_packed_slot_floats(rows, 128), dtype=torch.float32)
        so, sl = sh.packed_views(slot, w.batch, w.n_q, w.num_q_heads)
        so.copy_(torch.from_numpy(o.astype(np.float32)))
        sl.copy_(torch.from_numpy(lse.astype(np.float32)))
        parts = sh.gather_packed(slot)
        assert parts.shape == (world, slot.numel())
        # rank order: this rank's own slot sits at its index
        assert torch.equal(parts[rank], slot)
        views = [sh.packed_views(parts[r], w.batch, w.n_q, w.num_q_heads) for r in range(world)]
        part_o = torch.stack([v[0].reshape(rows, 128) for v in views])
        part_l = torch.stack([v[1].reshape(rows) for v in views])
        out, out_lse = oracle.combine(part_o.numpy().astype(np.float64), part_l.numpy().astype(np.float64))
        ref, ref_lse = oracle.decode_attn(pool, q, bt, list(w.seqlens), w.softmax_scale, w.causal)
        results[rank] = (float(np.abs(out - ref).max()), float(np.abs(out_lse - ref_lse).max()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [
    (2, dict(cached=(1500, 600), n_new=4, n_q=4, num_q_heads=8, num_kv_heads=2, causal=True)),
    (3, dict(cached=(700, 2000, 100), n_new=1, n_q=1, num_q_heads=4, num_kv_heads=1, causal=False)),
])
def test_sharded_partials_merge_to_the_whole(world, case):
    mgr = mp.Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), case, results), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        err_o, err_l = results[r]
        # fp32 exchange of fp64 partials: relative 2^-24 per value
        assert err_o < 1e-6 and err_l < 1e-5


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_local_pool_table_holds_each_shard_in_its_own_pool(world):
    # a rank storing only its shard: local blocks are numbered from 0, and
    # local position p of sequence b maps to global position first * 256 + p
    seqlens = [5, 256, 1000, 4096 + 3]
    specs = sharded.shard_plan(seqlens, 4, world, causal=True)
    covered = [set() for _ in seqlens]
    for s in specs:
        t = sharded.local_pool_table(s)
        ids = t[t >= 0].tolist()
        assert sorted(ids) == list(range(sum(s.n_blocks)))   # every local block used once
        for b in range(len(seqlens)):
            pos = sharded.shard_positions(s, b)
            assert len(pos) == s.lengths[b]
            assert all(t[b, (p - pos.start) // 256] >= 0 for p in pos)
            covered[b].update(pos)
    assert [sorted(c) for c in covered] == [list(range(L)) for L in seqlens]
