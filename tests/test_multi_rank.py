"""The N > 1 path of bench.py on CPU: world_size-2 gloo process groups.

Decode attention for one request runs on one GPU; with N GPUs the bench runs N
independent replicas (weak scaling) and the job's time is the slowest rank's.
These tests check that reduction and the whole-job throughput on real
process groups, without a GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, results):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank])
        value = bench.job_throughput(1000.0, dist.get_world_size(), ms)
        dist.barrier()
        results[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("times", [(2.0, 3.5), (4.25, 1.0)])
def test_slowest_rank_sets_job_time(times):
    world = 2
    mgr = mp.Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), times, results), nprocs=world,
                       join=True, start_method="spawn")
    slow = max(times)
    for r in range(world):
        ms, value = results[r]
        assert ms == slow
        # 1000 KV tokens per rank, two ranks, over the slowest rank's time
        assert value == pytest.approx(2 * 1000.0 / (slow / 1e3))


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks(7.5) == 7.5
    assert bench.job_throughput(500.0, 1, 2.0) == pytest.approx(250000.0)
