"""Multi-rank host logic of the bench on CPU: two gloo ranks on 127.0.0.1.

The bench's multi-GPU mode runs one independent workload per rank (weak
scaling, no data-path collective); the only cross-rank steps are the timing
reductions.  These tests run them on a real two-process gloo group.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # per-rank timings: rank r is slower in one field, faster in another
        local = [1.0 + rank, 5.0 - rank, 2.5, 0.1 * (rank + 1)]
        got = bench.max_over_ranks(torch, dist, local, "cpu")
        rate = bench.whole_job_rate(100.0, world, got[0])
        seeds = [bench.rank_seed(2000, i, rank) for i in range(4)]
        gathered = [None] * world
        dist.all_gather_object(gathered, seeds)
        out[rank] = (got, rate, gathered)
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_timing_reduction_and_seeds():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert set(out.keys()) == {0, 1}
    for rank in range(world):
        got, rate, gathered = out[rank]
        assert got == [2.0, 5.0, 2.5, 0.2]                   # element-wise max, same on every rank
        assert rate == pytest.approx(world * 100.0 / 2.0)     # all ranks' units / slowest rank's time
        flat = [s for seeds in gathered for s in seeds]
        assert len(set(flat)) == len(flat)                    # every rank draws its own inputs


def test_single_process_helpers_without_group():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(torch, dist, [3.0, 1.5], "cpu") == [3.0, 1.5]
    assert bench.whole_job_rate(10.0, 1, 2.0) == 5.0
    assert bench.rank_seed(4000, 2, 0) != bench.rank_seed(4000, 2, 1)
