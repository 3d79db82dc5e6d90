"""Multi-rank host logic on CPU: two gloo ranks on 127.0.0.1.

The bench's multi-GPU mode runs one independent workload per rank (weak
scaling, no data-path collective); its only cross-rank steps are the timing
reductions.  A tensor whose rows are split over ranks is quantized with one
4-byte all-reduce(MAX) of max |x| (nvfp4_quantize_row_shard).  These tests run
both on a real two-process gloo group; the row-shard test stands the oracle in
for the three device calls, since this machine has no GPU, and checks the
collective step and the order of the calls.
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


def _row_shard_worker(rank, world, port, out):
    import numpy as np
    import phase_disaggregated_quantized_b200 as nvq
    from oracle import nvfp4 as onv
    from phase_disaggregated_quantized_b200 import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = synth.activations(256, 128, seed=5, n_outliers=2)
        x[:128] = 0                                   # rank 0's rows are all zero: its own t would be 1
        mine = x[128 * rank:128 * (rank + 1)].contiguous()
        f64 = lambda t: onv.bf16_bits_to_f64(t.contiguous().view(torch.int16).numpy().view(np.uint16))
        calls = []

        def fake_amax(xl, **kw):
            calls.append("amax")
            a = f64(xl)
            return torch.tensor([float(np.max(np.abs(a))) if a.size else 0.0], dtype=torch.float32)

        def fake_scale(amax, **kw):
            calls.append("scale")
            return torch.tensor([onv.tensor_scale_from_amax(float(amax.item()))], dtype=torch.float32)

        def fake_quantize(xl, t, **kw):
            calls.append("quantize")
            codes, s, tt = onv.quantize(f64(xl), t_in=float(t.item()))
            return onv.pack_codes(codes), s, tt

        nvq.nvfp4_amax, nvq.nvfp4_scale_from_amax, nvq.nvfp4_quantize = fake_amax, fake_scale, fake_quantize
        codes, s, t = nvq.nvfp4_quantize_row_shard(mine)
        whole_codes, whole_s, whole_t = onv.quantize(f64(x))
        out[rank] = (calls, t, whole_t, bool((codes == onv.pack_codes(whole_codes)[128 * rank:128 * (rank + 1)]).all()),
                     bool((s == whole_s[128 * rank:128 * (rank + 1)]).all()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_row_shard_quantize_uses_the_whole_tensor_scale():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_row_shard_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    for rank in range(world):
        calls, t, whole_t, codes_ok, scales_ok = out[rank]
        assert calls == ["amax", "scale", "quantize"]
        assert t == whole_t != 1.0                  # the zero shard took the other rank's amax, not t = 1
        assert codes_ok and scales_ok
