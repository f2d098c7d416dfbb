"""Multi-rank host logic of the benchmark on CPU: two gloo ranks on 127.0.0.1.

The path is data parallel (each rank quantises and multiplies its own token batch
against the same weights; no collective on the data path), so what spans ranks is
the timing: the max over ranks, and whole-job throughput = all ranks' work / that
time (weak scaling).
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, r, local = bench.dist_setup()
        # rank-dependent timings: the slowest rank decides every figure
        vals = [10.0 + rank, 5.0 - rank, 1.0 + 0.5 * rank]
        got = bench.reduce_max(vals)
        # each rank's batch is its own seeded draw
        x = synth.activations(4, 256, seed=rank)
        xs = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(xs, x)
        distinct = not torch.equal(xs[0].view(torch.int16), xs[1].view(torch.int16))
        q.put((rank, (w, r, local), got, distinct))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, env, got, distinct in res:
        assert env == (world, rank, rank)
        assert got == [11.0, 5.0, 1.5]
        assert distinct


def test_single_process_identity():
    assert not dist.is_initialized()
    assert bench.reduce_max([3.0, 1.0]) == [3.0, 1.0]


@pytest.mark.parametrize("world", [1, 2, 8])
def test_weak_scaling_value(world):
    # 2*M*N*K per rank-step; 10 steps in 9 ms on every rank
    fl = 2.0 * 4096 * 28672 * 8192
    v = bench.weak_scaling_tflops(fl, world, 10, 9.0)
    assert v == pytest.approx(fl * world * 10 / 9e-3 / 1e12)
    assert bench.weak_scaling_tflops(fl, world, 10, 9.0) == pytest.approx(world * bench.weak_scaling_tflops(fl, 1, 10, 9.0))
