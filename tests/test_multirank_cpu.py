"""Multi-rank host logic of the benchmark on CPU with two gloo ranks: every rank solves an
independent problem (no data-path collective); the step time is the max over ranks and the
whole-job value counts the work of all ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, step_ms, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(step_ms[rank], dist, "cpu")
        value, tmax = bench.aggregate([t] * world, 1e12)
        q.put((rank, t, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    world = 2
    step_ms = [10.0, 12.5]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, step_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, t, value in got:
        assert t == pytest.approx(12.5)
        # 2 ranks x 1 TFLOP in 12.5 ms = 160 TFLOP/s
        assert value == pytest.approx(2 * 1e12 / 12.5e-3 / 1e12)


def test_aggregate_single_rank():
    v, t = bench.aggregate([20.0], 1e12)
    assert t == 20.0 and v == pytest.approx(50.0)
    assert bench.max_over_ranks(3.0) == 3.0
