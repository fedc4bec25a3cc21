"""Multi-rank host logic on CPU with gloo ranks: in the benchmark every rank solves an
independent problem (no data-path collective), the step time is the max over ranks and the
whole-job value counts the work of all ranks; one problem split over ranks by (batch, head)
slices reassembles exactly."""
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


def test_clock_samples_are_kept_only_inside_timed_windows():
    """The benchmark's clock summary uses only nvidia-smi samples taken while a timed loop ran."""
    import datetime

    def line(t, sm, pw, cap):
        ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"{ts}, {sm}, 1965, {pw}, Not Active, Not Active, Not Active, {'Active' if cap else 'Not Active'}"

    base = 1_800_000_000.0
    lines = [line(base + 0.0, 1965, 200.0, False), line(base + 1.0, 1400, 990.0, True),
             line(base + 1.1, 1420, 995.0, True), line(base + 2.0, 1965, 210.0, False), "garbage"]
    rows = bench.ClockSampler.parse(lines)
    assert len(rows) == 4 and rows[1][4] == {"sw_power_cap"}
    s = bench.ClockSampler(0)
    s.proc = None
    assert s.stop([(base + 0.5, base + 1.5)])["sm_mhz"] is None  # no sampler process: reported as unavailable

    class Done:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            pass

    s.proc, s.lines = Done(), lines
    got = s.stop([(base + 0.5, base + 1.5)])
    assert got["samples"] == 2 and got["in_timed_region"]
    assert got["sm_mhz"] == 1410 and got["reasons"] == ["sw_power_cap"] and got["power_w"] == 992.5


def test_traffic_is_reported_only_for_the_profiled_kernel_sources(monkeypatch):
    """The roofline's DRAM traffic is tied to the kernel sources it was measured on."""
    h = bench.fwd_source_hash()
    monkeypatch.setattr(bench, "FWD_TRAFFIC", {"w": (123.0, h), "stale": (5.0, "0" * 16)})
    assert bench.fwd_traffic("w") == 123.0
    assert bench.fwd_traffic("stale") is None
    assert bench.fwd_traffic("unknown") is None


def test_nvml_sampler_reads_reasons_from_a_fake_nvml():
    """The NVML sampler decodes the clock-event bitmask and keeps only timed-region samples."""
    import time as _time

    class FakeNvml:
        NVML_CLOCK_SM = 1
        nvmlClocksEventReasonSwPowerCap = 0x4
        nvmlClocksEventReasonHwSlowdown = 0x8
        nvmlClocksEventReasonSwThermalSlowdown = 0x20
        nvmlClocksEventReasonHwThermalSlowdown = 0x40
        nvmlClocksEventReasonHwPowerBrakeSlowdown = 0x80

        def nvmlDeviceGetMaxClockInfo(self, h, which):
            return 1965

        def nvmlDeviceGetClockInfo(self, h, which):
            return 1500

        def nvmlDeviceGetPowerUsage(self, h):
            return 990_000

        def nvmlDeviceGetCurrentClocksEventReasons(self, h):
            return 0x4 | 0x1  # power cap and idle (idle is not a slowdown reason)

    s = bench.NvmlSampler(FakeNvml(), handle=None, period_s=0.001)
    t0 = _time.time()
    s.start()
    _time.sleep(0.05)
    got = s.stop([(t0, _time.time())])
    assert got["samples"] > 5 and got["in_timed_region"]
    assert got["sm_mhz"] == 1500 and got["sm_max_mhz"] == 1965 and got["power_w"] == 990.0
    assert got["reasons"] == ["sw_power_cap"] and got["source"] == "nvml"


def test_head_range_covers_every_slice_once():
    import video_dit_sparse_dsa_b200 as dsa

    for n in (1, 2, 5, 24, 48):
        for world in (1, 2, 3, 4, 8):
            ranges = [dsa.head_range(n, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [hi - lo for lo, hi in ranges]
            assert max(sizes) - min(sizes) <= 1


def _head_split_worker(rank, world, port, q):
    # one OpenMP thread: the oracle's dK, dV sums then run in one fixed order, so results
    # can be compared bit for bit (torch shares the process's OpenMP runtime with the
    # oracle's library and sets its thread count)
    torch.set_num_threads(1)
    import numpy as np

    import oracle
    import video_dit_sparse_dsa_b200 as dsa
    from dsa_inputs import Workload, make_inputs

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = Workload("split", 2, 3, 16, (4, 4, 6), (2, 2, 2), (2, 1, 3), (-2, 2), "bf16", 71, backward=True)
        inp = make_inputs(w)
        BH = w.B * w.heads
        lo, hi = dsa.head_range(BH, rank, world)
        flat = lambda t: t.reshape((BH, 1) + tuple(w.grid) + (w.d,))[lo:hi]
        part = w.replace(B=hi - lo, heads=1)
        geo = oracle.Geometry.of(part)
        out, lse = oracle.forward(geo, flat(inp.q), flat(inp.k), flat(inp.v), inp.offsets)
        grads = oracle.backward(geo, flat(inp.q), flat(inp.k), flat(inp.v), flat(inp.dout), inp.offsets)
        # ranks hold different numbers of slices: pad to the longest, gather, trim
        most = -(-BH // world)
        pieces = []
        for a in (out, lse) + tuple(grads):
            a = torch.from_numpy(np.ascontiguousarray(a.reshape(hi - lo, -1)))
            pad = torch.zeros((most, a.shape[1]), dtype=a.dtype)
            pad[: hi - lo] = a
            got = [torch.zeros_like(pad) for _ in range(world)]
            dist.all_gather(got, pad)
            pieces.append(torch.cat([g[: dsa.head_range(BH, r, world)[1] - dsa.head_range(BH, r, world)[0]]
                                     for r, g in enumerate(got)]))
        if rank == 0:
            full = oracle.Geometry.of(w)
            ref_o, ref_l = oracle.forward(full, inp.q, inp.k, inp.v, inp.offsets)
            ref_g = oracle.backward(full, inp.q, inp.k, inp.v, inp.dout, inp.offsets)
            refs = [ref_o, ref_l] + list(ref_g)
            same = [bool(np.array_equal(p.numpy(), np.asarray(r).reshape(BH, -1))) for p, r in zip(pieces, refs)]
            q.put(same)
    finally:
        dist.destroy_process_group()


def test_one_problem_split_by_heads_over_two_gloo_ranks_reassembles_exactly():
    """Two gloo ranks each take their (batch, head) slices of one seeded problem, run the
    forward and backward oracle on them alone and gather the results: bit for bit the
    single-rank oracle's (slices are independent, so the split needs no other exchange)."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_head_split_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    assert q.get(timeout=5) == [True] * 5
