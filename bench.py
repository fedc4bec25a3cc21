"""Benchmark of 3D Deformable Slide Attention on B200: effective TFLOP/s and the fraction of
the dense bf16 tensor peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl dsa|reference]

A step is one pass of the whole hot path over one batch of synthetic input: the window
planner and the forward kernel (dsa_fwd), plus the backward (dsa_bwd) for workloads with
a backward.  Effective FLOP per step = 4 * B * heads * N * keys_per_query * d forward,
2.5x that backward.  Inputs (2.1 GB for the 720p-shaped workload) are larger than the
126 MB L2, so no flush is needed between steps.  Multi-GPU (torchrun, one rank per GPU):
every rank solves its own independent problem of the same shape (weak scaling, no
data-path collective); the step time is the max over ranks.

Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle instead, on a
bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dsa_inputs import WORKLOADS, Workload, make_inputs, make_text_inputs, text_length  # noqa: E402

METRIC = "3D-DSA fwd/bwd effective TFLOP/s and % of B200 dense BF16 peak"
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_BF16_TFLOPS = 1590.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# ----------------------------------------------------------------------------- DRAM traffic
# DRAM bytes (read + write) of one fwd_bf16_kernel launch per workload, from a
# single-pass ncu capture (dram__bytes_read.sum + dram__bytes_write.sum) of the full-size
# launch.  The figure holds only for the kernel sources it was taken on, identified by a
# hash of them; with any other sources the line reports null.
FWD_TRAFFIC = {"bf16_720p": (3.40e9, "26f42e3c38a0249f")}
FWD_SOURCES = ("dsa_fwd_bf16.cuh", "sm100.cuh")


def fwd_source_hash() -> str:
    import hashlib

    h = hashlib.sha256()
    for name in FWD_SOURCES:
        with open(os.path.join(ROOT, "video_dit_sparse_dsa_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def fwd_traffic(workload: str):
    entry = FWD_TRAFFIC.get(workload)
    if entry is None:
        return None
    try:
        return entry[0] if fwd_source_hash() == entry[1] else None
    except OSError:
        return None


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clocks, power and throttle reasons with nvidia-smi every 20 ms; stop()
    keeps only the samples taken inside the timed regions (TIMED_WINDOWS, host wall-clock
    intervals around each CUDA-event-timed loop)."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    @staticmethod
    def parse(lines):
        """-> list of (epoch seconds, sm MHz, max sm MHz, power W, set of active reasons)."""
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        out = []
        for line in lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                t = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, smax = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            try:
                pw = float(parts[3])
            except ValueError:
                pw = None
            reasons = {n for n, v in zip(names, parts[4:8]) if v.lower().startswith("active")}
            out.append((t, sm, smax, pw, reasons))
        return out

    def stop(self, windows):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        return summarise_clocks(self.parse(self.lines), windows)


def summarise_clocks(rows, windows):
    """Median SM clock and power, max clock and the union of active reasons over the samples
    (epoch seconds, sm MHz, max sm MHz, power W, reasons) inside the timed windows."""
    inside = [r for r in rows if any(a <= r[0] <= b for a, b in windows)]
    use = inside if inside else rows
    power = [r[3] for r in use if r[3] is not None]
    return {"sm_mhz": statistics.median(r[1] for r in use) if use else None,
            "sm_max_mhz": max(r[2] for r in use) if use else None,
            "power_w": statistics.median(power) if power else None,
            "samples": len(use), "in_timed_region": bool(inside),
            "reasons": sorted(set().union(*[r[4] for r in use])) if use else []}


class NvmlSampler:
    """Samples the SM clock, power and throttle reasons through NVML (read-only queries)
    every 2 ms from a thread, so that even a timed region of a tenth of a second holds
    dozens of samples; same stop() result as ClockSampler."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, nvml, handle, period_s: float = 0.002):
        self.nvml, self.handle, self.period = nvml, handle, period_s
        self.rows = []
        self.stop_flag = threading.Event()
        self.thread = None

    @classmethod
    def for_device(cls, device_index: int):
        """The sampler of the CUDA device (matched by UUID, then PCI bus id), or None."""
        try:
            import pynvml as nvml

            nvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            handle = None
            try:
                uuid = str(props.uuid)
                handle = nvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                handle = nvml.nvmlDeviceGetHandleByPciBusId(bus)
            return cls(nvml, handle)
        except Exception:
            return None

    def _sample(self):
        n = self.nvml
        smax = n.nvmlDeviceGetMaxClockInfo(self.handle, n.NVML_CLOCK_SM)
        while not self.stop_flag.is_set():
            try:
                t = time.time()
                sm = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
                pw = n.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                reasons = {name for name, attr in self.REASONS if mask & getattr(n, attr, 0)}
                self.rows.append((t, float(sm), float(smax), pw, reasons))
            except Exception:
                pass
            self.stop_flag.wait(self.period)

    def start(self):
        self.thread = threading.Thread(target=self._sample, daemon=True)
        self.thread.start()

    def stop(self, windows):
        self.stop_flag.set()
        if self.thread:
            self.thread.join(timeout=2)
        out = summarise_clocks(list(self.rows), windows)
        out["source"] = "nvml"
        return out


# host wall-clock intervals of the CUDA-event-timed loops of the headline workload
TIMED_WINDOWS = []


# ----------------------------------------------------------------------------- inputs
def host_inputs(w: Workload, rank: int = 0):
    """The seeded inputs of the parity tests (dsa_inputs, drawn on the CPU); rank r > 0 of a
    multi-GPU run draws its own independent problem of the same shape from seed + r."""
    return make_inputs(w, seed=w.seed + rank) if rank else make_inputs(w)


def device_inputs(w: Workload, device, rank: int = 0):
    inp = host_inputs(w, rank)
    dout = inp.dout.to(device) if inp.dout is not None else None
    return inp.q.to(device), inp.k.to(device), inp.v.to(device), dout, inp.offsets.to(device), inp


# ----------------------------------------------------------------------------- GPU arm
def time_steps(step, steps: int, warmup: int, stream, record: bool = True):
    """W untimed steps, then K steps each between two CUDA events on `stream`, with a
    synchronize before and after.  Returns {median, mean, min, max} ms per step."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    t0 = time.time()
    ev[0].record(stream)
    for i in range(steps):
        step()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    if record:
        TIMED_WINDOWS.append((t0, time.time()))
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    return {"median": statistics.median(per), "mean": ev[0].elapsed_time(ev[steps]) / steps, "min": min(per),
            "max": max(per)}


def pct_of_peaks(tflops: float) -> dict:
    burst, sustained, src = peaks()
    return {"pct_nominal_2250": 100 * tflops / NOMINAL_BF16_TFLOPS, f"pct_{src}_burst": 100 * tflops / burst}


def run_workload(dsa, w: Workload, device, steps: int, warmup: int, rank: int = 0, with_e2e: bool = False,
                 record: bool = True):
    """Times the forward (planner + kernel, one dsa_fwd call) and, for workloads with a
    backward, the backward (one dsa_bwd call) on the workload's seeded inputs.  Times are
    medians over `steps` timed steps after `warmup` untimed ones."""
    stream = torch.cuda.current_stream(device)
    q, k, v, dout, off, host = device_inputs(w, device, rank)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:5], dtype=torch.float32, device=device)
    p = dsa.make_problem(w.B, w.heads, w.d, w.grid, w.tile, w.window, w.scale,
                         dsa.DSA_BF16 if w.dtype == "bf16" else dsa.DSA_F32)
    ws_f = dsa.workspace(p, device)
    res = {}

    def fwd():
        dsa.forward(q, k, v, off, w.tile, w.window, w.scale, out=out, lse=lse, ws=ws_f, stream=stream)

    fwd()
    t = time_steps(fwd, steps, warmup, stream, record)
    res["fwd_ms"] = t["median"]
    res["fwd_ms_mean"] = t["mean"]
    res["fwd_tflops"] = w.fwd_flops() / (res["fwd_ms"] * 1e-3) / 1e12
    launches = dsa.FWD_LAUNCHES
    step_ms = res["fwd_ms"]
    step_ms_mean = t["mean"]
    step_flops = w.fwd_flops()
    if w.backward:
        ws_b = dsa.workspace(p, device, backward=True)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)

        def bwd():
            dsa.backward(q, k, v, out, lse, dout, off, w.tile, w.window, w.scale, dq=dq, dk=dk, dv=dv, ws=ws_b,
                         stream=stream)

        bwd()
        t = time_steps(bwd, steps, warmup, stream, record)
        res["bwd_ms"] = t["median"]
        res["bwd_ms_mean"] = t["mean"]
        res["bwd_tflops"] = w.bwd_flops() / (res["bwd_ms"] * 1e-3) / 1e12
        step_ms += res["bwd_ms"]
        step_ms_mean += t["mean"]
        step_flops += w.bwd_flops()
        launches += dsa.BWD_LAUNCHES
    res["step_ms"] = step_ms
    res["step_ms_mean"] = step_ms_mean
    res["step_flops"] = step_flops
    res["launches_per_step"] = launches
    st = dsa.device_status(stream)
    if st[0] != 0:
        raise RuntimeError(f"device status {st} after {w.name}")
    if with_e2e:
        res["e2e"] = run_e2e(dsa, w, p, host, device, steps, warmup, stream)
    return res


def run_list_workload(dsa, w: Workload, device, steps: int, warmup: int, n_keep: int):
    """Block-sparse form on the grid of w: every (batch, head, query tile) keeps n_keep key
    tiles chosen at random (seeded) from the whole tile grid, as per-head key-tile lists
    (head-adaptive block masks); the forward's FLOPs count n_keep tiles per query."""
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    q, k, v, _, _, _ = device_inputs(w, device)
    BH = w.B * w.heads
    g = torch.Generator(device=device).manual_seed(7000 + w.seed)
    pick = torch.rand((BH, w.n_tiles, w.n_tiles), generator=g, device=device).argsort(dim=-1)[..., :n_keep]
    kv_list = pick.sort(dim=-1).values.to(torch.int32).reshape(-1).contiguous()
    row_ptr = (torch.arange(BH * (w.n_tiles + 1), device=device, dtype=torch.int64).reshape(BH, w.n_tiles + 1)
               - torch.arange(BH, device=device, dtype=torch.int64)[:, None])
    row_ptr = (row_ptr * n_keep).to(torch.int32).contiguous()
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:5], dtype=torch.float32, device=device)

    def fwd():
        dsa.forward_list(q, k, v, row_ptr, kv_list, w.tile, w.scale, out=out, lse=lse, stream=stream)

    fwd()
    ms = time_steps(fwd, steps, warmup, stream, record=False)["median"]
    flops = 4.0 * w.B * w.heads * w.n_tokens * (n_keep * w.tile_tokens) * w.d
    st = dsa.device_status(stream)
    if st[0] != 0:
        raise RuntimeError(f"device status {st} after the key-tile-list forward")
    return {"fwd_ms": ms, "fwd_tflops": flops / (ms * 1e-3) / 1e12, "keys_per_query": n_keep * w.tile_tokens}


def run_prefix_workload(dsa, w: Workload, device, steps: int, warmup: int):
    """Text prefix on the grid of w: about 1% of the sequence as text tokens, which attend to
    and are attended by every token; the video-video part keeps its windows.  FLOPs:
    4 * B * heads * d * (N * keys_per_query + 2 * N * L_text + L_text^2)."""
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    q, k, v, _, offsets, _ = device_inputs(w, device)
    L = text_length(w)
    txt = make_text_inputs(w, L, seed=1000 + w.seed)
    qt, kt, vt = (t.to(device) for t in (txt.q, txt.k, txt.v))
    p = dsa._problem_of(q, w.tile, w.window, w.scale)
    ws = torch.empty(dsa.prefix_workspace_size(p, L), dtype=torch.uint8, device=device)

    def fwd():
        dsa.forward_prefix(q, k, v, offsets, qt, kt, vt, w.tile, w.window, w.scale, ws=ws, stream=stream)

    fwd()
    ms = time_steps(fwd, steps, warmup, stream, record=False)["median"]
    st = dsa.device_status(stream)
    if st[0] != 0:
        raise RuntimeError(f"device status {st} after the text-prefix forward")
    N = w.n_tokens
    flops = 4.0 * w.B * w.heads * w.d * (N * w.keys_per_query + 2.0 * N * L + float(L) * L)
    res = {"fwd_ms": ms, "fwd_tflops": flops / (ms * 1e-3) / 1e12, "L_text": L}
    # backward of the same call (2.5x the forward's FLOPs), dO drawn like the inputs
    out, lse, out_t, lse_t = dsa.forward_prefix(q, k, v, offsets, qt, kt, vt, w.tile, w.window, w.scale, ws=ws,
                                                stream=stream)
    g = torch.Generator(device=device).manual_seed(9000 + w.seed)
    do = torch.randn(q.shape, generator=g, device=device, dtype=torch.float32).to(q.dtype)
    do_t = torch.randn(qt.shape, generator=g, device=device, dtype=torch.float32).to(q.dtype)
    ws_b = torch.empty(dsa.prefix_bwd_workspace_size(p, L), dtype=torch.uint8, device=device)

    def bwd():
        dsa.backward_prefix(q, k, v, out, lse, do, offsets, qt, kt, vt, out_t, lse_t, do_t, w.tile, w.window, w.scale,
                            ws=ws_b, stream=stream)

    bwd()
    b_ms = time_steps(bwd, steps, warmup, stream, record=False)["median"]
    st = dsa.device_status(stream)
    if st[0] != 0:
        raise RuntimeError(f"device status {st} after the text-prefix backward")
    res.update({"bwd_ms": b_ms, "bwd_tflops": 2.5 * flops / (b_ms * 1e-3) / 1e12})
    return res


def run_dense_map_workload(dsa, w: Workload, device, steps: int, warmup: int):
    """Dense attention on the grid of w (every tile listed for every query tile) and its
    block attention mass: times the dense forward and the map pass separately.  The map
    pass recomputes the scores only: 2 * B * heads * N^2 * d FLOP."""
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    q, k, v, _, _, _ = device_inputs(w, device)
    n = w.n_tiles
    row_ptr = torch.arange(n + 1, dtype=torch.int32, device=device) * n
    kv_list = torch.arange(n, dtype=torch.int32, device=device).repeat(n).contiguous()
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:5], dtype=torch.float32, device=device)
    bmap = torch.empty((w.B * w.heads, n, n), dtype=torch.float32, device=device)

    def fwd():
        dsa.forward_list(q, k, v, row_ptr, kv_list, w.tile, w.scale, out=out, lse=lse, stream=stream)

    def bm():
        dsa.block_map(q, k, lse, row_ptr, kv_list, w.tile, w.scale, out=bmap, stream=stream)

    fwd()
    bm()
    f_ms = time_steps(fwd, steps, warmup, stream, record=False)["median"]
    m_ms = time_steps(bm, steps, warmup, stream, record=False)["median"]
    st = dsa.device_status(stream)
    if st[0] != 0:
        raise RuntimeError(f"device status {st} after the dense map")
    pairs = float(w.B * w.heads) * w.n_tokens * w.n_tokens
    return {"fwd_ms": f_ms, "fwd_tflops": 4.0 * pairs * w.d / (f_ms * 1e-3) / 1e12,
            "map_ms": m_ms, "map_tflops": 2.0 * pairs * w.d / (m_ms * 1e-3) / 1e12}


def run_lstsq_workload(dsa, device, steps: int, warmup: int, m: int = 300 * 300, p: int = 3, batch: int = 24):
    """Pattern intensities of the 720p block maps: m = 300 x 300 map entries, p = 3 bases,
    one map per head (batch 24); the factor is computed once, the solve is timed.  Bound:
    HBM, reading S once (batch * m * 4 bytes) plus M (m * p * 4 bytes).  One solve is a
    single launch of a few microseconds, shorter than a host call through the binding, so
    it is timed as a CUDA graph of `reps` solves replayed (device time per solve), beside
    the rate of direct calls (bound by the host)."""
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    g = torch.Generator(device=device).manual_seed(123)
    M = torch.rand((m, p), generator=g, device=device)
    S = torch.rand((batch, m), generator=g, device=device)
    L = dsa.lstsq_factor(M, 1e-3, stream=stream)
    X = torch.empty((batch, p), dtype=torch.float32, device=device)

    def solve(s=stream):
        dsa.lstsq_solve(M, L, S, X=X, stream=s)

    solve()
    host_ms = time_steps(solve, steps, warmup, stream, record=False)["median"]
    reps = 20
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        solve(side)
    stream.wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for _ in range(reps):
            solve(side)
    ms = time_steps(graph.replay, steps, warmup, stream, record=False)["median"] / reps
    del graph
    # reference: a library reduction reading the same bytes (S and M once), timed the same way
    acc = torch.empty((), dtype=torch.float32, device=device)

    def read(s=stream):
        with torch.cuda.stream(s):
            acc.copy_(S.sum() + M.sum())

    with torch.cuda.stream(side):
        read(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for _ in range(reps):
            read(side)
    read_ms = time_steps(graph.replay, steps, warmup, stream, record=False)["median"] / reps
    del graph
    st = dsa.device_status(stream)
    if st[0] != 0:
        raise RuntimeError(f"device status {st} after the least-squares solve")
    gb = (batch * m + m * p) * 4 / 1e9
    return {"solve_ms": ms, "solve_gbs": gb / (ms * 1e-3), "solve_ms_host_call": host_ms,
            "read_same_bytes_ms": read_ms, "read_same_bytes_gbs": gb / (read_ms * 1e-3),
            "timing": f"CUDA graph of {reps} solves, device time per solve; read_same_bytes: torch sums of S "
                      f"and M in the same graph form"}


def run_e2e(dsa, w, p, host, device, steps, warmup, stream):
    """Same forward through the host-buffer entry point: H2D of q, k, v, offsets from pinned
    memory, planner + forward, D2H of out and lse, all inside the timed region."""
    qh, kh, vh = host.q.pin_memory(), host.k.pin_memory(), host.v.pin_memory()
    oh_ = host.offsets.pin_memory()
    outh = torch.empty_like(qh).pin_memory()
    lseh = torch.empty(qh.shape[:5], dtype=torch.float32).pin_memory()
    dev = torch.empty(dsa.forward_host_bytes(p), dtype=torch.uint8, device=device)

    def step():
        dsa.forward_host(p, qh, kh, vh, oh_, outh, lseh, dev, stream=stream)

    ms = time_steps(step, max(1, steps // 2), max(1, warmup // 2), stream, record=False)["median"]
    h2d = 3 * qh.numel() * qh.element_size() + oh_.numel() * 4
    d2h = outh.numel() * outh.element_size() + lseh.numel() * 4
    return {"value": w.fwd_flops() / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


# ----------------------------------------------------------------------------- oracle timing
def _slice0(w: Workload, host):
    """(workload of one (batch, head), its tensors): the first slice of the inputs the GPU ran."""
    one = w.replace(B=1, heads=1)
    sl = [None if t is None else t[:1, :1].contiguous() for t in (host.q, host.k, host.v, host.dout)]
    return one, sl


def _grow(run, n_max: int, target_s: float):
    """Calls run(n) with growing n (1, then scaled up to reach target_s) until one call takes
    at least target_s or n reaches n_max.  Returns (n, seconds of that call)."""
    n = 1
    while True:
        t0 = time.perf_counter()
        run(n)
        dt_s = time.perf_counter() - t0
        if dt_s >= target_s or n >= n_max:
            return n, dt_s
        n = min(n_max, max(n + 1, int(n * min(8.0, 1.2 * target_s / max(dt_s, 1e-3)))))


def oracle_fwd_rate(w: Workload, host, target_s: float):
    """The fp64 oracle (as it stands) timed on the query tiles of the first (batch, head)
    slice of the GPU's inputs, in raster order: growing samples until one run takes
    target_s, or the whole slice.  Returns a cpu_baseline object (TFLOP/s)."""
    import oracle

    one, (q, k, v, _) = _slice0(w, host)
    geo = oracle.Geometry.of(one)
    per_tile = 4.0 * w.tile_tokens * w.keys_per_query * w.d

    def run(n):
        oracle.forward_tiles(geo, q, k, v, host.offsets, (np.zeros(n, np.int32), np.arange(n, dtype=np.int32)))

    n, secs = _grow(run, geo.n_tiles, target_s)
    whole = n == geo.n_tiles
    return {"value": per_tile * n / secs / 1e12, "unit": "TFLOP/s", "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle", "seconds": secs, "extrapolated": not whole,
            "sample": ("the whole first (batch, head) slice" if whole else
                       f"query tiles 0..{n - 1} of {geo.n_tiles} of the first (batch, head) slice") +
                      f" ({n * w.tile_tokens} query rows), forward, {secs:.1f} s"}


def oracle_bwd_rate(w: Workload, host, target_s: float):
    """The fp64 oracle's backward timed on query tiles 0..n-1 (dQ) and key tiles 0..n-1
    (dK, dV) of the first (batch, head) slice, n grown until one run takes target_s.  Its
    effective FLOP: 2.5 x 4d x (query-key pairs of the dQ sample + pairs of the dK/dV
    sample) / 2, since every pair of the full backward is counted once for dQ and once for
    dK, dV."""
    import oracle

    one, (q, k, v, do) = _slice0(w, host)
    geo = oracle.Geometry.of(one)
    _, _, row_ptr, _ = oracle.plan(geo.G, geo.window, host.offsets)
    indeg = np.diff(row_ptr)
    tt = w.tile_tokens

    def run(n):
        sel = (np.zeros(n, np.int32), np.arange(n, dtype=np.int32))
        oracle.backward_dq_tiles(geo, q, k, v, do, host.offsets, sel)
        oracle.backward_dkdv_tiles(geo, q, k, v, do, host.offsets, sel)

    n, secs = _grow(run, geo.n_tiles, target_s)
    pairs = n * tt * w.keys_per_query + int(indeg[:n].sum()) * tt * tt
    return {"value": 2.5 * 4.0 * w.d * pairs / 2 / secs / 1e12, "unit": "TFLOP/s",
            "cores": len(os.sched_getaffinity(0)), "kind": "oracle", "seconds": secs, "extrapolated": True,
            "sample": f"dQ of query tiles 0..{n - 1} and dK, dV of key tiles 0..{n - 1} of {geo.n_tiles}, first "
                      f"(batch, head) slice, backward, {secs:.1f} s"}


def workload_config(w: Workload, world: int) -> dict:
    """The `config` object of both arms' JSON lines."""
    return {"workload": w.name, "B": w.B, "heads": w.heads, "d": w.d, "grid": list(w.grid), "tile": list(w.tile),
            "window": list(w.window), "offsets": list(w.offset_range), "keys_per_query": w.keys_per_query,
            "dtype": w.dtype, "pass": "fwd+bwd" if w.backward else "fwd",
            "l2": "inputs larger than L2 (no flush)" if 3 * w.B * w.heads * w.n_tokens * w.d * 2 > 126e6 else
                  "inputs smaller than L2 (no flush; L2-resident)",
            "inputs": "dsa_inputs seeded CPU draws (the parity tests' inputs)",
            "parallelism": f"independent problem per rank x{world}"}


def reference_arm(args, w: Workload):
    """The oracle as it stands on the host cores: each step is a bounded sample of the
    workload (forward query tiles, plus the backward sample for workloads with one), and the
    line's ms_per_step is the measured time of one such sample step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    host = host_inputs(w.replace(B=1, heads=1))
    per_step = max(0.5, min(5.0, 150.0 / max(1, args.steps + args.warmup)))
    rates, secs = [], []
    fwd = bwd = None
    for i in range(args.warmup + args.steps):
        fwd = oracle_fwd_rate(w, host, per_step)
        t = fwd["seconds"]
        r = fwd["value"]
        if w.backward:
            bwd = oracle_bwd_rate(w, host, per_step)
            t += bwd["seconds"]
            # the step's rate: fwd + bwd effective FLOP of the samples over their time
            r = (fwd["value"] * fwd["seconds"] + bwd["value"] * bwd["seconds"]) / t
        if i >= args.warmup:
            rates.append(r)
            secs.append(t)
    value = statistics.median(rates)
    flops = w.fwd_flops() + (w.bwd_flops() if w.backward else 0)
    sample = fwd["sample"] + ("; " + bwd["sample"] if bwd else "")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.median(secs) * 1e3,
            "ms_per_step_is": "measured time of one bounded sample step (not the whole workload)",
            "full_workload_ms_extrapolated": flops / (value * 1e12) * 1e3, "extrapolated": True,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": fwd["cores"], "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- main
def aggregate(per_rank_ms, flops_per_rank):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    t = max(per_rank_ms)
    return len(per_rank_ms) * flops_per_rank / (t * 1e-3) / 1e12, t


def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """Max of a per-rank scalar over all ranks (every rank gets it); identity without a
    process group."""
    if dist is None:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="bf16_720p", choices=list(WORKLOADS))
    ap.add_argument("--impl", default="dsa", choices=["dsa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the per-workload table")
    ap.add_argument("--extra-only", choices=["text_prefix", "lists", "dense_map", "lstsq"],
                    help="run one entry of the per-workload table on the workload alone and print it (profiling)")
    ap.add_argument("--batch", type=int, help="run the workload with this batch size instead (profiling captures)")
    ap.add_argument("--heads", type=int, help="run the workload with this many heads instead (profiling captures)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = WORKLOADS[args.workload]
    if args.batch or args.heads:  # a reduced copy of the workload, named for what it is
        w = w.replace(B=args.batch or w.B, heads=args.heads or w.heads)
        w = w.replace(name=f"{args.workload}_B{w.B}_h{w.heads}")
    if args.impl == "reference":
        reference_arm(args, w)
        return

    import video_dit_sparse_dsa_b200 as dsa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = None
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    dsa.load_library()
    if args.extra_only:
        if world > 1:
            raise SystemExit("--extra-only runs on one GPU")
        runs = {"text_prefix": lambda: run_prefix_workload(dsa, w, device, args.steps, args.warmup),
                "lists": lambda: run_list_workload(dsa, w, device, args.steps, args.warmup, w.window_tiles),
                "dense_map": lambda: run_dense_map_workload(dsa, w, device, args.steps, args.warmup),
                "lstsq": lambda: run_lstsq_workload(dsa, device, args.steps, args.warmup)}
        print(json.dumps({"extra": args.extra_only, "workload": w.name, **runs[args.extra_only]()}), flush=True)
        return

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    sampler = None
    if rank == 0:
        sampler = NvmlSampler.for_device(device.index if device.index is not None else 0) or ClockSampler(local)
    barrier()
    if sampler:
        sampler.start()
    res = run_workload(dsa, w, device, args.steps, args.warmup, rank=rank, with_e2e=True)
    barrier()
    timed = list(TIMED_WINDOWS)
    clocks = sampler.stop(timed) if sampler else None
    step_ms = max_over_ranks(res["step_ms"], dist, device)
    step_ms_mean = max_over_ranks(res["step_ms_mean"], dist, device)
    value, _ = aggregate([step_ms] * world, res["step_flops"])

    # every rank runs the host-buffer path on its own problem: whole-job rate over the slowest
    e2e_ms = max_over_ranks(res["e2e"]["ms_per_step"], dist, device)
    e2e = None
    extra = {}
    cpu = None
    if rank == 0:
        e2e = dict(res["e2e"])
        e2e["ms_per_step"] = e2e_ms
        e2e["value"] = aggregate([e2e_ms] * world, w.fwd_flops())[0]
    # the per-workload table (every configuration, each with the oracle timed beside it on
    # this machine's host cores) and the CPU baseline run at N = 1 only (the scaling runs time the
    # headline workload alone, and the other ranks do not wait at a barrier meanwhile)
    if rank == 0 and world == 1 and not args.no_extra:
        for name, ow in WORKLOADS.items():
            try:
                r = res if name == w.name else run_workload(dsa, ow, device, max(20, args.steps),
                                                            max(5, args.warmup), record=False)
                row = {k2: round(v2, 4) for k2, v2 in r.items() if k2.endswith("_ms") or k2.endswith("_tflops")
                       or k2.endswith("_ms_mean")}
                row["steps"], row["warmup"] = max(20, args.steps), max(5, args.warmup)
                row["fwd_pct"] = {k2: round(v2, 2) for k2, v2 in pct_of_peaks(r["fwd_tflops"]).items()}
                if "bwd_tflops" in r:
                    row["bwd_pct"] = {k2: round(v2, 2) for k2, v2 in pct_of_peaks(r["bwd_tflops"]).items()}
                if not args.no_cpu_baseline:
                    host = host_inputs(ow.replace(B=1, heads=1))
                    row["oracle_fwd"] = oracle_fwd_rate(ow, host, 12.0 if name == w.name else 6.0)
                    if name == w.name:
                        cpu = dict(row["oracle_fwd"])
                    if ow.backward:
                        row["oracle_bwd"] = oracle_bwd_rate(ow, host, 8.0)
                extra[name] = row
            except Exception as e:  # report, do not hide: the line carries the error
                extra[name] = {"error": str(e)}
        try:
            r = run_lstsq_workload(dsa, device, max(20, args.steps), 5)
            extra["lstsq_24x90000x3"] = {k2: (round(v2, 5) if isinstance(v2, float) else v2) for k2, v2 in r.items()}
        except Exception as e:
            extra["lstsq_24x90000x3"] = {"error": str(e)}
        dense = WORKLOADS.get("bf16_16x32x32")
        if dense is not None:
            try:
                r = run_dense_map_workload(dsa, dense, device, max(20, args.steps), 5)
                extra["bf16_16x32x32_dense_map"] = {k2: round(v2, 4) for k2, v2 in r.items()}
            except Exception as e:
                extra["bf16_16x32x32_dense_map"] = {"error": str(e)}
        if w.dtype == "bf16":
            name = f"{w.name}_lists{w.window_tiles}"
            try:
                r = run_list_workload(dsa, w, device, max(20, args.steps), 5, w.window_tiles)
                extra[name] = {k2: (round(v2, 4) if isinstance(v2, float) else v2) for k2, v2 in r.items()}
            except Exception as e:
                extra[name] = {"error": str(e)}
            name = f"{w.name}_text_prefix"
            try:
                r = run_prefix_workload(dsa, w, device, max(20, args.steps), 5)
                extra[name] = {k2: (round(v2, 4) if isinstance(v2, float) else v2) for k2, v2 in r.items()}
            except Exception as e:
                extra[name] = {"error": str(e)}
    elif rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_fwd_rate(w, host_inputs(w.replace(B=1, heads=1)), 12.0)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    burst, sustained, src = peaks()
    fwd_tflops = res["fwd_tflops"]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "ms_per_step_mean": step_ms_mean,
        "timing": "median of the per-step CUDA-event times of the timed steps (max over ranks)",
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": workload_config(w, world),
        "pct_of_peak": {"nominal_2250": 100 * fwd_tflops / NOMINAL_BF16_TFLOPS,
                        f"{src}_{burst:g}": 100 * fwd_tflops / burst},
        "roofline": {"bound": "tensor", "kernel": "fwd_bf16_kernel (timed with the planner, one dsa_fwd call)",
                     "achieved": fwd_tflops, "peak": burst, "peak_kind": f"{src} burst bf16", "unit": "TFLOP/s",
                     "frac": fwd_tflops / burst, "traffic": fwd_traffic(w.name), "traffic_unit": "bytes per launch",
                     "peak_sustained": sustained, "frac_sustained": fwd_tflops / sustained},
        "e2e": e2e, "gpu_launches": res["launches_per_step"] * args.steps, "clocks": clocks,
        "cpu_baseline": cpu, "workloads": extra,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
