"""GPU forward (C ABI through the Python binding) against the fp64 oracle.

Small problems are compared element by element in full; the full-size workloads are
compared on sampled query tiles (every row of each sampled tile, including the first and
last tile of the grid), in the same launch configuration the benchmark times."""
import numpy as np
import pytest
import torch

import oracle
import video_dit_sparse_dsa_b200 as dsa
from dsa_inputs import WORKLOADS, Workload, make_inputs
from tests._parity import assert_close, assert_lse_close, errors

pytestmark = pytest.mark.gpu


def run_gpu(w: Workload, inp):
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    off = inp.offsets.cuda()
    out, lse = dsa.forward(q, k, v, off, w.tile, w.window, w.scale)
    st, site, block = dsa.device_status()
    assert st == 0, f"device status {st} at site {site} block {block}"
    return out, lse


def compare_full(w: Workload, inp, out, lse):
    geo = oracle.Geometry.of(w)
    ref, ref_lse = oracle.forward(geo, inp.q, inp.k, inp.v, inp.offsets)
    assert_close(out.float().cpu().numpy(), ref, w.dtype, "out")
    assert_lse_close(lse.cpu().numpy(), ref_lse, w.dtype)


def compare_sampled(w: Workload, inp, out, lse, n_samples=6, seed=0):
    geo = oracle.Geometry.of(w)
    rng = np.random.default_rng(seed)
    BH = w.B * w.heads
    bh = np.concatenate([[0, BH - 1], rng.integers(0, BH, n_samples)]).astype(np.int32)
    tiles = np.concatenate([[0, geo.n_tiles - 1], rng.integers(0, geo.n_tiles, n_samples)]).astype(np.int32)
    ref, ref_lse = oracle.forward_tiles(geo, inp.q, inp.k, inp.v, inp.offsets, (bh, tiles))
    tok = geo.tile_token_index()
    o = out.reshape(BH, geo.n_tokens, w.d)
    l = lse.reshape(BH, geo.n_tokens)
    idx_b = torch.as_tensor(np.repeat(bh, geo.tile_tokens), device=out.device, dtype=torch.long)
    idx_t = torch.as_tensor(tok[tiles].reshape(-1), device=out.device, dtype=torch.long)
    got = o[idx_b, idx_t].float().cpu().numpy().reshape(ref.shape)
    got_lse = l[idx_b, idx_t].cpu().numpy().reshape(ref_lse.shape)
    assert_close(got, ref, w.dtype, "out")
    assert_lse_close(got_lse, ref_lse, w.dtype)


def test_tiny_f32_full():
    w = WORKLOADS["tiny_f32"]
    inp = make_inputs(w)
    out, lse = run_gpu(w, inp)
    compare_full(w, inp, out, lse)


@pytest.mark.parametrize("d", [64, 128])
def test_f32_ragged_tiles_full(d):
    """fp32 path with a tile of 3x2x5 tokens (not a power of two) and clamped windows."""
    w = Workload("f32_odd", 2, 2, d, (6, 4, 10), (3, 2, 5), (3, 1, 2), (-2, 2), "f32", 11)
    inp = make_inputs(w)
    out, lse = run_gpu(w, inp)
    compare_full(w, inp, out, lse)


SMALL_BF16 = [
    # several tiles, clamped windows at every edge, random offsets
    Workload("bf16_small_a", 1, 3, 128, (8, 16, 24), (4, 8, 8), (3, 3, 3), (-2, 2), "bf16", 21),
    # 384-token tiles (three 128-row chunks), window wider than the tile grid on one axis
    Workload("bf16_small_b", 2, 1, 128, (12, 16, 16), (6, 8, 8), (5, 3, 1), (-1, 1), "bf16", 22),
    # 128-token tiles of 2x8x8 and of 8x4x4 (one chunk = 4 h-planes ... whole planes)
    Workload("bf16_small_c", 1, 2, 128, (8, 16, 16), (2, 8, 8), (3, 2, 2), (-3, 3), "bf16", 23),
    Workload("bf16_small_d", 1, 2, 128, (16, 8, 8), (8, 4, 4), (1, 3, 3), (-1, 1), "bf16", 24),
    # window covering the whole grid: dense attention
    Workload("bf16_small_dense", 1, 2, 128, (8, 8, 16), (4, 8, 8), (9, 9, 9), (0, 0), "bf16", 25),
    # 1x1x1 window: block-diagonal
    Workload("bf16_small_diag", 1, 2, 128, (8, 16, 16), (4, 8, 8), (1, 1, 1), (0, 0), "bf16", 26),
    # a grid of one tile (every window is that tile, whatever the offsets)
    Workload("bf16_one_tile", 1, 3, 128, (4, 8, 8), (4, 8, 8), (3, 3, 3), (-2, 2), "bf16", 27),
    # many (batch, head) slices on a small grid: 160 of them
    Workload("bf16_many_heads", 8, 20, 128, (4, 16, 8), (4, 8, 8), (1, 3, 1), (-1, 1), "bf16", 28),
]


@pytest.mark.parametrize("w", SMALL_BF16, ids=lambda w: w.name)
def test_bf16_small_full(w):
    inp = make_inputs(w)
    out, lse = run_gpu(w, inp)
    compare_full(w, inp, out, lse)


# Near-one-hot softmax rows carry the bf16 rounding of P (relative half-ulp 2^-8) straight
# into O: |err| <= 2^-8 * max|v| ~ 0.02 for |v| <= 5.  These stress inputs are checked
# against that bound (max-abs 4e-2) and, as everywhere, relative L2 <= 1e-2.
STRESS_MAX_ABS = 4e-2


def compare_stress(w, inp, out, lse):
    geo = oracle.Geometry.of(w)
    ref, ref_lse = oracle.forward(geo, inp.q, inp.k, inp.v, inp.offsets)
    got = out.float().cpu().numpy()
    mx, mean, rel = errors(got, ref)
    assert np.isfinite(got).all()
    assert mx <= STRESS_MAX_ABS and rel <= 1e-2, f"max-abs {mx:.3e}, rel-L2 {rel:.3e}"
    assert_lse_close(lse.cpu().numpy(), ref_lse, w.dtype)


def test_bf16_peaky_scores():
    """Q and K scaled by 4: large score spread exercises the running-max rescale."""
    w = Workload("bf16_peaky", 1, 2, 128, (8, 16, 16), (4, 8, 8), (3, 3, 3), (-1, 1), "bf16", 27)
    inp = make_inputs(w)
    inp.q = (inp.q.float() * 4).to(torch.bfloat16)
    inp.k = (inp.k.float() * 4).to(torch.bfloat16)
    out, lse = run_gpu(w, inp)
    compare_stress(w, inp, out, lse)


def test_bf16_growing_scores_force_rescales():
    """Scores grow with the key's time index, and key tiles are visited in ascending order,
    so each row's maximum climbs by far more than the lazy-rescale threshold several times."""
    w = Workload("bf16_growing", 1, 2, 128, (16, 8, 16), (4, 8, 8), (4, 1, 2), (0, 0), "bf16", 35)
    inp = make_inputs(w)
    T = w.grid[0]
    g = torch.arange(T, dtype=torch.float32).view(1, 1, T, 1, 1, 1) * (8.0 / (T - 1))
    u = torch.ones(w.d)
    inp.q = (0.5 * inp.q.float() + 0.25 * u).to(torch.bfloat16)
    inp.k = (0.3 * inp.k.float() + g * u).to(torch.bfloat16)
    out, lse = run_gpu(w, inp)
    compare_stress(w, inp, out, lse)


def test_bf16_every_output_written():
    """Outputs prefilled with NaN: every element must be overwritten."""
    w = SMALL_BF16[1]
    inp = make_inputs(w)
    q, k, v, off = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.offsets.cuda()
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:5], float("nan"), device=q.device)
    dsa.forward(q, k, v, off, w.tile, w.window, w.scale, out=out, lse=lse)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


MANY_UNITS = [
    # more work units than SMs, so every CTA of the persistent kernel runs several units
    Workload("bf16_many_units_s2", 4, 16, 128, (8, 16, 16), (4, 8, 8), (3, 3, 3), (-1, 1), "bf16", 28),
    # 384-token tiles: a two-slot unit and a one-slot unit per tile, many of each per CTA
    Workload("bf16_many_units_s3", 2, 16, 128, (12, 16, 16), (6, 8, 8), (3, 3, 3), (-1, 1), "bf16", 29),
    # 128-token tiles: one-slot units only
    Workload("bf16_many_units_s1", 2, 24, 128, (8, 16, 16), (2, 8, 8), (3, 3, 3), (-2, 2), "bf16", 30),
]


@pytest.mark.parametrize("w", MANY_UNITS, ids=lambda w: w.name)
def test_bf16_many_units_sampled(w):
    inp = make_inputs(w)
    out, lse = run_gpu(w, inp)
    compare_sampled(w, inp, out, lse, n_samples=24, seed=3)


@pytest.mark.parametrize("name", ["bf16_16x32x32", "bf16_480p", "bf16_720p", "adapt_480p_b2"])
def test_bf16_workload_sampled(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    out, lse = run_gpu(w, inp)
    compare_sampled(w, inp, out, lse)


HOST_CASES = [SMALL_BF16[0],
              # ten (batch, head) slices: the host path pipelines them in ten groups of one
              Workload("bf16_host_10", 2, 5, 128, (8, 16, 16), (4, 8, 8), (3, 3, 3), (-2, 2), "bf16", 24),
              # the exact-fp32 path through the same pipeline
              WORKLOADS["tiny_f32"]]


@pytest.mark.parametrize("w", HOST_CASES, ids=lambda w: w.name)
def test_forward_host_matches_device(w):
    """The host-buffer entry point (copies pipelined over head groups on internal streams)
    gives bit-for-bit the device entry point's results."""
    inp = make_inputs(w)
    out, lse = run_gpu(w, inp)
    p = dsa.make_problem(w.B, w.heads, w.d, w.grid, w.tile, w.window, w.scale,
                         dsa.DSA_BF16 if w.dtype == "bf16" else dsa.DSA_F32)
    dev = torch.empty(dsa.forward_host_bytes(p), dtype=torch.uint8, device="cuda")
    qh, kh, vh = inp.q.pin_memory(), inp.k.pin_memory(), inp.v.pin_memory()
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty(qh.shape[:5], dtype=torch.float32).pin_memory()
    dsa.forward_host(p, qh, kh, vh, inp.offsets.contiguous(), oh, lh, dev)
    torch.cuda.synchronize()
    assert torch.equal(oh, out.cpu()) and torch.equal(lh, lse.cpu())


def test_bounded_wait_runs_out_and_the_context_survives():
    """The failure path every kernel relies on: a wait nothing completes runs out after its
    limit, the device status reports DSA_ERR_TIMEOUT at the self-test's site, and the next
    forward on the same context runs and is correct."""
    dsa.device_status()  # start from a clear status word
    dsa.selftest_wait()
    st, site, _ = dsa.device_status()
    assert st == 4 and site == 99, (st, site)  # DSA_ERR_TIMEOUT
    w = SMALL_BF16[0]
    inp = make_inputs(w)
    out, lse = run_gpu(w, inp)
    assert dsa.device_status()[0] == 0
    compare_full(w, inp, out, lse)


def test_forward_and_backward_replay_from_a_cuda_graph():
    """The planner, forward and backward launches can be captured in a CUDA graph and
    replayed (every launch goes to the caller's stream; no allocation, no synchronisation
    inside the calls); replays give the eager results."""
    w = Workload("graph_bf16", 1, 2, 128, (8, 16, 16), (4, 8, 8), (3, 3, 3), (-1, 1), "bf16", 29, backward=True)
    inp = make_inputs(w)
    q, k, v, dout, off = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.dout.cuda(), inp.offsets.cuda()
    p = dsa.make_problem(w.B, w.heads, w.d, w.grid, w.tile, w.window, w.scale)
    ws_f, ws_b = dsa.workspace(p, q.device), dsa.workspace(p, q.device, backward=True)
    out, lse = torch.empty_like(q), torch.empty(q.shape[:5], dtype=torch.float32, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ref_o, ref_l = dsa.forward(q, k, v, off, w.tile, w.window, w.scale)
    ref_g = dsa.backward(q, k, v, ref_o, ref_l, dout, off, w.tile, w.window, w.scale)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside the capture (attribute setup, encoder lookup)
        dsa.forward(q, k, v, off, w.tile, w.window, w.scale, out=out, lse=lse, ws=ws_f, stream=s)
        dsa.backward(q, k, v, out, lse, dout, off, w.tile, w.window, w.scale, dq=dq, dk=dk, dv=dv, ws=ws_b, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        dsa.forward(q, k, v, off, w.tile, w.window, w.scale, out=out, lse=lse, ws=ws_f, stream=s)
        dsa.backward(q, k, v, out, lse, dout, off, w.tile, w.window, w.scale, dq=dq, dk=dk, dv=dv, ws=ws_b, stream=s)
    for tensor in (out, lse, dq, dk, dv):
        tensor.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert dsa.device_status()[0] == 0
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
    # every gradient is summed in a fixed order: the replays match the direct call bit for bit
    assert torch.equal(dq, ref_g[0]) and torch.equal(dk, ref_g[1]) and torch.equal(dv, ref_g[2])
    del g
