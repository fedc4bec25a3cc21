"""GPU text-prefix forward against the fp64 oracle (the MOD-DiT page, "Token-Type-Aware
Masking": in a unified text + video sequence, text tokens attend to and are attended by
everything; only video-video attention is sparse).  Text lengths cover a partial last key
chunk in each half of a step (77, 200), a step whose second half holds no key (300), a
single token, none at all (bit-exact with the window forward) and the ~1% share of a 720p
grid (sampled rows)."""
import numpy as np
import pytest
import torch

import oracle
import video_dit_sparse_dsa_b200 as dsa
from dsa_inputs import WORKLOADS, Workload, make_inputs, make_text_inputs, text_length
from tests._parity import assert_close, assert_lse_close

pytestmark = pytest.mark.gpu

SMALL = Workload("prefix_small", 1, 2, 128, (8, 16, 24), (4, 8, 8), (3, 3, 3), (-1, 1), "bf16", 51)


def run(w, inp, txt):
    dev = torch.device("cuda")
    res = dsa.forward_prefix(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.offsets.to(dev), txt.q.to(dev),
                             txt.k.to(dev), txt.v.to(dev), w.tile, w.window, w.scale)
    torch.cuda.synchronize()
    st, site, _ = dsa.device_status()
    assert st == 0, f"device status {st} at site {site}"
    return res


@pytest.mark.parametrize("L", [1, 77, 200, 300])
def test_prefix_small_full(L):
    w = SMALL
    inp = make_inputs(w)
    txt = make_text_inputs(w, L, seed=100 + L)
    out, lse, out_x, lse_x = run(w, inp, txt)
    geo = oracle.Geometry.of(w)
    ref, ref_lse, ref_x, ref_lse_x = oracle.forward_prefix(geo, inp.q, inp.k, inp.v, inp.offsets, txt.q, txt.k,
                                                           txt.v)
    assert_close(out.float().cpu().numpy(), ref, w.dtype, "video out")
    assert_lse_close(lse.cpu().numpy(), ref_lse, w.dtype, "video lse")
    assert_close(out_x.float().cpu().numpy(), ref_x, w.dtype, "text out")
    assert_lse_close(lse_x.cpu().numpy(), ref_lse_x, w.dtype, "text lse")


def test_prefix_without_text_is_the_window_forward():
    w = SMALL
    inp = make_inputs(w)
    txt = make_text_inputs(w, 0, seed=7)
    out, lse, out_x, lse_x = run(w, inp, txt)
    dev = torch.device("cuda")
    ref, ref_lse = dsa.forward(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.offsets.to(dev), w.tile, w.window,
                               w.scale)
    assert torch.equal(out, ref) and torch.equal(lse, ref_lse)
    assert out_x.numel() == 0 and lse_x.numel() == 0


def test_prefix_text_is_order_free_over_keys():
    """The text rows see one softmax over all keys: permuting the text keys (with their
    values) changes nothing beyond rounding, and the video rows likewise."""
    w = SMALL
    inp = make_inputs(w)
    txt = make_text_inputs(w, 200, seed=9)
    a = run(w, inp, txt)
    perm = torch.randperm(200, generator=torch.Generator().manual_seed(1))
    txt2 = type(txt)(txt.q, txt.k[:, :, perm].contiguous(), txt.v[:, :, perm].contiguous())
    b = run(w, inp, txt2)
    for x, y, name in zip(a, b, ("out", "lse", "out_text", "lse_text")):
        assert_close(x.float().cpu().numpy(), y.float().cpu().numpy().astype(np.float64), w.dtype, name)


def test_prefix_720p_sampled():
    w = WORKLOADS["bf16_720p"]
    L = text_length(w)
    inp = make_inputs(w)
    txt = make_text_inputs(w, L, seed=1000 + w.seed)
    out, lse, out_x, lse_x = run(w, inp, txt)
    geo = oracle.Geometry.of(w)
    BH = w.B * w.heads
    rng = np.random.default_rng(5)
    bh = np.concatenate([[0, BH - 1], rng.integers(0, BH, 4)]).astype(np.int32)
    tiles = np.concatenate([[0, geo.n_tiles - 1], rng.integers(0, geo.n_tiles, 4)]).astype(np.int32)
    ref, ref_lse = oracle.forward_prefix_tiles(geo, inp.q, inp.k, inp.v, inp.offsets, txt.k, txt.v, (bh, tiles))
    tok = geo.tile_token_index()
    o = out.reshape(BH, geo.n_tokens, w.d)
    l = lse.reshape(BH, geo.n_tokens)
    idx_b = torch.as_tensor(np.repeat(bh, geo.tile_tokens), device=out.device, dtype=torch.long)
    idx_t = torch.as_tensor(tok[tiles].reshape(-1), device=out.device, dtype=torch.long)
    assert_close(o[idx_b, idx_t].float().cpu().numpy().reshape(ref.shape), ref, w.dtype, "video out")
    assert_lse_close(l[idx_b, idx_t].cpu().numpy().reshape(ref_lse.shape), ref_lse, w.dtype, "video lse")
    rows = np.concatenate([[0, L - 1], rng.integers(0, L, 6)])
    ref_x, ref_lse_x = oracle.forward_prefix_text(geo, txt.q, txt.k, txt.v, inp.k, inp.v, rows)
    assert_close(out_x[:, :, rows].float().cpu().numpy(), ref_x, w.dtype, "text out")
    assert_lse_close(lse_x[:, :, rows].cpu().numpy(), ref_lse_x, w.dtype, "text lse")


# ------------------------------------------------------------------------------------
# backward of the text prefix


def _dout(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def run_backward(w, inp, txt, seed):
    dev = torch.device("cuda")
    q, k, v, off = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.offsets.to(dev)
    qt, kt, vt = txt.q.to(dev), txt.k.to(dev), txt.v.to(dev)
    out, lse, out_t, lse_t = dsa.forward_prefix(q, k, v, off, qt, kt, vt, w.tile, w.window, w.scale)
    do, do_t = _dout(tuple(q.shape), seed), _dout(tuple(qt.shape), seed + 1)
    grads = dsa.backward_prefix(q, k, v, out, lse, do.to(dev), off, qt, kt, vt, out_t, lse_t, do_t.to(dev), w.tile,
                                w.window, w.scale)
    torch.cuda.synchronize()
    st, site, _ = dsa.device_status()
    assert st == 0, f"device status {st} at site {site}"
    return grads, do, do_t


def check_backward(w, inp, txt, grads, do, do_t):
    geo = oracle.Geometry.of(w)
    (rq, rk, rv), (rqt, rkt, rvt) = oracle.backward_prefix(geo, inp.q, inp.k, inp.v, do, inp.offsets, txt.q, txt.k,
                                                           txt.v, do_t)
    for got, ref, name in zip(grads, (rq, rk, rv, rqt, rkt, rvt), ("dq", "dk", "dv", "dq_text", "dk_text", "dv_text")):
        assert_close(got.float().cpu().numpy(), ref, w.dtype, name)


@pytest.mark.parametrize("L", [1, 77, 200])
def test_prefix_backward_small_full(L):
    w = SMALL
    inp = make_inputs(w)
    txt = make_text_inputs(w, L, seed=200 + L)
    grads, do, do_t = run_backward(w, inp, txt, 300 + L)
    check_backward(w, inp, txt, grads, do, do_t)


def test_prefix_backward_without_text_is_the_window_backward():
    w = SMALL
    inp = make_inputs(w)
    txt = make_text_inputs(w, 0, seed=9)
    grads, do, _ = run_backward(w, inp, txt, 11)
    dev = torch.device("cuda")
    q, k, v, off = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.offsets.to(dev)
    out, lse = dsa.forward(q, k, v, off, w.tile, w.window, w.scale)
    ref = dsa.backward(q, k, v, out, lse, do.to(dev), off, w.tile, w.window, w.scale)
    # without text the prefix backward is the window backward: the same kernels, every sum
    # in a fixed order, so the gradients are identical bit for bit
    assert torch.equal(grads[0], ref[0]) and torch.equal(grads[1], ref[1]) and torch.equal(grads[2], ref[2])
    assert all(g.numel() == 0 for g in grads[3:])


def test_prefix_backward_16x32x32_grid_full():
    """A 16384-token grid (64 tiles, 3x3x3 windows) with 163 text tokens: every text key
    sees 256 video query chunks cut into parts."""
    w = Workload("prefix_16x32x32", 1, 1, 128, (16, 32, 32), (4, 8, 8), (3, 3, 3), (-1, 1), "bf16", 61)
    inp = make_inputs(w)
    txt = make_text_inputs(w, 163, seed=62)
    grads, do, do_t = run_backward(w, inp, txt, 63)
    check_backward(w, inp, txt, grads, do, do_t)


def test_prefix_backward_720p_sampled():
    """The 720p grid with its ~1% of text tokens, as the benchmark times it: gradients of two
    (batch, head) slices on sampled rows (video and text queries and keys, first and last
    rows)."""
    w = WORKLOADS["bf16_720p"]
    L = text_length(w)
    inp = make_inputs(w)
    txt = make_text_inputs(w, L, seed=1000 + w.seed)
    grads, do, do_t = run_backward(w, inp, txt, 77)
    geo = oracle.Geometry.of(w)
    rng = np.random.default_rng(6)
    N = geo.n_tokens
    BH = w.B * w.heads
    for h in (7, BH - 1):
        q_rows = np.concatenate([[0, N - 1], rng.integers(0, N, 6)])
        k_rows = np.concatenate([[1, N - 2], rng.integers(0, N, 6)])
        t_rows = np.concatenate([[0, L - 1], rng.integers(0, L, 4)])
        ref = oracle.backward_prefix_sampled(geo, inp.q, inp.k, inp.v, do, inp.offsets, txt.q, txt.k, txt.v, do_t,
                                             h, q_rows, t_rows, k_rows, t_rows)

        def rows(t, idx):
            return t.reshape(BH, -1, w.d)[h][torch.as_tensor(idx, device=t.device)].float().cpu().numpy()

        got = (rows(grads[0], q_rows), rows(grads[3], t_rows), rows(grads[1], k_rows), rows(grads[2], k_rows),
               rows(grads[4], t_rows), rows(grads[5], t_rows))
        for g, r, name in zip(got, ref, ("dq", "dq_text", "dk", "dv", "dk_text", "dv_text")):
            assert_close(g, r, w.dtype, f"{name} of (batch, head) {h}")


def test_prefix_backward_is_bit_identical_across_runs():
    """No gradient of the text prefix is summed with atomics (parts are added in part order):
    two runs of the backward give the same bits."""
    w = Workload("prefix_repeat", 1, 2, 128, (8, 16, 24), (4, 8, 8), (3, 3, 3), (-2, 2), "bf16", 64)
    inp = make_inputs(w)
    txt = make_text_inputs(w, 150, seed=65)
    first, _, _ = run_backward(w, inp, txt, 66)
    again, _, _ = run_backward(w, inp, txt, 66)
    for a, b, name in zip(first, again, ("dq", "dk", "dv", "dq_text", "dk_text", "dv_text")):
        assert torch.equal(a, b), f"{name} differs between runs"
