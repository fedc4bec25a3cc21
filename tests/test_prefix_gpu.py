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
