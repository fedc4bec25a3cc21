"""Seeded random problem shapes through the bf16 tensor-core path (window, text-prefix and
key-tile-list forms), forward and backward,
each compared in full with the fp64 oracle: tile planes of 8x8, 4x8, 8x4, 4x4, 2x8 and 8x2
tokens (a 128-token chunk spans 128 / (th tw) t-planes), tile grids of 1-3 tiles per axis,
windows of 1-4 tiles (often wider than the grid), offsets in [-2, 2], 1-2 batch entries
and heads."""
import numpy as np
import pytest
import torch

import oracle
import video_dit_sparse_dsa_b200 as dsa
from dsa_inputs import Workload, make_inputs
from tests._parity import assert_close, assert_lse_close

pytestmark = pytest.mark.gpu

PLANES = [(8, 8), (4, 8), (8, 4), (4, 4), (2, 8), (8, 2)]


def random_workload(seed: int, offsets=(-2, 2)) -> Workload:
    rng = np.random.default_rng(seed)
    th, tw = PLANES[rng.integers(len(PLANES))]
    tt = (128 // (th * tw)) * int(rng.integers(1, 3))
    G = [int(x) for x in rng.integers(1, 4, 3)]
    if tt * th * tw * G[0] * G[1] * G[2] > 6144:  # keep the oracle quick
        G = [1, G[1], min(G[2], 2)]
    window = tuple(int(x) for x in rng.integers(1, 5, 3))
    return Workload(f"rand{seed}", int(rng.integers(1, 3)), int(rng.integers(1, 3)), 128,
                    (tt * G[0], th * G[1], tw * G[2]), (tt, th, tw), window, offsets, "bf16", 500 + seed,
                    backward=True)


@pytest.mark.parametrize("seed", range(20))
def test_random_shape_forward_and_backward(seed):
    # seeds 16-19: offsets up to 9 tiles, far past the grid: every window is pinned to an edge
    w = random_workload(seed) if seed < 16 else random_workload(seed, offsets=(-9, 9))
    inp = make_inputs(w)
    q, k, v, dout, off = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.dout.cuda(), inp.offsets.cuda()
    out, lse = dsa.forward(q, k, v, off, w.tile, w.window, w.scale)
    st, site, _ = dsa.device_status()
    assert st == 0, f"{w}: device status {st} at site {site}"
    geo = oracle.Geometry.of(w)
    ref, ref_lse = oracle.forward(geo, inp.q, inp.k, inp.v, inp.offsets)
    assert_close(out.float().cpu().numpy(), ref, w.dtype, f"{w.name} out {w.tile} {w.grid} {w.window}")
    assert_lse_close(lse.cpu().numpy(), ref_lse, w.dtype, f"{w.name} lse")
    if w.tile[2] % 4 != 0:  # the backward's LSE / D boxes need tw a multiple of 4: refused up front
        with pytest.raises(dsa.DsaError) as e:
            dsa.backward(q, k, v, out, lse, dout, off, w.tile, w.window, w.scale)
        assert e.value.status == 2  # DSA_ERR_UNSUPPORTED
        return
    dq, dk, dv = dsa.backward(q, k, v, out, lse, dout, off, w.tile, w.window, w.scale)
    st, site, _ = dsa.device_status()
    assert st == 0, f"{w}: device status {st} at site {site}"
    rq, rk, rv = oracle.backward(geo, inp.q, inp.k, inp.v, inp.dout, inp.offsets)
    for got, r, name in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        assert_close(got.float().cpu().numpy(), r, w.dtype, f"{w.name} {name} {w.tile} {w.grid} {w.window}")


@pytest.mark.parametrize("seed", range(6))
def test_random_shape_text_prefix(seed):
    """Random shapes with a random number of text tokens: prefix forward and backward in full."""
    w = random_workload(100 + seed)
    if w.tile[2] % 4 != 0:  # keep the backward's tile-width rule
        w = w.replace(tile=(w.tile[0], w.tile[2], w.tile[1]), grid=(w.grid[0], w.grid[2], w.grid[1]))
    rng = np.random.default_rng(900 + seed)
    L = int(rng.integers(1, 400))
    from dsa_inputs import make_text_inputs

    inp = make_inputs(w)
    txt = make_text_inputs(w, L, seed=950 + seed)
    dev = torch.device("cuda")
    q, k, v, off = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.offsets.to(dev)
    qt, kt, vt = txt.q.to(dev), txt.k.to(dev), txt.v.to(dev)
    out, lse, out_t, lse_t = dsa.forward_prefix(q, k, v, off, qt, kt, vt, w.tile, w.window, w.scale)
    do_t = torch.randn(tuple(qt.shape), generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    grads = dsa.backward_prefix(q, k, v, out, lse, inp.dout.to(dev), off, qt, kt, vt, out_t, lse_t, do_t.to(dev),
                                w.tile, w.window, w.scale)
    st, site, _ = dsa.device_status()
    assert st == 0, f"{w}, L={L}: device status {st} at site {site}"
    geo = oracle.Geometry.of(w)
    ro, rl, rot, rlt = oracle.forward_prefix(geo, inp.q, inp.k, inp.v, inp.offsets, txt.q, txt.k, txt.v)
    tag = f"{w.name} {w.tile} {w.grid} {w.window} L={L}"
    assert_close(out.float().cpu().numpy(), ro, w.dtype, f"out {tag}")
    assert_close(out_t.float().cpu().numpy(), rot, w.dtype, f"out_text {tag}")
    assert_lse_close(lse.cpu().numpy(), rl, w.dtype, f"lse {tag}")
    assert_lse_close(lse_t.cpu().numpy(), rlt, w.dtype, f"lse_text {tag}")
    (rq, rk, rv), (rqt, rkt, rvt) = oracle.backward_prefix(geo, inp.q, inp.k, inp.v, inp.dout, inp.offsets, txt.q,
                                                           txt.k, txt.v, do_t)
    for got, r, name in zip(grads, (rq, rk, rv, rqt, rkt, rvt), ("dq", "dk", "dv", "dq_text", "dk_text", "dv_text")):
        assert_close(got.float().cpu().numpy(), r, w.dtype, f"{name} {tag}")


@pytest.mark.parametrize("seed", range(6))
def test_random_shape_key_tile_lists(seed):
    """Random shapes with random per-(batch, head) key-tile lists (empty rows, repeats):
    forward, backward and block map in full against the oracle's list form."""
    w = random_workload(200 + seed)
    if w.tile[2] % 4 != 0:
        w = w.replace(tile=(w.tile[0], w.tile[2], w.tile[1]), grid=(w.grid[0], w.grid[2], w.grid[1]))
    geo = oracle.Geometry.of(w)
    rng = np.random.default_rng(700 + seed)
    BH, n = w.B * w.heads, geo.n_tiles
    rows, row_ptr = [], np.zeros((BH, n + 1), np.int64)
    total = 0
    for h in range(BH):
        row_ptr[h, 0] = total  # absolute positions: head h's rows continue where head h - 1's end
        for i in range(n):
            cnt = int(rng.integers(0, 6))
            rows.append(rng.integers(0, n, cnt))
            total += cnt
            row_ptr[h, i + 1] = total
    kv_list = np.concatenate(rows).astype(np.int32) if total else np.zeros(0, np.int32)
    rp = row_ptr.astype(np.int32)
    inp = make_inputs(w)
    dev = torch.device("cuda")
    q, k, v, dout = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.dout.to(dev)
    rpd, kvd = torch.from_numpy(rp).to(dev), torch.from_numpy(kv_list).to(dev)
    out, lse = dsa.forward_list(q, k, v, rpd, kvd, w.tile, w.scale)
    dq, dk, dv = dsa.backward_list(q, k, v, out, lse, dout, rpd, kvd, w.tile, w.scale)
    bmap = dsa.block_map(q, k, lse, rpd, kvd, w.tile, w.scale)
    st, site, _ = dsa.device_status()
    assert st == 0, f"{w}: device status {st} at site {site}"
    tag = f"{w.name} {w.tile} {w.grid}"
    ref, ref_lse = oracle.forward_list(geo, inp.q, inp.k, inp.v, rp, kv_list)
    got_o, got_l = out.float().cpu().numpy(), lse.cpu().numpy()
    finite = np.isfinite(ref_lse)  # empty lists: O = 0, LSE = -inf on both sides
    assert np.array_equal(np.isfinite(got_l), finite)
    assert_close(got_o, ref, w.dtype, f"out {tag}")
    assert_lse_close(got_l[finite], ref_lse[finite], w.dtype, f"lse {tag}")
    rq, rk, rv = oracle.backward_list(geo, inp.q, inp.k, inp.v, inp.dout, rp, kv_list)
    for got, r, name in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        assert_close(got.float().cpu().numpy(), r, w.dtype, f"{name} {tag}")
    # block map: the list tests' gate (entries carry the bf16 forward's LSE error, ~1e-3 relative)
    rmap = np.asarray(oracle.block_map_list(geo, inp.q, inp.k, rp, kv_list)).reshape(bmap.shape)
    err = float(np.abs(bmap.cpu().numpy() - rmap).max())
    assert err <= 3e-3, f"map {tag}: max-abs {err:.2e}"
