"""Pins for the fp64 oracle: facts the definition fixes, checked without the oracle's own code.

The operator is 3D Deformable Slide Attention ("MegaSlide-DiT: Memory-Centric Adaptation
and Deformable Local Attention for Efficient Video Diffusion", abstract) in the
tile-granular sliding-window form of "Fast Video Generation with Sliding Tile Attention"
(abstract).  The pages print no worked example, so the oracle is pinned by:

* hand-worked plans (tests/golden/plan_hand.txt);
* an independent characterisation of the window start (the in-grid start whose centre is
  nearest the shifted centre), by brute force over all tiny grids;
* a window covering the grid = dense attention (a separately written numpy formula and
  torch's scaled_dot_product_attention in float64);
* a 1x1x1 window = block-diagonal attention;
* softmax rows sum to one (V = 1 gives O = 1; V = identity exposes P), and the LSE
  normalises each row;
* masked dense attention with the brute-force mask = the windowed oracle;
* backward = central finite differences of L = sum(O * dO) in float64 (the per-tile C
  functions and the whole-head function grouped by query tile), and with a covering window
  the whole-head backward = torch autograd of dense attention;
* dv = P^T dO with P read off the forward (V = identity).
"""
import os

import numpy as np
import pytest
import torch

import oracle
from dsa_inputs import WORKLOADS, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------------------
# independent helpers (written from the definition, sharing nothing with the oracle)

def nearest_start(centre: int, w_eff: int, G: int) -> int:
    """Among in-grid starts s in [0, G - w'], the one whose window centre s + floor(w'/2)
    is nearest the shifted centre (the distance is V-shaped in s, so the minimiser is unique)."""
    cands = list(range(0, G - w_eff + 1))
    dist = [abs(s + w_eff // 2 - centre) for s in cands]
    best = min(dist)
    assert dist.count(best) == 1
    return cands[dist.index(best)]


def brute_mask(grid, tile, window, offsets):
    """[N, N] boolean: key token m is in the window of query token n."""
    T, H, W = grid
    tt, th, tw = tile
    G = (T // tt, H // th, W // tw)
    weff = [min(w, g) for w, g in zip(window, G)]
    off = np.asarray(offsets).reshape(-1, 3)
    coords = np.array([(t, h, w) for t in range(T) for h in range(H) for w in range(W)])
    tcoord = coords // np.array(tile)
    lin = (tcoord[:, 0] * G[1] + tcoord[:, 1]) * G[2] + tcoord[:, 2]
    N = len(coords)
    mask = np.zeros((N, N), bool)
    for n in range(N):
        i = tcoord[n]
        o = off[lin[n]]
        s = [nearest_start(int(i[a] + o[a]), weff[a], G[a]) for a in range(3)]
        inside = np.ones(N, bool)
        for a in range(3):
            inside &= (tcoord[:, a] >= s[a]) & (tcoord[:, a] < s[a] + weff[a])
        mask[n] = inside
    return mask


def dense_attention_np(q, k, v, scale, mask=None):
    """Plain softmax attention in float64 over [BH, N, d] arrays, optional [N, N] mask."""
    s = np.einsum("bnc,bmc->bnm", q, k) * scale
    if mask is not None:
        s = np.where(mask[None], s, -np.inf)
    mx = s.max(axis=-1, keepdims=True)
    e = np.exp(s - mx)
    z = e.sum(axis=-1, keepdims=True)
    return np.einsum("bnm,bmc->bnc", e / z, v), (mx + np.log(z))[..., 0]


def flat(x, geo):
    return np.asarray(x, dtype=np.float64).reshape(geo.B * geo.heads, geo.n_tokens, geo.d)


def rand_inputs(geo, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    shape = (geo.B, geo.heads) + geo.grid + (geo.d,)
    return [torch.randn(shape, generator=g, dtype=torch.float64) * scale for _ in range(4)]


def rand_offsets(geo, lo, hi, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi + 1, (geo.n_tiles, 3), generator=g).to(torch.int32)


# ------------------------------------------------------------------------------------
# plan

def _golden_cases():
    cases = []
    with open(os.path.join(GOLDEN, "plan_hand.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = [list(map(int, p.split())) for p in line.split("|")]
            cases.append(parts)
    return cases


@pytest.mark.parametrize("case", _golden_cases())
def test_plan_hand_worked(case):
    G, window, tile, off, start, keys = case
    n = G[0] * G[1] * G[2]
    offsets = np.zeros((n, 3), np.int32)
    i = (tile[0] * G[1] + tile[1]) * G[2] + tile[2]
    offsets[i] = off
    starts, kv, _, _ = oracle.plan(G, window, offsets)
    assert list(starts[i]) == start
    assert list(kv[i]) == keys


def test_plan_nearest_centre_brute_force():
    """Every 1D grid G <= 6, window <= 7, offset in [-G, G]: start = nearest in-grid start."""
    for G in range(1, 7):
        for w in range(1, 8):
            for axis in range(3):
                for o in range(-G, G + 1):
                    Gs = [1, 1, 1]
                    Gs[axis] = G
                    ws = [1, 1, 1]
                    ws[axis] = w
                    offsets = np.zeros((G, 3), np.int32)
                    offsets[:, axis] = o
                    starts, kv, _, _ = oracle.plan(Gs, ws, offsets)
                    weff = min(w, G)
                    for i in range(G):
                        assert starts[i, axis] == nearest_start(i + o, weff, G)
                        assert list(kv[i]) == list(range(starts[i, axis], starts[i, axis] + weff))


def test_plan_inverse_is_transpose():
    rng = np.random.default_rng(0)
    for trial in range(40):
        G = list(rng.integers(1, 6, size=3))
        window = list(rng.integers(1, 7, size=3))
        n = int(np.prod(G))
        offsets = rng.integers(-4, 5, size=(n, 3)).astype(np.int32)
        starts, kv, row_ptr, q_tiles = oracle.plan(G, window, offsets)
        wt = int(np.prod([min(w, g) for w, g in zip(window, G)]))
        assert kv.shape == (n, wt)
        assert row_ptr[-1] == n * wt
        pairs_fwd = {(int(i), int(j)) for i in range(n) for j in kv[i]}
        pairs_inv = set()
        for j in range(n):
            row = q_tiles[row_ptr[j]:row_ptr[j + 1]]
            assert list(row) == sorted(row)
            pairs_inv |= {(int(i), j) for i in row}
        assert pairs_fwd == pairs_inv
        for i in range(n):
            assert list(kv[i]) == sorted(kv[i])
            assert len(set(kv[i])) == wt


# ------------------------------------------------------------------------------------
# forward

def test_full_window_equals_dense_attention():
    """A window at least as large as the tile grid covers every key: dense attention."""
    geo = oracle.Geometry(2, 2, 16, (4, 4, 6), (2, 2, 3), (3, 2, 5))
    q, k, v, _ = rand_inputs(geo, 1)
    off = rand_offsets(geo, -3, 3, 2)
    out, lse = oracle.forward(geo, q, k, v, off)
    ref_np, lse_np = dense_attention_np(flat(q, geo), flat(k, geo), flat(v, geo), geo.scale)
    np.testing.assert_allclose(flat(out, geo), ref_np, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(lse_np.shape), lse_np, rtol=0, atol=1e-12)
    sdpa = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(flat(q, geo)), torch.from_numpy(flat(k, geo)), torch.from_numpy(flat(v, geo)),
        scale=geo.scale)
    np.testing.assert_allclose(flat(out, geo), sdpa.numpy(), rtol=0, atol=1e-12)


def test_peaky_scores_full_window():
    """Large scores exercise the max subtraction: still equal to dense attention."""
    geo = oracle.Geometry(1, 2, 8, (2, 4, 4), (1, 2, 2), (4, 4, 4))
    q, k, v, _ = rand_inputs(geo, 3, scale=6.0)
    off = torch.zeros((geo.n_tiles, 3), dtype=torch.int32)
    out, lse = oracle.forward(geo, q, k, v, off)
    sdpa = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(flat(q, geo)), torch.from_numpy(flat(k, geo)), torch.from_numpy(flat(v, geo)),
        scale=geo.scale)
    assert np.isfinite(lse).all()
    np.testing.assert_allclose(flat(out, geo), sdpa.numpy(), rtol=0, atol=1e-10)


def test_unit_window_equals_block_diagonal():
    geo = oracle.Geometry(1, 3, 8, (2, 4, 6), (1, 2, 3), (1, 1, 1))
    q, k, v, _ = rand_inputs(geo, 4)
    off = torch.zeros((geo.n_tiles, 3), dtype=torch.int32)
    out, _ = oracle.forward(geo, q, k, v, off)
    tok = geo.tile_token_index()
    qf, kf, vf, of = flat(q, geo), flat(k, geo), flat(v, geo), flat(out, geo)
    for t in range(geo.n_tiles):
        idx = tok[t]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qf[:, idx]), torch.from_numpy(kf[:, idx]), torch.from_numpy(vf[:, idx]),
            scale=geo.scale)
        np.testing.assert_allclose(of[:, idx], ref.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("window,lo,hi", [((2, 1, 3), -2, 2), ((3, 3, 3), -1, 1), ((1, 2, 2), -3, 3),
                                          ((2, 2, 1), 0, 0)])
def test_masked_dense_brute_force(window, lo, hi):
    geo = oracle.Geometry(1, 2, 8, (3, 4, 6), (1, 2, 2), window)
    q, k, v, _ = rand_inputs(geo, 5)
    off = rand_offsets(geo, lo, hi, 6)
    out, lse = oracle.forward(geo, q, k, v, off)
    mask = brute_mask(geo.grid, geo.tile, geo.window, off.numpy())
    assert (mask.sum(1) == geo.n_window_tiles * geo.tile_tokens).all()
    ref, ref_lse = dense_attention_np(flat(q, geo), flat(k, geo), flat(v, geo), geo.scale, mask)
    np.testing.assert_allclose(flat(out, geo), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(ref_lse.shape), ref_lse, rtol=0, atol=1e-12)
    sdpa = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(flat(q, geo)), torch.from_numpy(flat(k, geo)), torch.from_numpy(flat(v, geo)),
        attn_mask=torch.from_numpy(mask), scale=geo.scale)
    np.testing.assert_allclose(flat(out, geo), sdpa.numpy(), rtol=0, atol=1e-12)


def test_rows_sum_to_one_and_lse_normalises():
    geo = oracle.Geometry(1, 1, 48, (2, 4, 6), (1, 2, 3), (2, 1, 1))
    q, k, _, _ = rand_inputs(geo, 7)
    off = rand_offsets(geo, -1, 1, 8)
    # V = 1 gives O = 1
    ones = torch.ones_like(q)
    out1, _ = oracle.forward(geo, q, k, ones, off)
    np.testing.assert_allclose(out1, 1.0, rtol=0, atol=1e-13)
    # V = identity (d = N) exposes the softmax rows
    eye = torch.eye(geo.n_tokens, dtype=torch.float64).reshape((1, 1) + geo.grid + (geo.n_tokens,))
    out, lse = oracle.forward(geo, q, k, eye, off)
    P = flat(out, geo)[0]
    mask = brute_mask(geo.grid, geo.tile, geo.window, off.numpy())
    np.testing.assert_allclose(P.sum(1), 1.0, rtol=0, atol=1e-13)
    assert (P[~mask] == 0).all()
    assert (P[mask] > 0).all()
    s = flat(q, geo)[0] @ flat(k, geo)[0].T * geo.scale
    lse = lse.reshape(-1)
    z = np.where(mask, np.exp(s - lse[:, None]), 0.0).sum(1)
    np.testing.assert_allclose(z, 1.0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(P[mask], np.exp(s - lse[:, None])[mask], rtol=1e-12, atol=0)


def test_oracle_selection_matches_full():
    """Sampled (bh, tile) calls give the rows of the full call."""
    geo = oracle.Geometry(2, 3, 16, (4, 4, 4), (2, 2, 2), (1, 2, 2))
    q, k, v, _ = rand_inputs(geo, 9)
    off = rand_offsets(geo, -1, 1, 10)
    out, lse = oracle.forward(geo, q, k, v, off)
    sel_bh = np.array([5, 0, 3], np.int32)
    sel_t = np.array([7, 2, 0], np.int32)
    o_t, l_t = oracle.forward_tiles(geo, q, k, v, off, (sel_bh, sel_t))
    tok = geo.tile_token_index()
    of, lf = flat(out, geo), lse.reshape(geo.B * geo.heads, -1)
    for s in range(3):
        np.testing.assert_array_equal(o_t[s], of[sel_bh[s], tok[sel_t[s]]])
        np.testing.assert_array_equal(l_t[s], lf[sel_bh[s], tok[sel_t[s]]])


# ------------------------------------------------------------------------------------
# backward

def _loss(geo, q, k, v, dout, off):
    out, _ = oracle.forward(geo, q, k, v, off)
    return float((out * dout.numpy()).sum())


@pytest.mark.parametrize("window", [(2, 1, 1), (1, 1, 2), (3, 2, 2)])
def test_backward_finite_differences(window):
    geo = oracle.Geometry(1, 1, 3, (3, 2, 4), (1, 2, 2), window)
    q, k, v, dout = rand_inputs(geo, 11)
    off = rand_offsets(geo, -1, 1, 12)
    dq, dk, dv = oracle.backward(geo, q, k, v, dout, off)
    h = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros(x.numel())
        xf = x.reshape(-1)
        for e in range(x.numel()):
            old = float(xf[e])
            xf[e] = old + h
            lp = _loss(geo, q, k, v, dout, off)
            xf[e] = old - h
            lm = _loss(geo, q, k, v, dout, off)
            xf[e] = old
            fd[e] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g.reshape(-1), fd, rtol=0, atol=2e-9, err_msg=name)


def test_dv_is_pt_dout():
    """dv = P^T dO, with P read off the forward by V = identity."""
    geo = oracle.Geometry(1, 1, 24, (2, 2, 6), (1, 2, 2), (2, 1, 2))
    q, k, v, _ = rand_inputs(geo, 13)
    off = rand_offsets(geo, -1, 1, 14)
    eye = torch.eye(geo.n_tokens, dtype=torch.float64).reshape((1, 1) + geo.grid + (geo.n_tokens,))
    P = flat(oracle.forward(geo, q, k, eye, off)[0], geo)[0]
    g = torch.Generator().manual_seed(15)
    dout = torch.randn(q.shape, generator=g, dtype=torch.float64)
    _, _, dv = oracle.backward(geo, q, k, v, dout, off)
    np.testing.assert_allclose(flat(dv, geo)[0], P.T @ flat(dout, geo)[0], rtol=0, atol=1e-12)


def test_backward_selection_matches_full():
    geo = oracle.Geometry(2, 1, 8, (2, 4, 4), (1, 2, 2), (2, 1, 2))
    q, k, v, dout = rand_inputs(geo, 16)
    off = rand_offsets(geo, -1, 1, 17)
    dq, dk, dv = oracle.backward(geo, q, k, v, dout, off)
    sel = (np.array([1, 0], np.int32), np.array([3, 6], np.int32))
    dq_t = oracle.backward_dq_tiles(geo, q, k, v, dout, off, sel)
    dk_t, dv_t = oracle.backward_dkdv_tiles(geo, q, k, v, dout, off, sel)
    tok = geo.tile_token_index()
    for s in range(2):
        bh, t = sel[0][s], sel[1][s]
        # dk/dv sum per-thread partials in a thread-dependent order: equal up to rounding
        np.testing.assert_allclose(dq_t[s], flat(dq, geo)[bh, tok[t]], rtol=0, atol=1e-13)
        np.testing.assert_allclose(dk_t[s], flat(dk, geo)[bh, tok[t]], rtol=0, atol=1e-13)
        np.testing.assert_allclose(dv_t[s], flat(dv, geo)[bh, tok[t]], rtol=0, atol=1e-13)


@pytest.mark.parametrize("window", [(2, 1, 2), (3, 2, 2)])
def test_backward_head_finite_differences(window):
    """The whole-head backward (grouped by query tile) against central finite differences of
    L = sum(O * dO), computed from the forward alone."""
    geo = oracle.Geometry(1, 2, 3, (3, 2, 4), (1, 2, 2), window)
    q, k, v, dout = rand_inputs(geo, 18)
    off = rand_offsets(geo, -1, 1, 19)
    h, hh = 1e-5, 1
    grads = oracle.backward_head(geo, q, k, v, dout, off, hh)
    for x, g, name in zip((q, k, v), grads, ("q", "k", "v")):
        xf = x.reshape(geo.B * geo.heads, -1)[hh]
        fd = np.zeros(xf.numel())
        for e in range(xf.numel()):
            old = float(xf[e])
            xf[e] = old + h
            lp = _loss(geo, q, k, v, dout, off)
            xf[e] = old - h
            lm = _loss(geo, q, k, v, dout, off)
            xf[e] = old
            fd[e] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g.reshape(-1), fd, rtol=0, atol=2e-9, err_msg=name)


def test_backward_head_full_window_is_autograd_of_dense_attention():
    """With a window covering the grid, the whole-head backward is the gradient of dense
    softmax attention (torch autograd, float64)."""
    geo = oracle.Geometry(1, 2, 8, (2, 4, 4), (1, 2, 2), (2, 2, 2))
    q, k, v, dout = rand_inputs(geo, 20)
    off = rand_offsets(geo, -2, 2, 21)
    BH, N, d = geo.B * geo.heads, geo.n_tokens, geo.d
    qa, ka, va = (t.reshape(BH, N, d).clone().requires_grad_(True) for t in (q, k, v))
    o = torch.softmax(geo.scale * qa @ ka.transpose(1, 2), dim=-1) @ va
    (o * dout.reshape(BH, N, d)).sum().backward()
    for hh in range(BH):
        got = oracle.backward_head(geo, q, k, v, dout, off, hh)
        for g, ref in zip(got, (qa.grad[hh], ka.grad[hh], va.grad[hh])):
            np.testing.assert_allclose(g, ref.numpy(), rtol=0, atol=1e-12)


def test_backward_head_equals_tile_functions():
    """The whole-head backward equals the C oracle's per-tile backward on every head."""
    geo = oracle.Geometry(2, 2, 16, (4, 4, 6), (2, 2, 2), (2, 1, 3))
    q, k, v, dout = rand_inputs(geo, 22)
    off = rand_offsets(geo, -2, 2, 23)
    dq, dk, dv = oracle.backward(geo, q, k, v, dout, off)
    for hh in range(geo.B * geo.heads):
        got = oracle.backward_head(geo, q, k, v, dout, off, hh)
        for g, ref in zip(got, (dq, dk, dv)):
            np.testing.assert_allclose(g, flat(ref, geo)[hh], rtol=0, atol=1e-12)


# ------------------------------------------------------------------------------------
# workloads

def test_workload_sizes():
    """Derived sizes of the five workloads (effective window, keys per query, FLOP)."""
    expect = {
        "tiny_f32": (16, 12, 192, 2.52e7),
        "bf16_16x32x32": (64, 27, 6912, 1.392e12),
        "bf16_480p": (140, 45, 11520, 2.537e12),
        "bf16_720p": (300, 27, 10368, 1.4677e13),
        "adapt_480p_b2": (140, 45, 11520, 5.073e12),
    }
    for name, (nt, wt, kpq, flops) in expect.items():
        w = WORKLOADS[name]
        assert w.n_tiles == nt and w.window_tiles == wt and w.keys_per_query == kpq
        assert abs(w.fwd_flops() / flops - 1) < 2e-3  # the table rounds to 4 digits


def test_tiny_workload_inputs_are_seeded():
    w = WORKLOADS["tiny_f32"]
    a = make_inputs(w)
    b = make_inputs(w)
    assert torch.equal(a.q, b.q) and torch.equal(a.offsets, b.offsets)
    assert a.q.dtype == torch.float32 and (a.offsets == 0).all()
    w2 = WORKLOADS["bf16_16x32x32"].replace(heads=1, grid=(4, 8, 8))
    c = make_inputs(w2)
    assert c.q.dtype == torch.bfloat16
    assert int(c.offsets.min()) >= -1 and int(c.offsets.max()) <= 1


# ------------------------------------------------------------------------------------
# key-tile lists (block-sparse form): pinned against multiset-weighted dense attention
# written here with torch (autograd gives the backward), sharing nothing with the oracle

def tile_of_token(geo):
    """[N] linear tile index of every token of the raster grid."""
    T, H, W = geo.grid
    tt, th, tw = geo.tile
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    return (((t // tt) * geo.G[1] + h // th) * geo.G[2] + w // tw).reshape(-1)


def list_counts(geo, row_ptr, kv_list):
    """[nTiles, nTiles] how often query tile i lists key tile j."""
    c = np.zeros((geo.n_tiles, geo.n_tiles), np.int64)
    for i in range(geo.n_tiles):
        for e in range(row_ptr[i], row_ptr[i + 1]):
            c[i, kv_list[e]] += 1
    return c


def multiset_attention(geo, q, k, v, row_ptr, kv_list):
    """Dense fp64 attention with each key weighted by how often its tile is listed:
    o_n = sum_m c_nm e^{s_nm} v_m / sum_m c_nm e^{s_nm}, lse_n = ln sum_m c_nm e^{s_nm};
    rows with no key: o = 0, lse = -inf.  Differentiable in q, k, v."""
    tot = tile_of_token(geo)
    cnt = torch.tensor(list_counts(geo, row_ptr, kv_list)[tot][:, tot], dtype=torch.float64)  # [N, N]
    BH = geo.B * geo.heads
    qf, kf, vf = (t.reshape(BH, geo.n_tokens, geo.d) for t in (q, k, v))
    s = torch.einsum("hnd,hmd->hnm", qf, kf) * geo.scale
    logw = torch.where(cnt > 0, torch.log(cnt.clamp(min=1)), torch.full_like(cnt, -torch.inf))
    has = (cnt > 0).any(dim=-1)  # [N] rows with at least one key
    # rows without keys get a finite stand-in row (no NaN in autograd) and are zeroed
    z = torch.where(has[:, None], s + logw, torch.zeros_like(s))
    lse = torch.logsumexp(z, dim=-1)
    p = torch.exp(z - lse[..., None]) * has[:, None]
    o = p @ vf
    lse = torch.where(has, lse, torch.full_like(lse, -torch.inf))
    return o.reshape(q.shape), lse.reshape(q.shape[:-1])


def random_lists(geo, seed, max_len, allow_empty=True, allow_dup=True):
    rng = np.random.default_rng(seed)
    rows = []
    for i in range(geo.n_tiles):
        n = int(rng.integers(0 if allow_empty else 1, max_len + 1))
        if allow_empty and i == geo.n_tiles // 2:
            n = 0  # every such case holds an empty list
        if allow_dup:
            rows.append(rng.integers(0, geo.n_tiles, n))
        else:
            rows.append(rng.permutation(geo.n_tiles)[:n])
    row_ptr = np.zeros(geo.n_tiles + 1, np.int32)
    row_ptr[1:] = np.cumsum([len(r) for r in rows])
    kv_list = np.concatenate(rows).astype(np.int32) if row_ptr[-1] else np.zeros(0, np.int32)
    return row_ptr, kv_list


def small_inputs(geo, seed):
    g = torch.Generator().manual_seed(seed)
    shape = (geo.B, geo.heads) + geo.grid + (geo.d,)
    return [torch.randn(shape, generator=g, dtype=torch.float64) for _ in range(4)]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_lists_forward_equal_multiset_attention(seed):
    """Random lists (empty rows, repeated tiles, any order) = weighted dense attention."""
    geo = oracle.Geometry(1, 2, 16, (2, 4, 6), (1, 2, 2), (1, 1, 1))
    q, k, v, _ = small_inputs(geo, seed)
    row_ptr, kv_list = random_lists(geo, seed, 5)
    assert (np.diff(row_ptr) == 0).any(), "the case must hold an empty list"
    out, lse = oracle.forward_list(geo, q, k, v, row_ptr, kv_list)
    ref_o, ref_lse = multiset_attention(geo, q, k, v, row_ptr, kv_list)
    np.testing.assert_allclose(out, ref_o.numpy(), rtol=0, atol=1e-12)
    finite = np.isfinite(ref_lse.numpy())
    assert np.array_equal(np.isfinite(lse), finite)
    np.testing.assert_allclose(lse[finite], ref_lse.numpy()[finite], rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1])
def test_lists_backward_equal_autograd_of_multiset_attention(seed):
    geo = oracle.Geometry(1, 2, 8, (2, 4, 4), (1, 2, 2), (1, 1, 1))
    q, k, v, do = small_inputs(geo, 10 + seed)
    row_ptr, kv_list = random_lists(geo, 10 + seed, 4)
    dq, dk, dv = oracle.backward_list(geo, q, k, v, do, row_ptr, kv_list)
    qr, kr, vr = (t.clone().requires_grad_(True) for t in (q, k, v))
    o, _ = multiset_attention(geo, qr, kr, vr, row_ptr, kv_list)
    (o * do).sum().backward()
    for got, ref in ((dq, qr.grad), (dk, kr.grad), (dv, vr.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-11)


def test_lists_repeated_tiles_closed_form():
    """Listing every tile of a list twice leaves O unchanged and adds ln 2 to the LSE."""
    geo = oracle.Geometry(1, 1, 16, (2, 4, 4), (1, 2, 2), (1, 1, 1))
    q, k, v, _ = small_inputs(geo, 5)
    row_ptr, kv_list = random_lists(geo, 5, 4, allow_empty=False, allow_dup=False)
    doubled = np.concatenate([np.concatenate([kv_list[row_ptr[i]:row_ptr[i + 1]]] * 2)
                              for i in range(geo.n_tiles)]).astype(np.int32)
    o1, l1 = oracle.forward_list(geo, q, k, v, row_ptr, kv_list)
    o2, l2 = oracle.forward_list(geo, q, k, v, 2 * row_ptr, doubled)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l2, l1 + np.log(2.0), rtol=0, atol=1e-13)


def test_lists_of_the_window_plan_equal_the_windowed_oracle():
    geo = oracle.Geometry(1, 2, 16, (4, 4, 6), (1, 2, 2), (3, 1, 3))
    q, k, v, do = small_inputs(geo, 7)
    off = torch.randint(-1, 2, (geo.n_tiles, 3), generator=torch.Generator().manual_seed(7)).to(torch.int32)
    _, kv, _, _ = oracle.plan(geo.G, geo.window, off)
    row_ptr = (np.arange(geo.n_tiles + 1) * kv.shape[1]).astype(np.int32)
    o_box, l_box = oracle.forward(geo, q, k, v, off)
    o_list, l_list = oracle.forward_list(geo, q, k, v, row_ptr, kv.reshape(-1))
    np.testing.assert_allclose(o_list, o_box, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l_list, l_box, rtol=0, atol=1e-13)
    for a, b in zip(oracle.backward_list(geo, q, k, v, do, row_ptr, kv.reshape(-1)), oracle.backward(geo, q, k, v, do, off)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_lists_reject_invalid_csr():
    geo = oracle.Geometry(1, 1, 8, (1, 2, 2), (1, 1, 1), (1, 1, 1))
    q, k, v, _ = small_inputs(geo, 0)
    bad = [(np.array([0, 1, 1, 1, 2], np.int32), np.array([0, 4], np.int32)),   # tile out of range
           (np.array([0, 2, 1, 2, 2], np.int32), np.array([0, 1], np.int32)),   # decreasing row_ptr
           (np.array([1, 1, 1, 1, 2], np.int32), np.array([0, 1], np.int32))]   # row_ptr[0] != 0
    for rp, kl in bad:
        with pytest.raises(RuntimeError):
            oracle.forward_list(geo, q, k, v, rp, kl)


def test_lists_per_head_equal_multiset_attention_per_head():
    """A list per (batch, head): each head's rows against its own weighted dense attention."""
    geo = oracle.Geometry(2, 2, 16, (2, 4, 4), (1, 2, 2), (1, 1, 1))
    q, k, v, do = small_inputs(geo, 21)
    BH = geo.B * geo.heads
    rps, lists, base = [], [], 0
    for h in range(BH):
        rp, kl = random_lists(geo, 30 + h, 4)
        rps.append(rp + base)
        lists.append(kl)
        base += len(kl)
    row_ptr = np.stack(rps).astype(np.int32)
    kv_list = np.concatenate(lists).astype(np.int32)
    out, lse = oracle.forward_list(geo, q, k, v, row_ptr, kv_list)
    dq, dk, dv = oracle.backward_list(geo, q, k, v, do, row_ptr, kv_list)
    one = oracle.Geometry(1, 1, 16, geo.grid, geo.tile, (1, 1, 1))
    for h in range(BH):
        b, j = divmod(h, geo.heads)
        sl = [t[b:b + 1, j:j + 1] for t in (q, k, v, do)]
        rp = rps[h] - rps[h][0]
        ref_o, ref_l = multiset_attention(one, sl[0], sl[1], sl[2], rp, lists[h])
        np.testing.assert_allclose(out[b, j], ref_o.numpy()[0, 0], rtol=0, atol=1e-12)
        fin = np.isfinite(ref_l.numpy()[0, 0])
        np.testing.assert_allclose(lse[b, j][fin], ref_l.numpy()[0, 0][fin], rtol=0, atol=1e-12)
        qr, kr, vr = (t.clone().requires_grad_(True) for t in sl[:3])
        o, _ = multiset_attention(one, qr, kr, vr, rp, lists[h])
        (o * sl[3]).sum().backward()
        for got, ref in ((dq, qr.grad), (dk, kr.grad), (dv, vr.grad)):
            np.testing.assert_allclose(got[b, j], ref.numpy()[0, 0], rtol=0, atol=1e-11)


def test_block_map_equals_blocked_dense_probabilities():
    """The block attention mass is the dense softmax matrix summed over key tiles and
    averaged over query tiles (weighted by list multiplicity); rows sum to one."""
    geo = oracle.Geometry(1, 2, 16, (2, 4, 6), (1, 2, 2), (1, 1, 1))
    q, k, _, _ = small_inputs(geo, 3)
    row_ptr, kv_list = random_lists(geo, 3, 5)
    bm = oracle.block_map_list(geo, q, k, row_ptr, kv_list)
    tot = tile_of_token(geo)
    cnt = torch.tensor(list_counts(geo, row_ptr, kv_list)[tot][:, tot], dtype=torch.float64)
    BH = geo.B * geo.heads
    s = torch.einsum("hnd,hmd->hnm", q.reshape(BH, -1, geo.d), k.reshape(BH, -1, geo.d)) * geo.scale
    has = (cnt > 0).any(dim=-1)  # rows with at least one key
    z = torch.where(cnt > 0, s + torch.log(cnt.clamp(min=1)), torch.full_like(s, -torch.inf))
    z = torch.where(has[:, None], z, torch.zeros_like(z))  # a finite stand-in for empty rows
    P = (torch.softmax(z, dim=-1) * has[:, None]).numpy()  # [BH, N, N], multiplicity-weighted
    onehot_t = np.eye(geo.n_tiles)[tot]  # [N, nTiles]
    ref = np.einsum("hnm,mj,ni->hij", P, onehot_t, onehot_t) / geo.tile_tokens
    np.testing.assert_allclose(bm, ref, rtol=0, atol=1e-13)
    sums = bm.sum(axis=-1)
    empty = np.diff(row_ptr) == 0
    np.testing.assert_allclose(sums[:, ~empty], 1.0, rtol=0, atol=1e-13)
    assert np.all(sums[:, empty] == 0.0)


# ------------------------------------------------------------------------------------
# regularised least squares: pinned to a different algorithm and to exact recovery

def test_lstsq_equals_augmented_least_squares():
    """(M^T M + lam I) x = M^T s is the minimiser of |M x - s|^2 + lam |x|^2, which numpy's
    SVD-based lstsq finds from the augmented system [M; sqrt(lam) I] x = [s; 0]."""
    rng = np.random.default_rng(0)
    for m, p, lam in ((200, 3, 0.1), (500, 17, 1e-3), (50, 32, 2.0)):
        M = rng.standard_normal((m, p))
        S = rng.standard_normal((6, m))
        X = oracle.lstsq(M, lam, S)
        A = np.vstack([M, np.sqrt(lam) * np.eye(p)])
        for b in range(S.shape[0]):
            ref = np.linalg.lstsq(A, np.concatenate([S[b], np.zeros(p)]), rcond=None)[0]
            np.testing.assert_allclose(X[b], ref, rtol=0, atol=1e-10)


def test_lstsq_recovers_exact_intensities():
    rng = np.random.default_rng(1)
    M = rng.standard_normal((300, 3))
    X0 = rng.standard_normal((4, 3))
    np.testing.assert_allclose(oracle.lstsq(M, 0.0, X0 @ M.T), X0, rtol=0, atol=1e-12)


# ------------------------------------------------------------------------------------
# text prefix (the MOD-DiT page, "Token-Type-Aware Masking": in a unified text + video
# sequence, text tokens keep full attention and only video-video attention is sparse)

def rand_text(geo, L, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn((geo.B, geo.heads, L, geo.d), generator=g, dtype=torch.float64) * scale for _ in range(3)]


@pytest.mark.parametrize("window,L,lo,hi", [((2, 1, 3), 5, -2, 2), ((1, 2, 2), 1, -1, 1), ((3, 3, 3), 9, 0, 0)])
def test_prefix_equals_masked_dense_over_unified_sequence(window, L, lo, hi):
    """Unified sequence [video; text] under the mask: video -> window (brute force) and
    every text token; text -> everything.  Dense attention over it = the prefix oracle."""
    geo = oracle.Geometry(1, 2, 8, (3, 4, 6), (1, 2, 2), window)
    q, k, v, _ = rand_inputs(geo, 31)
    qt, kt, vt = rand_text(geo, L, 32)
    off = rand_offsets(geo, lo, hi, 33)
    out, lse, out_x, lse_x = oracle.forward_prefix(geo, q, k, v, off, qt, kt, vt)
    N = geo.n_tokens
    mask = np.ones((N + L, N + L), bool)
    mask[:N, :N] = brute_mask(geo.grid, geo.tile, geo.window, off.numpy())
    BH = geo.B * geo.heads
    cat = [np.concatenate([flat(a, geo), np.asarray(b).reshape(BH, L, geo.d)], axis=1) for a, b in
           ((q, qt), (k, kt), (v, vt))]
    ref, ref_lse = dense_attention_np(*cat, geo.scale, mask)
    np.testing.assert_allclose(flat(out, geo), ref[:, :N], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(BH, N), ref_lse[:, :N], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out_x.reshape(BH, L, geo.d), ref[:, N:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_x.reshape(BH, L), ref_lse[:, N:], rtol=0, atol=1e-12)
    sdpa = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(c) for c in cat),
                                                            attn_mask=torch.from_numpy(mask), scale=geo.scale)
    np.testing.assert_allclose(flat(out, geo), sdpa.numpy()[:, :N], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out_x.reshape(BH, L, geo.d), sdpa.numpy()[:, N:], rtol=0, atol=1e-12)


def test_prefix_without_text_is_the_window_forward():
    geo = oracle.Geometry(1, 2, 8, (3, 4, 6), (1, 2, 2), (2, 2, 2))
    q, k, v, _ = rand_inputs(geo, 34)
    qt, kt, vt = rand_text(geo, 0, 35)
    off = rand_offsets(geo, -2, 2, 36)
    out, lse, out_x, lse_x = oracle.forward_prefix(geo, q, k, v, off, qt, kt, vt)
    ref, ref_lse = oracle.forward(geo, q, k, v, off)
    np.testing.assert_array_equal(out, ref)
    np.testing.assert_array_equal(lse, ref_lse)
    assert out_x.size == 0 and lse_x.size == 0


def test_prefix_text_copy_of_video_closed_form():
    """Text = a copy of every video token and a window covering the grid: every key appears
    twice, so every output equals dense video attention and every LSE gains ln 2."""
    geo = oracle.Geometry(1, 2, 8, (2, 4, 4), (1, 2, 2), (2, 2, 2))
    q, k, v, _ = rand_inputs(geo, 37, scale=2.0)
    off = torch.zeros((geo.n_tiles, 3), dtype=torch.int32)
    BH, N = geo.B * geo.heads, geo.n_tokens
    as_text = [torch.from_numpy(flat(a, geo)).reshape(geo.B, geo.heads, N, geo.d) for a in (q, k, v)]
    out, lse, out_x, lse_x = oracle.forward_prefix(geo, q, k, v, off, *as_text)
    dense = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(flat(q, geo)), torch.from_numpy(flat(k, geo)), torch.from_numpy(flat(v, geo)),
        scale=geo.scale).numpy()
    s = np.einsum("bnc,bmc->bnm", flat(q, geo), flat(k, geo)) * geo.scale
    dense_lse = np.log(np.exp(s).sum(-1))
    np.testing.assert_allclose(flat(out, geo), dense, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out_x.reshape(BH, N, geo.d), dense, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(BH, N), dense_lse + np.log(2.0), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_x.reshape(BH, N), dense_lse + np.log(2.0), rtol=0, atol=1e-12)


def _unified_autograd(geo, tensors, text, mask):
    """Masked dense attention over the unified [video; text] sequence in float64 and the
    autograd gradients of sum(O * dO) (written independently of the oracle)."""
    BH = geo.B * geo.heads
    L = text[0].shape[2]
    cat = [torch.cat([torch.as_tensor(flat(a, geo)), torch.as_tensor(np.asarray(b)).reshape(BH, L, geo.d)], 1)
           for a, b in zip(tensors, text)]
    q, k, v = (c.clone().requires_grad_(True) for c in cat[:3])
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(mask), scale=geo.scale)
    (o * cat[3]).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("window,L,lo,hi", [((2, 1, 3), 5, -2, 2), ((1, 2, 2), 1, -1, 1), ((3, 3, 3), 9, 0, 0)])
def test_prefix_backward_equals_autograd_of_unified_attention(window, L, lo, hi):
    geo = oracle.Geometry(1, 2, 8, (3, 4, 6), (1, 2, 2), window)
    q, k, v, do = rand_inputs(geo, 41)
    qt, kt, vt = rand_text(geo, L, 42)
    dot = rand_text(geo, L, 43)[0]
    off = rand_offsets(geo, lo, hi, 44)
    (dq, dk, dv), (dqt, dkt, dvt) = oracle.backward_prefix(geo, q, k, v, do, off, qt, kt, vt, dot, block=7)
    N = geo.n_tokens
    mask = np.ones((N + L, N + L), bool)
    mask[:N, :N] = brute_mask(geo.grid, geo.tile, geo.window, off.numpy())
    gq, gk, gv = _unified_autograd(geo, (q, k, v, do), (qt, kt, vt, dot), mask)
    BH = geo.B * geo.heads
    for got_v, got_t, ref, name in ((dq, dqt, gq, "dq"), (dk, dkt, gk, "dk"), (dv, dvt, gv, "dv")):
        np.testing.assert_allclose(flat(got_v, geo), ref[:, :N], rtol=0, atol=1e-11, err_msg=name)
        np.testing.assert_allclose(np.asarray(got_t).reshape(BH, L, geo.d), ref[:, N:], rtol=0, atol=1e-11,
                                   err_msg=name + "_text")


def test_prefix_backward_without_text_is_the_window_backward():
    geo = oracle.Geometry(1, 2, 8, (3, 4, 6), (1, 2, 2), (2, 2, 2))
    q, k, v, do = rand_inputs(geo, 45)
    qt, kt, vt = rand_text(geo, 0, 46)
    off = rand_offsets(geo, -2, 2, 47)
    (dq, dk, dv), (dqt, _, _) = oracle.backward_prefix(geo, q, k, v, do, off, qt, kt, vt, qt)
    rq, rk, rv = oracle.backward(geo, q, k, v, do, off)
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    assert dqt.size == 0


def test_prefix_backward_sampled_rows_equal_the_full_oracle():
    """The row-sampled prefix backward (used at full sizes) agrees with the full one."""
    geo = oracle.Geometry(1, 2, 8, (4, 4, 6), (2, 2, 2), (2, 1, 2))
    q, k, v, do = rand_inputs(geo, 51)
    L = 6
    qt, kt, vt = rand_text(geo, L, 52)
    dot = rand_text(geo, L, 53)[0]
    off = rand_offsets(geo, -2, 2, 54)
    (dq, dk, dv), (dqt, dkt, dvt) = oracle.backward_prefix(geo, q, k, v, do, off, qt, kt, vt, dot)
    N, h = geo.n_tokens, 1
    qr, kr, tr = np.array([0, 7, N - 1]), np.array([3, 40, N - 2]), np.array([0, L - 1])
    got = oracle.backward_prefix_sampled(geo, q, k, v, do, off, qt, kt, vt, dot, h, qr, tr, kr, tr)
    f = lambda a: np.asarray(a).reshape(geo.B * geo.heads, -1, geo.d)[h]
    refs = (f(dq)[qr], f(dqt)[tr], f(dk)[kr], f(dv)[kr], f(dkt)[tr], f(dvt)[tr])
    for a, b in zip(got, refs):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
