"""GPU key-tile-list (block-sparse) forward and backward against the fp64 oracle's list
form: query tile i attends to the key tiles listed for it in a CSR instead of its window
box (the MOD-DiT page, Method section, Stage 2 "Online Block Masking").  Lists here hold
empty rows, repeated tiles and unsorted rows; the window plan written as lists must give
bit-for-bit the output of the window entry point (same kernel, same key order)."""
import numpy as np
import pytest
import torch

import oracle
import video_dit_sparse_dsa_b200 as dsa
from dsa_inputs import Workload, make_inputs
from tests._parity import assert_close, assert_lse_close

pytestmark = pytest.mark.gpu

DSA_ERR_DEVICE = 6


def random_lists(n_tiles, seed, max_len, dup=True):
    """int32 CSR (row_ptr [n_tiles + 1], kv_list [nnz]); row n_tiles // 2 is empty."""
    rng = np.random.default_rng(seed)
    rows = []
    for i in range(n_tiles):
        n = 0 if i == n_tiles // 2 else int(rng.integers(1, max_len + 1))
        rows.append(rng.integers(0, n_tiles, n) if dup else rng.permutation(n_tiles)[:n])
    row_ptr = np.zeros(n_tiles + 1, np.int32)
    row_ptr[1:] = np.cumsum([len(r) for r in rows])
    return row_ptr, np.concatenate(rows).astype(np.int32)


CASES = [
    Workload("list_a", 1, 2, 128, (8, 16, 24), (4, 8, 8), (1, 1, 1), (0, 0), "bf16", 41, backward=True),
    # 384-token tiles: three 128-token chunks per tile, so odd lists end in a half step
    Workload("list_b", 2, 1, 128, (12, 16, 16), (6, 8, 8), (1, 1, 1), (0, 0), "bf16", 42, backward=True),
]


def split_rows(lse, geo, row_ptr):
    """Boolean [B, heads, T, H, W]: token's query tile has an empty list."""
    empty_tiles = np.diff(row_ptr) == 0
    tile_of = np.zeros(geo.n_tokens, np.int64)
    tile_of[geo.tile_token_index().reshape(-1)] = np.repeat(np.arange(geo.n_tiles), geo.tile_tokens)
    return np.broadcast_to(empty_tiles[tile_of].reshape(geo.grid), lse.shape)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_list_forward_against_oracle(w):
    inp = make_inputs(w)
    geo = oracle.Geometry.of(w)
    row_ptr, kv_list = random_lists(geo.n_tiles, w.seed, 7)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    out, lse = dsa.forward_list(q, k, v, torch.from_numpy(row_ptr).cuda(), torch.from_numpy(kv_list).cuda(), w.tile,
                                w.scale)
    st, site, _ = dsa.device_status()
    assert st == 0, f"device status {st} at site {site}"
    ref_o, ref_l = oracle.forward_list(geo, inp.q, inp.k, inp.v, row_ptr, kv_list)
    got_o, got_l = out.float().cpu().numpy(), lse.cpu().numpy()
    empty = split_rows(got_l, geo, row_ptr)
    assert empty.any() and not empty.all()
    assert np.all(got_o[empty] == 0.0) and np.all(np.isneginf(got_l[empty]))
    assert_close(got_o[~empty], ref_o[~empty], "bf16", "out")
    assert_lse_close(got_l[~empty], ref_l[~empty], "bf16")


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_list_backward_against_oracle(w):
    inp = make_inputs(w)
    geo = oracle.Geometry.of(w)
    row_ptr, kv_list = random_lists(geo.n_tiles, w.seed + 100, 6)
    q, k, v, dout = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.dout.cuda()
    rp, kl = torch.from_numpy(row_ptr).cuda(), torch.from_numpy(kv_list).cuda()
    out, lse = dsa.forward_list(q, k, v, rp, kl, w.tile, w.scale)
    dq, dk, dv = dsa.backward_list(q, k, v, out, lse, dout, rp, kl, w.tile, w.scale)
    st, site, _ = dsa.device_status()
    assert st == 0, f"device status {st} at site {site}"
    rq, rk, rv = oracle.backward_list(geo, inp.q, inp.k, inp.v, inp.dout, row_ptr, kv_list)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        assert_close(got.float().cpu().numpy(), ref, "bf16", name)


# The window form of tiles with an even number of 128-token chunks runs on the CTA-pair
# kernel, the list form always on the single-CTA kernel: with the plan's windows as lists
# the two must agree bit for bit (same products in the same order, same softmax).
PLAN_AS_LISTS = [
    Workload("list_plan_s3", 1, 2, 128, (12, 16, 24), (6, 8, 8), (3, 1, 3), (-1, 1), "bf16", 43),  # single vs single
    Workload("list_plan_s2", 2, 2, 128, (12, 16, 24), (4, 8, 8), (3, 3, 3), (-2, 2), "bf16", 44),  # pair vs single
    Workload("list_plan_s4", 1, 3, 128, (16, 16, 24), (8, 8, 8), (1, 3, 3), (-1, 1), "bf16", 45),  # 2 pairs per tile
]


@pytest.mark.parametrize("w", PLAN_AS_LISTS, ids=lambda w: w.name)
def test_window_plan_as_lists_is_bit_exact(w):
    inp = make_inputs(w)
    geo = oracle.Geometry.of(w)
    q, k, v, off = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.offsets.cuda()
    out_box, lse_box = dsa.forward(q, k, v, off, w.tile, w.window, w.scale)
    p = dsa.make_problem(w.B, w.heads, w.d, w.grid, w.tile, w.window, w.scale)
    _, kv = dsa.plan(p, off, inverse=False)
    row_ptr = torch.arange(0, geo.n_tiles + 1, dtype=torch.int32, device="cuda") * kv.shape[1]
    out_l, lse_l = dsa.forward_list(q, k, v, row_ptr, kv.reshape(-1).contiguous(), w.tile, w.scale)
    assert dsa.device_status()[0] == 0
    assert torch.equal(out_l, out_box) and torch.equal(lse_l, lse_box)


def test_empty_lists_give_zero_and_minus_infinity():
    w = CASES[0]
    inp = make_inputs(w)
    geo = oracle.Geometry.of(w)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    rp = torch.zeros(geo.n_tiles + 1, dtype=torch.int32, device="cuda")
    out, lse = dsa.forward_list(q, k, v, rp, None, w.tile, w.scale)
    assert dsa.device_status()[0] == 0
    assert torch.count_nonzero(out).item() == 0 and bool(torch.isneginf(lse).all())


def test_invalid_lists_are_reported_not_faulted():
    """Out-of-range tiles and a decreasing row_ptr: the device check records a bounds
    error; the kernels clamp every index taken from the lists, so nothing outside the
    buffers is touched."""
    w = CASES[0]
    inp = make_inputs(w)
    geo = oracle.Geometry.of(w)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    row_ptr, kv_list = random_lists(geo.n_tiles, 7, 4)
    bad_list = kv_list.copy()
    bad_list[0] = geo.n_tiles + 5
    bad_list[-1] = -3
    out, lse = dsa.forward_list(q, k, v, torch.from_numpy(row_ptr).cuda(), torch.from_numpy(bad_list).cuda(), w.tile,
                                w.scale)
    st, site, _ = dsa.device_status()
    assert st == DSA_ERR_DEVICE and site == 92
    bad_ptr = row_ptr.copy()
    bad_ptr[3], bad_ptr[4] = bad_ptr[4], bad_ptr[3] - 1  # a decreasing step
    dsa.forward_list(q, k, v, torch.from_numpy(bad_ptr).cuda(), torch.from_numpy(kv_list).cuda(), w.tile, w.scale)
    st, site, _ = dsa.device_status()
    assert st == DSA_ERR_DEVICE and site in (90, 91)
    # the library is still usable afterwards
    dsa.forward_list(q, k, v, torch.from_numpy(row_ptr).cuda(), torch.from_numpy(kv_list).cuda(), w.tile, w.scale)
    assert dsa.device_status()[0] == 0


def test_block_sparse_lists_at_480p_sampled():
    """MOD-DiT-like block masks on the 480p-shaped grid: every query tile keeps 40 key tiles
    chosen at random (of 140), compared with the oracle on sampled query tiles."""
    w = Workload("list_480p", 1, 12, 128, (20, 32, 56), (4, 8, 8), (1, 1, 1), (0, 0), "bf16", 44)
    inp = make_inputs(w)
    geo = oracle.Geometry.of(w)
    rng = np.random.default_rng(5)
    rows = [np.sort(rng.permutation(geo.n_tiles)[:40]) for _ in range(geo.n_tiles)]
    row_ptr = np.arange(geo.n_tiles + 1, dtype=np.int32) * 40
    kv_list = np.concatenate(rows).astype(np.int32)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    out, lse = dsa.forward_list(q, k, v, torch.from_numpy(row_ptr).cuda(), torch.from_numpy(kv_list).cuda(), w.tile,
                                w.scale)
    assert dsa.device_status()[0] == 0
    bh = rng.integers(0, w.B * w.heads, 8).astype(np.int32)
    tiles = rng.integers(0, geo.n_tiles, 8).astype(np.int32)
    ref_o, ref_l = oracle.forward_list(geo, inp.q, inp.k, inp.v, row_ptr, kv_list, sel=(bh, tiles))
    tok = geo.tile_token_index()
    flat_o = out.reshape(w.B * w.heads, geo.n_tokens, w.d)
    flat_l = lse.reshape(w.B * w.heads, geo.n_tokens)
    for s in range(len(bh)):
        idx = torch.as_tensor(tok[tiles[s]], device="cuda", dtype=torch.long)
        assert_close(flat_o[int(bh[s])][idx].float().cpu().numpy(), ref_o[s], "bf16", f"out sample {s}")
        assert_lse_close(flat_l[int(bh[s])][idx].cpu().numpy(), ref_l[s], "bf16")


def per_head_lists(geo, B, heads, seed, max_len):
    rps, lists, base = [], [], 0
    for h in range(B * heads):
        rp, kl = random_lists(geo.n_tiles, seed + h, max_len)
        rps.append(rp + base)
        lists.append(kl)
        base += len(kl)
    return np.stack(rps).astype(np.int32), np.concatenate(lists).astype(np.int32)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_per_head_lists_against_oracle(w):
    """Head-adaptive sparsity: a different key-tile list for every (batch, head)."""
    inp = make_inputs(w)
    geo = oracle.Geometry.of(w)
    row_ptr, kv_list = per_head_lists(geo, w.B, w.heads, w.seed + 200, 6)
    q, k, v, dout = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.dout.cuda()
    rp, kl = torch.from_numpy(row_ptr).cuda(), torch.from_numpy(kv_list).cuda()
    out, lse = dsa.forward_list(q, k, v, rp, kl, w.tile, w.scale)
    dq, dk, dv = dsa.backward_list(q, k, v, out, lse, dout, rp, kl, w.tile, w.scale)
    st, site, _ = dsa.device_status()
    assert st == 0, f"device status {st} at site {site}"
    ref_o, ref_l = oracle.forward_list(geo, inp.q, inp.k, inp.v, row_ptr, kv_list)
    got_o, got_l = out.float().cpu().numpy(), lse.cpu().numpy()
    fin = np.isfinite(ref_l)
    assert not fin.all() and np.all(np.isneginf(got_l[~fin])) and np.all(got_o[~fin] == 0.0)
    assert_close(got_o[fin], ref_o[fin], "bf16", "out")
    assert_lse_close(got_l[fin], ref_l[fin], "bf16")
    rq, rk, rv = oracle.backward_list(geo, inp.q, inp.k, inp.v, inp.dout, row_ptr, kv_list)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        assert_close(got.float().cpu().numpy(), ref, "bf16", name)


def test_per_head_offsets_against_the_windowed_oracle():
    """Per-(batch, head) window offsets, planned on the device into per-head lists, against
    the oracle's window form run head by head with that head's offsets."""
    w = Workload("heads_offsets", 2, 2, 128, (8, 16, 24), (4, 8, 8), (3, 1, 3), (-2, 2), "bf16", 45, backward=True)
    inp = make_inputs(w)
    geo = oracle.Geometry.of(w)
    BH = w.B * w.heads
    g = torch.Generator().manual_seed(99)
    offs = torch.randint(-2, 3, (BH, geo.n_tiles, 3), generator=g).to(torch.int32)
    p = dsa.make_problem(w.B, w.heads, w.d, w.grid, w.tile, w.window, w.scale)
    rp, kl = dsa.plan_heads(p, offs.cuda())
    q, k, v, dout = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.dout.cuda()
    out, lse = dsa.forward_list(q, k, v, rp, kl, w.tile, w.scale)
    dq, dk, dv = dsa.backward_list(q, k, v, out, lse, dout, rp, kl, w.tile, w.scale)
    assert dsa.device_status()[0] == 0
    one = oracle.Geometry(1, 1, w.d, w.grid, w.tile, w.window, w.scale)
    for h in range(BH):
        b, j = divmod(h, w.heads)
        sl = [t[b:b + 1, j:j + 1] for t in (inp.q, inp.k, inp.v, inp.dout)]
        ref_o, ref_l = oracle.forward(one, sl[0], sl[1], sl[2], offs[h])
        assert_close(out[b, j].float().cpu().numpy(), ref_o[0, 0], "bf16", f"out head {h}")
        assert_lse_close(lse[b, j].cpu().numpy(), ref_l[0, 0], "bf16")
        rq, rk, rv = oracle.backward(one, *sl, offs[h])
        for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            assert_close(got[b, j].float().cpu().numpy(), ref[0, 0], "bf16", f"{name} head {h}")


# ------------------------------------------------------------------------------------
# block attention mass (sparsity map).  Tolerance: an entry is a mean of probabilities
# exp(s - lse) <= 1.  The scores are exact products of the bf16 inputs summed in fp32
# (relative error ~1e-6); lse is the forward's, whose error against the exact value is the
# relative error of its row sum (fp32 sum of 2^x, each with relative error <= 7.6e-5 on the
# FMA-pipe share, ~1e-7 on MUFU: well under 1e-4); each probability adds its own 2^x error
# (<= 7.6e-5).  So an entry's relative error is below 2e-4 and, as entries are <= 1, its
# absolute error too: max-abs 5e-4 (and row sums within 5e-4 of 1) keeps a margin of 2.5x.
MAP_MAX_ABS = 5e-4


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("per_head", [False, True], ids=["shared", "per_head"])
def test_block_map_against_oracle(w, per_head):
    inp = make_inputs(w)
    geo = oracle.Geometry.of(w)
    if per_head:
        row_ptr, kv_list = per_head_lists(geo, w.B, w.heads, w.seed + 300, 6)
    else:
        row_ptr, kv_list = random_lists(geo.n_tiles, w.seed + 300, 6)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    rp, kl = torch.from_numpy(row_ptr).cuda(), torch.from_numpy(kv_list).cuda()
    _, lse = dsa.forward_list(q, k, v, rp, kl, w.tile, w.scale)
    bm = dsa.block_map(q, k, lse, rp, kl, w.tile, w.scale)
    st, site, _ = dsa.device_status()
    assert st == 0, f"device status {st} at site {site}"
    # one CTA sums each row of the map in a fixed order: a second run gives the same bits
    assert torch.equal(dsa.block_map(q, k, lse, rp, kl, w.tile, w.scale), bm)
    ref = oracle.block_map_list(geo, inp.q, inp.k, row_ptr, kv_list)
    got = bm.cpu().numpy()
    err = np.abs(got - ref).max()
    assert err <= MAP_MAX_ABS, f"block map max-abs {err:.2e}"
    sums = got.sum(axis=-1)
    ref_sums = ref.sum(axis=-1)
    assert np.all(np.abs(sums[ref_sums > 0] - 1.0) <= MAP_MAX_ABS)
    assert np.all(sums[ref_sums == 0] == 0.0)


def test_dense_block_map_sampled():
    """Dense attention (every tile listed for every query tile) on the 16x32x32 grid: the
    block map of sampled query tiles against the oracle; every row sums to one."""
    w = Workload("dense_map", 1, 4, 128, (16, 32, 32), (4, 8, 8), (1, 1, 1), (0, 0), "bf16", 46)
    inp = make_inputs(w)
    geo = oracle.Geometry.of(w)
    n = geo.n_tiles
    row_ptr = torch.arange(n + 1, dtype=torch.int32, device="cuda") * n
    kv_list = torch.arange(n, dtype=torch.int32, device="cuda").repeat(n).contiguous()
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    _, lse = dsa.forward_list(q, k, v, row_ptr, kv_list, w.tile, w.scale)
    bm = dsa.block_map(q, k, lse, row_ptr, kv_list, w.tile, w.scale)
    assert dsa.device_status()[0] == 0
    got = bm.cpu().numpy()
    np.testing.assert_allclose(got.sum(axis=-1), 1.0, rtol=0, atol=MAP_MAX_ABS)
    rng = np.random.default_rng(8)
    bh = rng.integers(0, w.B * w.heads, 6).astype(np.int32)
    tiles = rng.integers(0, n, 6).astype(np.int32)
    ref = oracle.block_map_list(geo, inp.q, inp.k, row_ptr.cpu().numpy(), kv_list.cpu().numpy(), sel=(bh, tiles))
    for s in range(len(bh)):
        err = np.abs(got[bh[s], tiles[s]] - ref[s]).max()
        assert err <= MAP_MAX_ABS, f"sample {s}: max-abs {err:.2e}"
