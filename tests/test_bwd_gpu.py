"""GPU backward (dQ, dK, dV of sum(O * dO)) against the fp64 oracle.

Small problems are compared in full; the full-size adaptation workload on two whole
(batch, head) slices and on sampled query tiles (dQ) and key tiles (dK, dV) of the others,
with the forward outputs the GPU produced."""
import numpy as np
import pytest
import torch

import oracle
import video_dit_sparse_dsa_b200 as dsa
from dsa_inputs import WORKLOADS, Workload, make_inputs
from tests._parity import assert_close

pytestmark = pytest.mark.gpu


def run_gpu(w: Workload, inp):
    q, k, v, dout = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.dout.cuda()
    off = inp.offsets.cuda()
    out, lse = dsa.forward(q, k, v, off, w.tile, w.window, w.scale)
    dq, dk, dv = dsa.backward(q, k, v, out, lse, dout, off, w.tile, w.window, w.scale)
    st, site, block = dsa.device_status()
    assert st == 0, f"device status {st} at site {site} block {block}"
    return dq, dk, dv


SMALL = [
    Workload("bwd_small_a", 1, 2, 128, (8, 16, 24), (4, 8, 8), (3, 3, 3), (-2, 2), "bf16", 31, backward=True),
    Workload("bwd_small_b", 2, 1, 128, (12, 16, 16), (6, 8, 8), (5, 3, 1), (-1, 1), "bf16", 32, backward=True),
    Workload("bwd_small_c", 1, 2, 128, (16, 8, 8), (8, 4, 4), (1, 3, 3), (-1, 1), "bf16", 33, backward=True),
    # offsets of 3 leave some key tiles in no window at all: their dK, dV must be zero
    Workload("bwd_small_shift", 1, 1, 128, (8, 32, 32), (4, 8, 8), (1, 1, 1), (3, 3), "bf16", 34, backward=True),
    # 64 (batch, head) slices on a small grid
    Workload("bwd_many_heads", 4, 16, 128, (4, 16, 8), (4, 8, 8), (1, 3, 1), (-1, 1), "bf16", 35, backward=True),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_bwd_small_full(w):
    inp = make_inputs(w)
    dq, dk, dv = run_gpu(w, inp)
    geo = oracle.Geometry.of(w)
    rq, rk, rv = oracle.backward(geo, inp.q, inp.k, inp.v, inp.dout, inp.offsets)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        assert_close(got.float().cpu().numpy(), ref, "bf16", name)


def test_bwd_adaptation_workload_sampled():
    """The full-size adaptation workload (B2 h12, 480p grid, 140 tiles, 3x3x5 windows):
    every dQ, dK, dV element of two whole (batch, head) slices (the first and the last, so
    every tile, both grid corners and every in-degree of the inverse plan), then 16 query
    tiles (dQ) and 16 key tiles (dK, dV) spread over the other slices: the key tiles with the
    largest and the smallest inverse-plan rows, the eight grid corners and random tiles."""
    w = WORKLOADS["adapt_480p_b2"]
    inp = make_inputs(w)
    dq, dk, dv = run_gpu(w, inp)
    geo = oracle.Geometry.of(w)
    BH = w.B * w.heads
    tok = geo.tile_token_index()
    rng = np.random.default_rng(1)

    def head(t, bh):
        return t.reshape(BH, geo.n_tokens, w.d)[bh].float().cpu().numpy()

    for bh in (0, BH - 1):
        ref = oracle.backward_head(geo, inp.q, inp.k, inp.v, inp.dout, inp.offsets, bh)
        for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            assert_close(head(got, bh), r, "bf16", f"{name} of (batch, head) {bh}")

    def gather(t, bh, tiles):
        flat = t.reshape(BH, geo.n_tokens, w.d)
        ib = torch.as_tensor(np.repeat(bh, geo.tile_tokens), device=t.device, dtype=torch.long)
        it = torch.as_tensor(tok[tiles].reshape(-1), device=t.device, dtype=torch.long)
        return flat[ib, it].float().cpu().numpy().reshape(len(bh), geo.tile_tokens, w.d)

    _, _, row_ptr, _ = oracle.plan(geo.G, geo.window, inp.offsets)
    indeg = np.diff(row_ptr)
    Gt, Gh, Gw = geo.G
    corners = [(t * Gh + h) * Gw + x for t in (0, Gt - 1) for h in (0, Gh - 1) for x in (0, Gw - 1)]
    kt = np.array([int(np.argmax(indeg)), int(np.argmin(indeg))] + corners, np.int32)
    kt = np.concatenate([kt, rng.choice(geo.n_tiles, 16 - len(kt), replace=False)]).astype(np.int32)
    kb = rng.integers(1, BH - 1, len(kt)).astype(np.int32)
    ref_dk, ref_dv = oracle.backward_dkdv_tiles(geo, inp.q, inp.k, inp.v, inp.dout, inp.offsets, (kb, kt))
    assert_close(gather(dk, kb, kt), ref_dk, "bf16", "dk")
    assert_close(gather(dv, kb, kt), ref_dv, "bf16", "dv")
    qt = np.concatenate([np.array(corners, np.int32), rng.choice(geo.n_tiles, 8, replace=False)]).astype(np.int32)
    qb = rng.integers(1, BH - 1, len(qt)).astype(np.int32)
    ref_dq = oracle.backward_dq_tiles(geo, inp.q, inp.k, inp.v, inp.dout, inp.offsets, (qb, qt))
    assert_close(gather(dq, qb, qt), ref_dq, "bf16", "dq")


def test_bwd_every_gradient_written():
    w = SMALL[3]
    inp = make_inputs(w)
    q, k, v, dout, off = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.dout.cuda(), inp.offsets.cuda()
    out, lse = dsa.forward(q, k, v, off, w.tile, w.window, w.scale)
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    dsa.backward(q, k, v, out, lse, dout, off, w.tile, w.window, w.scale, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()


def test_bwd_is_bit_identical_across_runs():
    """dQ is summed by one CTA per query row in the fixed order of the row's key list, dK and
    dV by one CTA per key row in the fixed order of the inverse lists: two runs of the
    backward on the same inputs give the same bits (the adaptation grid, 4 heads)."""
    w = WORKLOADS["adapt_480p_b2"].replace(name="bwd_repeat", B=1, heads=4, seed=36)
    inp = make_inputs(w)
    q, k, v, dout, off = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.dout.cuda(), inp.offsets.cuda()
    out, lse = dsa.forward(q, k, v, off, w.tile, w.window, w.scale)
    first = dsa.backward(q, k, v, out, lse, dout, off, w.tile, w.window, w.scale)
    for _ in range(2):
        again = dsa.backward(q, k, v, out, lse, dout, off, w.tile, w.window, w.scale)
        for a, b, name in zip(first, again, ("dq", "dk", "dv")):
            assert torch.equal(a, b), f"{name} differs between runs"
    st = dsa.device_status()
    assert st[0] == 0, f"device status {st}"
