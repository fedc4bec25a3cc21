"""GPU window planner against the oracle's plan, bit for bit (starts, key-tile lists and
the inverse CSR), on every workload and on random grids, windows and offsets."""
import numpy as np
import pytest
import torch

import oracle
import video_dit_sparse_dsa_b200 as dsa
from dsa_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _gpu_plan(G, window, offsets):
    p = dsa.make_problem(1, 1, 128, G, (1, 1, 1), window)
    off = torch.as_tensor(np.asarray(offsets, np.int32)).cuda().contiguous()
    starts, kv, row_ptr, q_tiles = dsa.plan(p, off)
    torch.cuda.synchronize()
    return starts.cpu().numpy(), kv.cpu().numpy(), row_ptr.cpu().numpy(), q_tiles.cpu().numpy()


def _compare(G, window, offsets):
    s, kv, rp, qt = _gpu_plan(G, window, offsets)
    s0, kv0, rp0, qt0 = oracle.plan(G, window, offsets)
    np.testing.assert_array_equal(s, s0)
    np.testing.assert_array_equal(kv, kv0)
    np.testing.assert_array_equal(rp, rp0)
    np.testing.assert_array_equal(qt, qt0)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_plan_workloads(name):
    w = WORKLOADS[name]
    inp = make_inputs(w.replace(heads=1, B=1) if w.dtype == "bf16" else w)
    _compare(w.tile_grid, w.window, inp.offsets.numpy())


def test_plan_random():
    rng = np.random.default_rng(123)
    for _ in range(60):
        G = [int(x) for x in rng.integers(1, 9, size=3)]
        window = [int(x) for x in rng.integers(1, 10, size=3)]
        n = G[0] * G[1] * G[2]
        off = rng.integers(-10, 11, size=(n, 3)).astype(np.int32)
        _compare(G, window, off)


def test_plan_large_grid_inverse():
    """More tiles than one 1024-thread pass of the planner (scan carries across passes)."""
    G = (12, 15, 16)
    rng = np.random.default_rng(5)
    off = rng.integers(-3, 4, size=(G[0] * G[1] * G[2], 3)).astype(np.int32)
    _compare(G, (3, 5, 3), off)


def test_plan_extreme_offsets_pin_edges():
    G = (5, 6, 10)
    n = G[0] * G[1] * G[2]
    for o in (-100, 100):
        off = np.full((n, 3), o, np.int32)
        s, kv, _, _ = _gpu_plan(G, (3, 3, 3), off)
        expect = 0 if o < 0 else np.array(G) - 3
        assert (s == expect).all()
        _compare(G, (3, 3, 3), off)
