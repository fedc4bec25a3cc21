"""CPU checks of the C ABI: the library loads, exports every declared symbol, and rejects
bad arguments synchronously (no GPU is touched on these paths)."""
import ctypes
import os
import re

import pytest

import video_dit_sparse_dsa_b200 as dsa
from video_dit_sparse_dsa_b200 import build as dsa_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dsa.h")


@pytest.fixture(scope="module")
def lib():
    dsa_build.build()
    return dsa.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names, "no declarations found"
    for n in names:
        assert hasattr(lib, n), f"{n} missing from the library"
    assert set(names) == set(dsa.EXPORTS)


def test_version_and_status_strings(lib):
    assert lib.dsa_version() >= 100
    for code in range(7):
        assert lib.dsa_status_string(code)


def _prob(**kw):
    args = dict(B=1, heads=2, d=128, grid=(16, 32, 32), tile=(4, 8, 8), window=(3, 3, 3), dtype=dsa.DSA_BF16)
    args.update(kw)
    return dsa.make_problem(args["B"], args["heads"], args["d"], args["grid"], args["tile"], args["window"],
                            dtype=args["dtype"])


def test_plan_shape(lib):
    assert dsa.plan_shape(_prob()) == (64, 27)
    assert dsa.plan_shape(_prob(grid=(4, 8, 8), tile=(1, 4, 4), d=64, dtype=dsa.DSA_F32)) == (16, 12)
    assert dsa.plan_shape(_prob(grid=(30, 48, 80), tile=(6, 8, 8))) == (300, 27)


def test_workspace_sizes(lib):
    p = _prob()
    assert dsa.workspace_size(p) >= 4 * (64 * 3 + 64 * 27)
    assert dsa.workspace_size(p, backward=True) > dsa.workspace_size(p)
    bad = _prob(grid=(15, 32, 32))
    assert dsa.workspace_size(bad) == 0


FAKE = ctypes.c_void_p(1 << 20)  # 256-byte aligned, never dereferenced on these paths


def _fwd(lib, p, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, off=FAKE, out=FAKE, lse=FAKE, ws=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    return lib.dsa_fwd(ctypes.byref(p), a["q"], a["k"], a["v"], a["off"], a["out"], a["lse"], a["ws"],
                       a["ws_bytes"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(grid=(15, 32, 32)), 1),            # T not divisible by tt
    (dict(window=(0, 3, 3)), 1),             # empty window
    (dict(B=0), 1),                          # empty batch
    (dict(d=64), 2),                         # bf16 needs d = 128
    (dict(tile=(4, 3, 8), grid=(16, 30, 32)), 2),  # a 128-token chunk is not whole (h, w) planes
    (dict(tile=(1, 8, 8), grid=(16, 32, 32)), 2),  # 64-token tile: no whole 128-token chunk
    (dict(d=96, dtype=dsa.DSA_F32), 2),      # fp32 path: d in {64, 128}
    (dict(B=4096, heads=4096), 2),           # 2^31 or more 128-row units: past the kernel's int32 unit index
    (dict(B=256, heads=512, d=64, dtype=dsa.DSA_F32, grid=(4, 8, 8), tile=(1, 4, 4)), 2),  # fp32 grid y > 65535
])
def test_fwd_rejects_bad_problems(lib, kw, status):
    assert _fwd(lib, _prob(**kw)) == status


def test_fwd_rejects_bad_pointers_and_workspace(lib):
    p = _prob()
    assert _fwd(lib, p, q=None) == 1
    assert _fwd(lib, p, out=ctypes.c_void_p((1 << 20) + 8)) == 1   # misaligned for TMA
    assert _fwd(lib, p, ws=None) == 5
    assert _fwd(lib, p, ws_bytes=16) == 5
    assert _fwd(lib, p, ws=ctypes.c_void_p((1 << 20) + 64)) == 5   # workspace not 256-aligned
    assert lib.dsa_fwd(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == 1
    p.scale = -1.0
    assert _fwd(lib, p) == 1


def test_bwd_rejects_bad_arguments(lib):
    p = _prob()
    f = FAKE
    # 8 x 2 tile planes: the backward refuses them before any launch (LSE / D boxes of 8 bytes)
    narrow = _prob(tile=(16, 8, 2), grid=(32, 16, 8))
    assert lib.dsa_bwd(ctypes.byref(narrow), f, f, f, f, f, f, f, f, f, f, f, 1 << 30, None) == 2
    assert lib.dsa_bwd(ctypes.byref(p), f, f, f, f, f, f, f, f, f, None, f, 1 << 30, None) == 1
    p32 = _prob(d=64, dtype=dsa.DSA_F32, grid=(4, 8, 8), tile=(1, 4, 4))
    assert lib.dsa_bwd(ctypes.byref(p32), f, f, f, f, f, f, f, f, f, f, f, 1 << 30, None) == 2
    assert lib.dsa_bwd(ctypes.byref(p), f, f, f, f, f, f, f, f, f, f, f, 16, None) == 5


def test_list_entry_points_reject_bad_arguments(lib):
    p = _prob()
    f = FAKE
    # forward: (p, q, k, v, row_ptr, list, nnz, per_head, out, lse, stream)
    assert lib.dsa_fwd_list(ctypes.byref(p), f, f, f, None, f, 4, 0, f, f, None) == 1      # no row_ptr
    assert lib.dsa_fwd_list(ctypes.byref(p), f, f, f, f, None, 4, 0, f, f, None) == 1      # nnz > 0 without a list
    assert lib.dsa_fwd_list(ctypes.byref(p), f, f, f, f, f, -1, 0, f, f, None) == 1        # negative nnz
    assert lib.dsa_fwd_list(ctypes.byref(p), f, f, f, f, f, 4, 2, f, f, None) == 1         # per_head not 0 / 1
    assert lib.dsa_fwd_list(ctypes.byref(p), f, f, f, f, f, 4, 0, ctypes.c_void_p((1 << 20) + 8), f, None) == 1
    p32 = _prob(d=64, dtype=dsa.DSA_F32, grid=(4, 8, 8), tile=(1, 4, 4))
    assert lib.dsa_fwd_list(ctypes.byref(p32), f, f, f, f, f, 4, 0, f, f, None) == 2       # bf16 only
    assert lib.dsa_fwd_list(ctypes.byref(_prob(d=64)), f, f, f, f, f, 4, 1, f, f, None) == 2
    # backward: (p, q, k, v, out, lse, dout, row_ptr, list, nnz, per_head, dq, dk, dv, ws, ws_bytes, stream)
    assert lib.dsa_bwd_list(ctypes.byref(p), f, f, f, f, f, f, None, f, 4, 0, f, f, f, f, 1 << 30, None) == 1
    assert lib.dsa_bwd_list(ctypes.byref(p), f, f, f, f, f, f, f, f, 4, 0, f, f, f, f, 16, None) == 5
    assert lib.dsa_bwd_list(ctypes.byref(p), f, f, f, f, f, f, f, f, 4, 1, f, f, f, None, 1 << 30, None) == 5
    # text prefix: (p, q, k, v, offsets, L_text, q_text, k_text, v_text, out, lse, out_text, lse_text, ws,
    # ws_bytes, stream)
    big = 1 << 40
    assert lib.dsa_fwd_prefix(ctypes.byref(p), f, f, f, None, 4, f, f, f, f, f, f, f, f, big, None) == 1
    assert lib.dsa_fwd_prefix(ctypes.byref(p), f, f, f, f, -1, f, f, f, f, f, f, f, f, big, None) == 1
    assert lib.dsa_fwd_prefix(ctypes.byref(p), f, f, f, f, 4, None, f, f, f, f, f, f, f, big, None) == 1
    assert lib.dsa_fwd_prefix(ctypes.byref(p), f, f, f, f, 4, f, f, f, f, f, None, f, f, big, None) == 1
    assert lib.dsa_fwd_prefix(ctypes.byref(p), f, f, f, f, 4, f, ctypes.c_void_p((1 << 20) + 8), f, f, f, f, f,
                              f, big, None) == 1
    assert lib.dsa_fwd_prefix(ctypes.byref(p32), f, f, f, f, 4, f, f, f, f, f, f, f, f, big, None) == 2
    assert lib.dsa_fwd_prefix(ctypes.byref(p), f, f, f, f, 4, f, f, f, f, f, f, f, f, 16, None) == 5
    assert lib.dsa_fwd_prefix(ctypes.byref(p), f, f, f, f, 4, f, f, f, f, f, f, f, None, big, None) == 5
    # prefix backward: (p, q, k, v, out, lse, dout, offsets, L_text, q_text, k_text, v_text, out_text,
    # lse_text, dout_text, dq, dk, dv, dq_text, dk_text, dv_text, ws, ws_bytes, stream)
    fb = [f] * 7
    tb = [f] * 6
    gb = [f] * 6
    assert lib.dsa_bwd_prefix(ctypes.byref(p), *fb[:6], None, 4, *tb, *gb, f, big, None) == 1   # no offsets
    assert lib.dsa_bwd_prefix(ctypes.byref(p), *fb, -3, *tb, *gb, f, big, None) == 1             # negative length
    assert lib.dsa_bwd_prefix(ctypes.byref(p), *fb, 4, None, *tb[1:], *gb, f, big, None) == 1    # text q missing
    assert lib.dsa_bwd_prefix(ctypes.byref(p), *fb, 4, *tb, *gb[:5], None, f, big, None) == 1    # dv_text missing
    assert lib.dsa_bwd_prefix(ctypes.byref(p32), *fb, 4, *tb, *gb, f, big, None) == 2
    assert lib.dsa_bwd_prefix(ctypes.byref(p), *fb, 4, *tb, *gb, f, 16, None) == 5
    b0 = lib.dsa_bwd_prefix_workspace_size(ctypes.byref(p), 0)
    assert 0 < b0 < lib.dsa_bwd_prefix_workspace_size(ctypes.byref(p), 1000)
    assert lib.dsa_bwd_prefix_workspace_size(ctypes.byref(p), -1) == 0
    w0 = lib.dsa_prefix_workspace_size(ctypes.byref(p), 0)
    assert 0 < w0 < lib.dsa_prefix_workspace_size(ctypes.byref(p), 1000)
    assert lib.dsa_prefix_workspace_size(ctypes.byref(p), -1) == 0
    # per-head planner: (p, offsets, row_ptr, list, stream)
    assert lib.dsa_plan_heads(ctypes.byref(p), None, f, f, None) == 1
    assert lib.dsa_plan_heads(ctypes.byref(_prob(window=(0, 1, 1))), f, f, f, None) == 1


def test_list_workspace_sizes(lib):
    p = _prob()
    assert lib.dsa_list_workspace_size(ctypes.byref(p), 100, 0, dsa.DSA_WS_FWD) == 0  # the forward needs none
    small = lib.dsa_list_workspace_size(ctypes.byref(p), 10, 0, dsa.DSA_WS_BWD)
    big = lib.dsa_list_workspace_size(ctypes.byref(p), 10000, 0, dsa.DSA_WS_BWD)
    heads = lib.dsa_list_workspace_size(ctypes.byref(p), 10, 1, dsa.DSA_WS_BWD)
    assert big > small > 4 * (2 * 16 * 32 * 32)  # at least D (dQ needs no accumulator: it is summed in one pass)
    assert heads > small  # an inverse map per head
    assert lib.dsa_list_workspace_size(ctypes.byref(p), -1, 0, dsa.DSA_WS_BWD) == 0


def test_lstsq_rejects_bad_arguments(lib):
    f = FAKE
    # the solve keeps its partial sums in shared memory: no workspace for any size
    assert lib.dsa_lstsq_workspace_size(1000, 3, 24) == 0
    assert lib.dsa_lstsq_workspace_size(1000, 33, 24) == 0
    assert lib.dsa_lstsq_factor(100, 3, None, 0.1, f, None) == 1
    assert lib.dsa_lstsq_factor(100, 3, f, -1.0, f, None) == 1     # negative lambda
    assert lib.dsa_lstsq_factor(100, 40, f, 0.1, f, None) == 2     # p > 32
    assert lib.dsa_lstsq_solve(0, 3, 4, f, f, f, f, None, 0, None) == 1
    assert lib.dsa_lstsq_solve(100, 3, 4, None, f, f, f, None, 0, None) == 1
    assert lib.dsa_lstsq_solve(100, 40, 4, f, f, f, f, None, 0, None) == 2     # p > 32
    assert lib.dsa_lstsq_solve(100, 3, 70000, f, f, f, f, None, 0, None) == 2  # batch > 65535


def test_plan_rejects_half_inverse(lib):
    p = _prob()
    assert lib.dsa_plan(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, None) == 1
    assert lib.dsa_plan(ctypes.byref(p), None, FAKE, FAKE, None, None, None) == 1


def test_product_path_has_no_cpu_fallback(tmp_path):
    with pytest.raises(RuntimeError):
        dsa.load_library(str(tmp_path / "missing.so"))
