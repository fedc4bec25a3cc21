"""The forward entry point that allocates nothing (dsa_fwd_noalloc), called through the C ABI.

It exists for callers that cannot allocate device memory at call time: a plugin whose host
engine owns all device memory, a loop that must not call cudaMalloc because it can
synchronize the device, a process whose memory budget was fixed at start-up.  Its scratch
is a fixed array of 65536 int32 inside the library.  It runs the same planner and forward
kernel as dsa_fwd, so its output must be bit-identical to dsa_fwd's.  This file checks
that on two calls in a row (different problems, so the second call must fully replace the
first call's plan), on a problem whose plan fills the array exactly, and that the first
problem past the limit (accepted by dsa_fwd) is refused.  The file sorts last so a run
that stops at the first failure has run every other test before it."""
import ctypes

import pytest
import torch

import video_dit_sparse_dsa_b200 as dsa
from dsa_inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

CAPACITY = 65536  # int32 entries of the fixed scratch array

CALLS = [
    Workload("noalloc_a", 1, 3, 128, (12, 16, 24), (6, 8, 8), (3, 3, 3), (-2, 2), "bf16", 41),
    Workload("noalloc_b", 2, 2, 128, (8, 24, 32), (4, 8, 8), (3, 1, 5), (-1, 1), "bf16", 42),
]

# tile grid 32 x 8 x 8 = 2048 tiles, window 29 x 1 x 1: roundup(3 * 2048, 64) + 2048 * 29
# = 6144 + 59392 = 65536 entries, the whole array
AT_CAPACITY = Workload("noalloc_full", 1, 1, 128, (64, 64, 64), (2, 8, 8), (29, 1, 1), (-2, 2), "bf16", 44)
# the same grid with a 30-tile window: 6144 + 61440 = 67584 entries, past the array
PAST_CAPACITY = AT_CAPACITY.replace(name="noalloc_over", window=(30, 1, 1))


def plan_entries(w: Workload) -> int:
    return (3 * w.n_tiles + 63) // 64 * 64 + w.n_tiles * w.window_tiles


def _noalloc(lib, w, q, k, v, off, out, lse):
    p = dsa.make_problem(w.B, w.heads, w.d, w.grid, w.tile, w.window, w.scale, dsa.DSA_BF16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.dsa_fwd_noalloc(ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                               ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(off.data_ptr()),
                               ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), stream)


def _check_against_dsa_fwd(lib, w):
    inp = make_inputs(w)
    q, k, v, off = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.offsets.cuda()
    ref_out, ref_lse = dsa.forward(q, k, v, off, w.tile, w.window, w.scale)
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:5], float("nan"), device=q.device)
    assert _noalloc(lib, w, q, k, v, off, out, lse) == 0
    st = dsa.device_status()
    assert st[0] == 0, f"device status {st}"
    # same planner, same kernel, same plan: the results are identical bit for bit
    assert torch.equal(out, ref_out), f"{w.name}: out differs from dsa_fwd"
    assert torch.equal(lse, ref_lse), f"{w.name}: lse differs from dsa_fwd"


def test_noalloc_two_calls_match_dsa_fwd():
    lib = dsa.load_library()
    for w in CALLS:
        _check_against_dsa_fwd(lib, w)


def test_noalloc_plan_filling_the_array_matches_dsa_fwd():
    assert plan_entries(AT_CAPACITY) == CAPACITY
    _check_against_dsa_fwd(dsa.load_library(), AT_CAPACITY)


def test_noalloc_refuses_first_problem_past_the_array():
    lib = dsa.load_library()
    w = PAST_CAPACITY
    assert plan_entries(w) > CAPACITY
    inp = make_inputs(w)
    q, k, v, off = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.offsets.cuda()
    # dsa_fwd takes this problem (its kernel limits allow it) ...
    out, lse = dsa.forward(q, k, v, off, w.tile, w.window, w.scale)
    torch.cuda.synchronize()
    assert torch.isfinite(lse).all()
    # ... the no-allocation forward refuses it for its fixed scratch alone, before launching
    out2 = torch.full_like(q, float("nan"))
    lse2 = torch.full(q.shape[:5], float("nan"), device=q.device)
    assert _noalloc(lib, w, q, k, v, off, out2, lse2) == 2
    torch.cuda.synchronize()
    assert torch.isnan(lse2).all()
