"""The forward entry point that allocates nothing (dsa_fwd_noalloc), called through the C ABI.

It exists for callers that cannot allocate device memory at call time: a plugin whose host
engine owns all device memory, a loop that must not call cudaMalloc because it can
synchronize the device, a process whose memory budget was fixed at start-up.  Its scratch
is a fixed array inside the library; this test checks two calls in a row (different
problems, so the second call must fully replace the first call's plan) against dsa_fwd,
and that a problem too large for the fixed array is refused.  The file sorts last so a
run that stops at the first failure has run every other test before it."""
import ctypes

import pytest
import torch

import video_dit_sparse_dsa_b200 as dsa
from dsa_inputs import Workload, make_inputs
from tests._parity import assert_close, assert_lse_close

pytestmark = pytest.mark.gpu

CALLS = [
    Workload("noalloc_a", 1, 3, 128, (12, 16, 24), (6, 8, 8), (3, 3, 3), (-2, 2), "bf16", 41),
    Workload("noalloc_b", 2, 2, 128, (8, 24, 32), (4, 8, 8), (3, 1, 5), (-1, 1), "bf16", 42),
]


def _noalloc(lib, w, q, k, v, off, out, lse):
    p = dsa.make_problem(w.B, w.heads, w.d, w.grid, w.tile, w.window, w.scale, dsa.DSA_BF16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.dsa_fwd_noalloc(ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                               ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(off.data_ptr()),
                               ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), stream)


def test_noalloc_two_calls_match_dsa_fwd():
    lib = dsa.load_library()
    for w in CALLS:
        inp = make_inputs(w)
        q, k, v, off = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.offsets.cuda()
        ref_out, ref_lse = dsa.forward(q, k, v, off, w.tile, w.window, w.scale)
        out = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:5], float("nan"), device=q.device)
        assert _noalloc(lib, w, q, k, v, off, out, lse) == 0
        st = dsa.device_status()
        assert st[0] == 0, f"device status {st}"
        assert_close(out.float().cpu().numpy(), ref_out.float().cpu().numpy(), "bf16", f"{w.name} out")
        assert_lse_close(lse.cpu().numpy(), ref_lse.cpu().numpy(), "bf16", f"{w.name} lse")


def test_noalloc_rejects_problem_beyond_fixed_scratch():
    lib = dsa.load_library()
    # 64 x 32 x 32 tiles with a 5x5x5 window: 65536 tiles x 125 entries, far beyond 65536 ints
    w = Workload("noalloc_big", 1, 1, 128, (64, 256, 256), (1, 8, 16), (5, 5, 5), (0, 0), "bf16", 43)
    p = dsa.make_problem(w.B, w.heads, w.d, w.grid, w.tile, w.window, w.scale, dsa.DSA_BF16)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    st = lib.dsa_fwd_noalloc(ctypes.byref(p), fake, fake, fake, fake, fake, fake, None)
    assert st == 2
