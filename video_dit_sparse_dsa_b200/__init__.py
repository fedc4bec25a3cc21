"""3D Deformable Slide Attention (3D-DSA) on NVIDIA B200 (sm_100a).

Thin Python binding of the C ABI in ``include/dsa.h`` (argument marshalling only: every
step of the computation runs in the library's CUDA kernels).  PyTorch provides device
memory and streams.  The library is built in-tree by ``video_dit_sparse_dsa_b200.build``;
if it is missing, every entry point raises: there is no CPU fallback.

Operator ("MegaSlide-DiT: Memory-Centric Adaptation and Deformable Local Attention for
Efficient Video Diffusion", abstract; tile-granular window as in "Fast Video Generation
with Sliding Tile Attention", abstract): for query tile i with integer offset o, the
window of w' = min(w, G) tiles per axis starts at clamp(i + o - floor(w'/2), 0, G - w');
each query token attends with softmax(scale q K^T) V to exactly the tokens of those tiles.

Tensors: q, k, v, out, dout, dq, dk, dv are ``[B, heads, T, H, W, d]`` contiguous CUDA
tensors (bf16 with d = 128, or fp32 with d in {64, 128} for the forward); lse is
``[B, heads, T, H, W]`` fp32; tile offsets are int32 ``[nTiles, 3]`` in tile units.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libdsa_b200.so")

DSA_F32, DSA_BF16 = 0, 1
DSA_WS_FWD, DSA_WS_BWD = 0, 1
_STATUS = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_CUDA",
           4: "DSA_ERR_TIMEOUT", 5: "DSA_ERR_WORKSPACE", 6: "DSA_ERR_DEVICE"}

# kernel launches of one dsa_fwd call (planner, forward) and of one dsa_bwd call (planner,
# the inverse map's count, scan and fill, D preprocess, backward, dQ conversion)
FWD_LAUNCHES = 2
BWD_LAUNCHES = 7

# every symbol include/dsa.h declares
EXPORTS = ("dsa_version", "dsa_status_string", "dsa_plan_shape", "dsa_workspace_size", "dsa_plan", "dsa_fwd",
           "dsa_fwd_host_bytes", "dsa_fwd_host", "dsa_bwd", "dsa_device_status", "dsa_fwd_noalloc",
           "dsa_list_workspace_size", "dsa_fwd_list", "dsa_bwd_list", "dsa_plan_heads", "dsa_block_map",
           "dsa_lstsq_workspace_size", "dsa_lstsq_factor", "dsa_lstsq_solve", "dsa_prefix_workspace_size",
           "dsa_fwd_prefix", "dsa_bwd_prefix_workspace_size", "dsa_bwd_prefix", "dsa_selftest_wait")


class DsaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_STATUS.get(status, status)}")


class Problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("heads", ctypes.c_int32), ("d", ctypes.c_int32), ("T", ctypes.c_int32),
                ("H", ctypes.c_int32), ("W", ctypes.c_int32), ("tile", ctypes.c_int32 * 3),
                ("window", ctypes.c_int32 * 3), ("scale", ctypes.c_float), ("dtype", ctypes.c_int32)]


_lib = None


def load_library(path: Optional[str] = None):
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"3D-DSA CUDA library not built ({p}); run python -m video_dit_sparse_dsa_b200.build")
    lib = ctypes.CDLL(p)
    vp, sz, i32, i32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)
    pp = ctypes.POINTER(Problem)
    lib.dsa_version.restype = i32
    lib.dsa_version.argtypes = []
    lib.dsa_status_string.restype = ctypes.c_char_p
    lib.dsa_status_string.argtypes = [ctypes.c_int]
    lib.dsa_plan_shape.argtypes = [pp, i32p, i32p]
    lib.dsa_workspace_size.restype = sz
    lib.dsa_workspace_size.argtypes = [pp, i32]
    lib.dsa_plan.argtypes = [pp, vp, vp, vp, vp, vp, vp]
    lib.dsa_fwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dsa_fwd_host_bytes.restype = sz
    lib.dsa_fwd_host_bytes.argtypes = [pp]
    lib.dsa_fwd_host.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dsa_bwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dsa_device_status.argtypes = [vp, i32p, i32p]
    lib.dsa_fwd_noalloc.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp]
    lib.dsa_list_workspace_size.restype = sz
    lib.dsa_list_workspace_size.argtypes = [pp, i32, i32, i32]
    lib.dsa_fwd_list.argtypes = [pp, vp, vp, vp, vp, vp, i32, i32, vp, vp, vp]
    lib.dsa_bwd_list.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, sz, vp]
    lib.dsa_plan_heads.argtypes = [pp, vp, vp, vp, vp]
    lib.dsa_block_map.argtypes = [pp, vp, vp, vp, vp, vp, i32, i32, vp, vp]
    lib.dsa_lstsq_workspace_size.restype = sz
    lib.dsa_lstsq_workspace_size.argtypes = [i32, i32, i32]
    lib.dsa_lstsq_factor.argtypes = [i32, i32, vp, ctypes.c_float, vp, vp]
    lib.dsa_lstsq_solve.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, sz, vp]
    lib.dsa_prefix_workspace_size.restype = sz
    lib.dsa_prefix_workspace_size.argtypes = [pp, i32]
    lib.dsa_fwd_prefix.argtypes = [pp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dsa_selftest_wait.argtypes = [vp]
    lib.dsa_bwd_prefix_workspace_size.restype = sz
    lib.dsa_bwd_prefix_workspace_size.argtypes = [pp, i32]
    lib.dsa_bwd_prefix.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                   vp, vp, sz, vp]
    for name in ("dsa_plan_shape", "dsa_plan", "dsa_fwd", "dsa_fwd_host", "dsa_bwd", "dsa_device_status",
                 "dsa_fwd_noalloc", "dsa_fwd_list", "dsa_bwd_list", "dsa_plan_heads", "dsa_block_map",
                 "dsa_lstsq_factor", "dsa_lstsq_solve", "dsa_fwd_prefix", "dsa_bwd_prefix",
                 "dsa_selftest_wait"):
        getattr(lib, name).restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def head_range(n_slices: int, rank: int, world: int):
    """The (batch, head) slices [lo, hi) of a problem with n_slices = B * heads that rank
    `rank` of `world` takes when one problem is split over GPUs by heads.  Slices are
    independent problems (each has its own softmax), so ranks run the same calls on their
    slices with no collective; contiguous ranges of near-equal size, the first
    n_slices % world ranks one slice longer."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    base, extra = divmod(int(n_slices), world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def make_problem(B, heads, d, grid, tile, window, scale=None, dtype=DSA_BF16) -> Problem:
    p = Problem()
    p.B, p.heads, p.d = int(B), int(heads), int(d)
    p.T, p.H, p.W = (int(x) for x in grid)
    for a in range(3):
        p.tile[a] = int(tile[a])
        p.window[a] = int(window[a])
    p.scale = float(1.0 / math.sqrt(d)) if scale is None else float(scale)
    p.dtype = int(dtype)
    return p


def _problem_of(q: torch.Tensor, tile, window, scale) -> Problem:
    if q.dim() != 6:
        raise ValueError("q must be [B, heads, T, H, W, d]")
    if q.dtype == torch.bfloat16:
        dt = DSA_BF16
    elif q.dtype == torch.float32:
        dt = DSA_F32
    else:
        raise ValueError(f"unsupported dtype {q.dtype}")
    B, heads, T, H, W, d = q.shape
    return make_problem(B, heads, d, (T, H, W), tile, window, scale, dt)


def _check(st: int, what: str):
    if st != 0:
        raise DsaError(st, what)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, like: torch.Tensor, dtype=None):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if t.device != like.device:
        raise ValueError(f"{name} is on {t.device}, q on {like.device}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def plan_shape(problem: Problem):
    lib = load_library()
    n, wt = ctypes.c_int32(), ctypes.c_int32()
    _check(lib.dsa_plan_shape(ctypes.byref(problem), ctypes.byref(n), ctypes.byref(wt)), "dsa_plan_shape")
    return n.value, wt.value


def workspace_size(problem: Problem, backward: bool = False) -> int:
    return int(load_library().dsa_workspace_size(ctypes.byref(problem), DSA_WS_BWD if backward else DSA_WS_FWD))


def workspace(problem: Problem, device, backward: bool = False) -> torch.Tensor:
    """A device workspace of the right size (torch's caching allocator returns 512-byte
    aligned blocks)."""
    return torch.empty(max(workspace_size(problem, backward), 256), dtype=torch.uint8, device=device)


def plan(problem: Problem, offsets: torch.Tensor, inverse: bool = True, stream=None):
    """Run the window planner.  Returns (starts, kv_tiles[, row_ptr, q_tiles]) on the device."""
    lib = load_library()
    n, wt = plan_shape(problem)
    dev = offsets.device
    if not offsets.is_cuda or offsets.dtype != torch.int32 or not offsets.is_contiguous() or offsets.numel() != 3 * n:
        raise ValueError("offsets must be a contiguous int32 CUDA tensor [nTiles, 3]")
    starts = torch.empty((n, 3), dtype=torch.int32, device=dev)
    kv = torch.empty((n, wt), dtype=torch.int32, device=dev)
    row_ptr = torch.empty(n + 1, dtype=torch.int32, device=dev) if inverse else None
    q_tiles = torch.empty(n * wt, dtype=torch.int32, device=dev) if inverse else None
    _check(lib.dsa_plan(ctypes.byref(problem), _ptr(offsets), _ptr(starts), _ptr(kv), _ptr(row_ptr), _ptr(q_tiles),
                        ctypes.c_void_p(_stream(stream))), "dsa_plan")
    return (starts, kv, row_ptr, q_tiles) if inverse else (starts, kv)


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, offsets: torch.Tensor, tile: Sequence[int],
            window: Sequence[int], scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
            lse: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """3D-DSA forward.  Returns (out, lse)."""
    lib = load_library()
    p = _problem_of(q, tile, window, scale)
    for t, name in ((k, "k"), (v, "v")):
        _need(t, name, q, q.dtype)
        if t.shape != q.shape:
            raise ValueError(f"{name} shape {tuple(t.shape)} != q shape {tuple(q.shape)}")
    _need(q, "q", q)
    _need(offsets, "offsets", q, torch.int32)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:5], dtype=torch.float32, device=q.device)
    _need(out, "out", q, q.dtype)
    _need(lse, "lse", q, torch.float32)
    if ws is None:
        ws = workspace(p, q.device)
    _check(lib.dsa_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(offsets), _ptr(out), _ptr(lse), _ptr(ws),
                       ws.numel(), ctypes.c_void_p(_stream(stream))), "dsa_fwd")
    return out, lse


def prefix_workspace_size(problem: Problem, L_text: int) -> int:
    return int(load_library().dsa_prefix_workspace_size(ctypes.byref(problem), int(L_text)))


def forward_prefix(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, offsets: torch.Tensor, q_text: torch.Tensor,
                   k_text: torch.Tensor, v_text: torch.Tensor, tile: Sequence[int], window: Sequence[int],
                   scale: Optional[float] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """3D-DSA with a text prefix: video queries over their windows and every text key, text
    queries over every key.  q, k, v: [B, heads, T, H, W, 128]; q_text, k_text, v_text:
    [B, heads, L_text, 128].  Returns (out, lse, out_text, lse_text)."""
    lib = load_library()
    p = _problem_of(q, tile, window, scale)
    for t, name in ((k, "k"), (v, "v")):
        _need(t, name, q, q.dtype)
        if t.shape != q.shape:
            raise ValueError(f"{name} shape {tuple(t.shape)} != q shape {tuple(q.shape)}")
    _need(q, "q", q)
    _need(offsets, "offsets", q, torch.int32)
    if q_text.dim() != 4 or tuple(q_text.shape[:2]) != tuple(q.shape[:2]) or q_text.shape[3] != q.shape[5]:
        raise ValueError(f"q_text shape {tuple(q_text.shape)} does not match q {tuple(q.shape)}")
    for t, name in ((q_text, "q_text"), (k_text, "k_text"), (v_text, "v_text")):
        _need(t, name, q, q.dtype)
        if t.shape != q_text.shape:
            raise ValueError(f"{name} shape {tuple(t.shape)} != q_text shape {tuple(q_text.shape)}")
    L_text = int(q_text.shape[2])
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:5], dtype=torch.float32, device=q.device)
    out_text = torch.empty_like(q_text)
    lse_text = torch.empty(q_text.shape[:3], dtype=torch.float32, device=q.device)
    if ws is None:
        ws = torch.empty(max(prefix_workspace_size(p, L_text), 256), dtype=torch.uint8, device=q.device)
    _check(lib.dsa_fwd_prefix(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(offsets), L_text, _ptr(q_text),
                              _ptr(k_text), _ptr(v_text), _ptr(out), _ptr(lse), _ptr(out_text), _ptr(lse_text),
                              _ptr(ws), ws.numel(), ctypes.c_void_p(_stream(stream))), "dsa_fwd_prefix")
    return out, lse, out_text, lse_text


def selftest_wait(stream=None):
    """Enqueue the failure-path self-test (a bounded wait that runs out after 2 s and records
    DSA_ERR_TIMEOUT at site 99); read the result with device_status()."""
    _check(load_library().dsa_selftest_wait(ctypes.c_void_p(_stream(stream))), "dsa_selftest_wait")


def prefix_bwd_workspace_size(problem: Problem, L_text: int) -> int:
    return int(load_library().dsa_bwd_prefix_workspace_size(ctypes.byref(problem), int(L_text)))


def backward_prefix(q, k, v, out, lse, dout, offsets, q_text, k_text, v_text, out_text, lse_text, dout_text,
                    tile: Sequence[int], window: Sequence[int], scale: Optional[float] = None,
                    ws: Optional[torch.Tensor] = None, stream=None):
    """Backward of forward_prefix (gradients of sum(out * dout) + sum(out_text * dout_text)).
    Returns (dq, dk, dv, dq_text, dk_text, dv_text)."""
    lib = load_library()
    p = _problem_of(q, tile, window, scale)
    for t, name in ((k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t, name, q, q.dtype)
        if t.shape != q.shape:
            raise ValueError(f"{name} shape {tuple(t.shape)} != q shape {tuple(q.shape)}")
    _need(q, "q", q)
    _need(lse, "lse", q, torch.float32)
    _need(offsets, "offsets", q, torch.int32)
    if q_text.dim() != 4 or tuple(q_text.shape[:2]) != tuple(q.shape[:2]) or q_text.shape[3] != q.shape[5]:
        raise ValueError(f"q_text shape {tuple(q_text.shape)} does not match q {tuple(q.shape)}")
    for t, name in ((q_text, "q_text"), (k_text, "k_text"), (v_text, "v_text"), (out_text, "out_text"),
                    (dout_text, "dout_text")):
        _need(t, name, q, q.dtype)
        if t.shape != q_text.shape:
            raise ValueError(f"{name} shape {tuple(t.shape)} != q_text shape {tuple(q_text.shape)}")
    _need(lse_text, "lse_text", q, torch.float32)
    L_text = int(q_text.shape[2])
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    dqt, dkt, dvt = torch.empty_like(q_text), torch.empty_like(q_text), torch.empty_like(q_text)
    if ws is None:
        ws = torch.empty(max(prefix_bwd_workspace_size(p, L_text), 256), dtype=torch.uint8, device=q.device)
    _check(lib.dsa_bwd_prefix(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout),
                              _ptr(offsets), L_text, _ptr(q_text), _ptr(k_text), _ptr(v_text), _ptr(out_text),
                              _ptr(lse_text), _ptr(dout_text), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dqt), _ptr(dkt),
                              _ptr(dvt), _ptr(ws), ws.numel(), ctypes.c_void_p(_stream(stream))), "dsa_bwd_prefix")
    return dq, dk, dv, dqt, dkt, dvt


def forward_host_bytes(problem: Problem) -> int:
    return int(load_library().dsa_fwd_host_bytes(ctypes.byref(problem)))


def forward_host(problem: Problem, q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor,
                 offsets_host: torch.Tensor, out_host: torch.Tensor, lse_host: torch.Tensor, dev: torch.Tensor,
                 stream=None):
    """3D-DSA forward from pinned host tensors through the caller's device buffer ``dev``
    (uint8, at least forward_host_bytes(problem) bytes); asynchronous on ``stream``."""
    lib = load_library()
    for t in (q_host, k_host, v_host, offsets_host, out_host, lse_host):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host tensors must be contiguous CPU tensors")
    _check(lib.dsa_fwd_host(ctypes.byref(problem), _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(offsets_host),
                            _ptr(out_host), _ptr(lse_host), _ptr(dev), dev.numel(), ctypes.c_void_p(_stream(stream))),
           "dsa_fwd_host")


def backward(q, k, v, out, lse, dout, offsets, tile, window, scale=None, dq=None, dk=None, dv=None, ws=None,
             stream=None):
    """3D-DSA backward of sum(out * dout).  Returns (dq, dk, dv)."""
    lib = load_library()
    p = _problem_of(q, tile, window, scale)
    for t, name in ((k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t, name, q, q.dtype)
        if t.shape != q.shape:
            raise ValueError(f"{name} shape {tuple(t.shape)} != q shape {tuple(q.shape)}")
    _need(q, "q", q)
    _need(lse, "lse", q, torch.float32)
    _need(offsets, "offsets", q, torch.int32)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for t, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, name, q, q.dtype)
    if ws is None:
        ws = workspace(p, q.device, backward=True)
    _check(lib.dsa_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(offsets),
                       _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(), ctypes.c_void_p(_stream(stream))),
           "dsa_bwd")
    return dq, dk, dv


def _list_args(q: torch.Tensor, row_ptr: torch.Tensor, kv_list: torch.Tensor, n_tiles: int):
    """-> (list pointer, nnz, per_head): row_ptr [nTiles + 1] is one list for every head,
    [B * heads, nTiles + 1] one list per (batch, head)."""
    _need(row_ptr, "row_ptr", q, torch.int32)
    BH = q.shape[0] * q.shape[1]
    if row_ptr.numel() == n_tiles + 1 and row_ptr.dim() == 1:
        per_head = 0
    elif tuple(row_ptr.shape) == (BH, n_tiles + 1):
        per_head = 1
    else:
        raise ValueError(f"row_ptr must be [nTiles + 1] or [B * heads, nTiles + 1], got {tuple(row_ptr.shape)}")
    if kv_list is not None and kv_list.numel() > 0:
        _need(kv_list, "kv_list", q, torch.int32)
        return _ptr(kv_list), int(kv_list.numel()), per_head
    return None, 0, per_head


def forward_list(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, row_ptr: torch.Tensor, kv_list: torch.Tensor,
                 tile: Sequence[int], scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, stream=None):
    """Block-sparse forward over key-tile lists: query tile i attends to the key tiles
    kv_list[row_ptr[i]:row_ptr[i+1]] (int32 CUDA tensors; tiles in raster order of the tile
    grid); row_ptr [nTiles + 1] is one list for every head, [B * heads, nTiles + 1] one per
    (batch, head) with absolute positions in kv_list.  Returns (out, lse); an empty row
    gives out = 0 and lse = -inf."""
    lib = load_library()
    p = _problem_of(q, tile, (1, 1, 1), scale)
    for t, name in ((k, "k"), (v, "v")):
        _need(t, name, q, q.dtype)
        if t.shape != q.shape:
            raise ValueError(f"{name} shape {tuple(t.shape)} != q shape {tuple(q.shape)}")
    _need(q, "q", q)
    n_tiles, _ = plan_shape(p)
    lst, nnz, per_head = _list_args(q, row_ptr, kv_list, n_tiles)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:5], dtype=torch.float32, device=q.device)
    _need(out, "out", q, q.dtype)
    _need(lse, "lse", q, torch.float32)
    _check(lib.dsa_fwd_list(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr), lst, nnz, per_head, _ptr(out),
                            _ptr(lse), ctypes.c_void_p(_stream(stream))), "dsa_fwd_list")
    return out, lse


def backward_list(q, k, v, out, lse, dout, row_ptr, kv_list, tile, scale=None, dq=None, dk=None, dv=None, ws=None,
                  stream=None):
    """Backward of sum(out * dout) for forward_list.  Returns (dq, dk, dv)."""
    lib = load_library()
    p = _problem_of(q, tile, (1, 1, 1), scale)
    for t, name in ((k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t, name, q, q.dtype)
        if t.shape != q.shape:
            raise ValueError(f"{name} shape {tuple(t.shape)} != q shape {tuple(q.shape)}")
    _need(q, "q", q)
    _need(lse, "lse", q, torch.float32)
    n_tiles, _ = plan_shape(p)
    lst, nnz, per_head = _list_args(q, row_ptr, kv_list, n_tiles)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for t, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, name, q, q.dtype)
    if ws is None:
        size = int(lib.dsa_list_workspace_size(ctypes.byref(p), nnz, per_head, DSA_WS_BWD))
        ws = torch.empty(max(size, 256), dtype=torch.uint8, device=q.device)
    _check(lib.dsa_bwd_list(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout),
                            _ptr(row_ptr), lst, nnz, per_head, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                            ctypes.c_void_p(_stream(stream))), "dsa_bwd_list")
    return dq, dk, dv


def block_map(q: torch.Tensor, k: torch.Tensor, lse: torch.Tensor, row_ptr: torch.Tensor, kv_list: torch.Tensor,
              tile: Sequence[int], scale: Optional[float] = None, out: Optional[torch.Tensor] = None, stream=None):
    """Block attention mass [B * heads, nTiles, nTiles] (fp32): mean attention probability
    of each query tile's tokens on each key tile, against the LSE forward_list wrote for
    the same lists."""
    lib = load_library()
    p = _problem_of(q, tile, (1, 1, 1), scale)
    _need(q, "q", q)
    _need(k, "k", q, q.dtype)
    _need(lse, "lse", q, torch.float32)
    n_tiles, _ = plan_shape(p)
    lst, nnz, per_head = _list_args(q, row_ptr, kv_list, n_tiles)
    BH = q.shape[0] * q.shape[1]
    if out is None:
        out = torch.empty((BH, n_tiles, n_tiles), dtype=torch.float32, device=q.device)
    _need(out, "out", q, torch.float32)
    _check(lib.dsa_block_map(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(lse), _ptr(row_ptr), lst, nnz, per_head,
                             _ptr(out), ctypes.c_void_p(_stream(stream))), "dsa_block_map")
    return out


def lstsq_factor(M: torch.Tensor, lam: float, stream=None) -> torch.Tensor:
    """Cholesky factor (fp64 [p, p], lower) of M^T M + lam I for a design matrix M (fp32
    CUDA [m, p], p <= 32), to be reused by lstsq_solve across heads and steps."""
    lib = load_library()
    if not M.is_cuda or M.dtype != torch.float32 or not M.is_contiguous() or M.dim() != 2:
        raise ValueError("M must be a contiguous fp32 CUDA tensor [m, p]")
    m, p = M.shape
    L = torch.empty((p, p), dtype=torch.float64, device=M.device)
    _check(lib.dsa_lstsq_factor(m, p, _ptr(M), float(lam), _ptr(L), ctypes.c_void_p(_stream(stream))),
           "dsa_lstsq_factor")
    return L


def lstsq_solve(M: torch.Tensor, L: torch.Tensor, S: torch.Tensor, X: Optional[torch.Tensor] = None, ws=None,
                stream=None) -> torch.Tensor:
    """X [batch, p] (fp32) with (M^T M + lam I) x_b = M^T s_b for every row s_b of S
    [batch, m] (fp32 CUDA), L from lstsq_factor."""
    lib = load_library()
    m, p = M.shape
    if not S.is_cuda or S.dtype != torch.float32 or not S.is_contiguous() or S.dim() != 2 or S.shape[1] != m:
        raise ValueError("S must be a contiguous fp32 CUDA tensor [batch, m]")
    batch = S.shape[0]
    if X is None:
        X = torch.empty((batch, p), dtype=torch.float32, device=S.device)
    n_ws = int(lib.dsa_lstsq_workspace_size(m, p, batch))
    if ws is None and n_ws > 0:
        ws = torch.empty(n_ws, dtype=torch.uint8, device=S.device)
    _check(lib.dsa_lstsq_solve(m, p, batch, _ptr(M), _ptr(L), _ptr(S), _ptr(X), _ptr(ws),
                               0 if ws is None else ws.numel(), ctypes.c_void_p(_stream(stream))), "dsa_lstsq_solve")
    return X


def plan_heads(problem: Problem, offsets: torch.Tensor, stream=None):
    """Per-(batch, head) window offsets [B * heads, nTiles, 3] (int32 CUDA) as per-head
    key-tile lists: returns (row_ptr [B * heads, nTiles + 1], kv_list) for forward_list /
    backward_list."""
    lib = load_library()
    n, wt = plan_shape(problem)
    BH = problem.B * problem.heads
    if not offsets.is_cuda or offsets.dtype != torch.int32 or not offsets.is_contiguous() or \
            offsets.numel() != BH * n * 3:
        raise ValueError("offsets must be a contiguous int32 CUDA tensor [B * heads, nTiles, 3]")
    row_ptr = torch.empty((BH, n + 1), dtype=torch.int32, device=offsets.device)
    kv_list = torch.empty(BH * n * wt, dtype=torch.int32, device=offsets.device)
    _check(lib.dsa_plan_heads(ctypes.byref(problem), _ptr(offsets), _ptr(row_ptr), _ptr(kv_list),
                              ctypes.c_void_p(_stream(stream))), "dsa_plan_heads")
    return row_ptr, kv_list


def device_status(stream=None):
    """Synchronise ``stream`` and read/clear the device status word: (status, site, block)."""
    lib = load_library()
    site, block = ctypes.c_int32(), ctypes.c_int32()
    st = lib.dsa_device_status(ctypes.c_void_p(_stream(stream)), ctypes.byref(site), ctypes.byref(block))
    return st, site.value, block.value
