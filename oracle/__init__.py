"""fp64 CPU oracle for 3D Deformable Slide Attention (3D-DSA).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this package; the product path never does.  It shares no
code with the CUDA library.  The arithmetic lives in ``dsa_oracle.c`` (plain C, double
precision, OpenMP over independent rows); this module compiles it with gcc, marshals
arguments with ctypes, and scatters the per-tile results back into full tensors.

Definition followed (the pages give the operator only in outline): "MegaSlide-DiT:
Memory-Centric Adaptation and Deformable Local Attention for Efficient Video Diffusion",
abstract (3D-DSA, a motion-adaptive local attention whose cost is linear in the sequence
length) and "Fast Video Generation with Sliding Tile Attention", abstract (attention over
a local spatial-temporal window, tile-granular).  The concrete window rule, softmax and
gradients are written out in the header of ``dsa_oracle.c``.

The key-tile-list functions (``forward_list``, ``backward_list``) take a CSR of key tiles
per query tile instead of window offsets: the block-sparse generalisation of the window
(the MOD-DiT page, Method section, Stage 2 "Online Block Masking", attends over selected
blocks of keys).  The block attention mass (``block_map_list``), the text prefix
(``forward_prefix*``, ``backward_prefix*``: the MOD-DiT page, "Token-Type-Aware Masking") and
the regularised least squares (``lstsq``: the MOD-DiT page, Method, Stage 1) follow their
definitions in the same plain way.

Every function here is pinned by the CPU tests in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libdsa_oracle.so")
_lib = None


class _Problem(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "heads", "d", "T", "H", "W", "tt", "th", "tw", "wt", "wh", "ww")] + [
        ("scale", ctypes.c_double)
    ]


def build(force: bool = False) -> str:
    """Compile the oracle into a shared library with gcc (no -ffast-math: IEEE double)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        i32p = ctypes.POINTER(ctypes.c_int32)
        fp = ctypes.POINTER(ctypes.c_double)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_plan.argtypes = [ctypes.c_int32] * 6 + [i32p] * 5
        lib.oracle_fwd.argtypes = [ctypes.POINTER(_Problem), fp, fp, fp, i32p, ctypes.c_int32, i32p, i32p, dp, dp]
        lib.oracle_bwd_dq.argtypes = [ctypes.POINTER(_Problem), fp, fp, fp, fp, i32p, ctypes.c_int32, i32p, i32p, dp]
        lib.oracle_bwd_dkdv.argtypes = [ctypes.POINTER(_Problem), fp, fp, fp, fp, i32p, ctypes.c_int32, i32p, i32p,
                                        dp, dp]
        lib.oracle_fwd_list.argtypes = [ctypes.POINTER(_Problem), fp, fp, fp, i32p, i32p, ctypes.c_int32, i32p, i32p,
                                        dp, dp]
        lib.oracle_bwd_dq_list.argtypes = [ctypes.POINTER(_Problem), fp, fp, fp, fp, i32p, i32p, ctypes.c_int32, i32p,
                                           i32p, dp]
        lib.oracle_bwd_dkdv_list.argtypes = [ctypes.POINTER(_Problem), fp, fp, fp, fp, i32p, i32p, ctypes.c_int32,
                                             i32p, i32p, dp, dp]
        lib.oracle_block_map_list.argtypes = [ctypes.POINTER(_Problem), fp, fp, i32p, i32p, ctypes.c_int32, i32p,
                                              i32p, dp]
        lib.oracle_fwd_prefix.argtypes = [ctypes.POINTER(_Problem), fp, fp, fp, i32p, ctypes.c_int32, fp, fp,
                                          ctypes.c_int32, i32p, i32p, dp, dp]
        for f in (lib.oracle_plan, lib.oracle_fwd, lib.oracle_bwd_dq, lib.oracle_bwd_dkdv, lib.oracle_fwd_list,
                  lib.oracle_bwd_dq_list, lib.oracle_bwd_dkdv_list, lib.oracle_block_map_list,
                  lib.oracle_fwd_prefix):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _f64(t) -> np.ndarray:
    """Widen a tensor (bf16, fp32 or fp64) to a contiguous float64 numpy array, exactly."""
    if isinstance(t, torch.Tensor):
        t = t.detach().to("cpu")
        if t.dtype != torch.float64:
            t = t.to(torch.float64)
        return np.ascontiguousarray(t.numpy())
    return np.ascontiguousarray(np.asarray(t, dtype=np.float64))


def _i32(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        t = t.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(t, dtype=np.int32))


class Geometry:
    """Shapes of one problem: token grid, tiles, window (all from the caller)."""

    def __init__(self, B, heads, d, grid, tile, window, scale=None):
        self.B, self.heads, self.d = int(B), int(heads), int(d)
        self.grid = tuple(int(x) for x in grid)
        self.tile = tuple(int(x) for x in tile)
        self.window = tuple(int(x) for x in window)
        self.scale = float(1.0 / np.sqrt(d)) if scale is None else float(scale)
        for g, t in zip(self.grid, self.tile):
            if t <= 0 or g % t:
                raise ValueError(f"grid {self.grid} is not divisible by tile {self.tile}")
        self.G = tuple(g // t for g, t in zip(self.grid, self.tile))
        self.weff = tuple(min(w, g) for w, g in zip(self.window, self.G))
        self.n_tiles = self.G[0] * self.G[1] * self.G[2]
        self.n_window_tiles = self.weff[0] * self.weff[1] * self.weff[2]
        self.tile_tokens = self.tile[0] * self.tile[1] * self.tile[2]
        self.n_tokens = self.grid[0] * self.grid[1] * self.grid[2]

    @classmethod
    def of(cls, w):
        """Geometry of a ``dsa_inputs.Workload``."""
        return cls(w.B, w.heads, w.d, w.grid, w.tile, w.window, w.scale)

    def c_problem(self) -> _Problem:
        T, H, W = self.grid
        tt, th, tw = self.tile
        wt, wh, ww = self.window
        return _Problem(self.B, self.heads, self.d, T, H, W, tt, th, tw, wt, wh, ww, self.scale)

    def tile_token_index(self) -> np.ndarray:
        """[nTiles, tile_tokens] token index of each tile's tokens in raster order."""
        T, H, W = self.grid
        tt, th, tw = self.tile
        idx = np.arange(self.n_tokens).reshape(T, H, W)
        idx = idx.reshape(self.G[0], tt, self.G[1], th, self.G[2], tw).transpose(0, 2, 4, 1, 3, 5)
        return np.ascontiguousarray(idx.reshape(self.n_tiles, self.tile_tokens))


def plan(G, window, offsets):
    """Window plan of the oracle: (starts[nTiles,3], kv_tiles[nTiles,Wt], row_ptr[nTiles+1], q_tiles[nnz])."""
    lib = _load()
    G = [int(x) for x in G]
    window = [int(x) for x in window]
    n = G[0] * G[1] * G[2]
    wt = 1
    for w, g in zip(window, G):
        wt *= min(w, g)
    off = _i32(offsets).reshape(n, 3)
    starts = np.zeros((n, 3), np.int32)
    kv = np.zeros((n, wt), np.int32)
    row_ptr = np.zeros(n + 1, np.int32)
    q_tiles = np.zeros(n * wt, np.int32)
    rc = lib.oracle_plan(*G, *window, _ptr(off, ctypes.c_int32), _ptr(starts, ctypes.c_int32),
                         _ptr(kv, ctypes.c_int32), _ptr(row_ptr, ctypes.c_int32), _ptr(q_tiles, ctypes.c_int32))
    if rc:
        raise ValueError(f"oracle_plan rejected G={G} window={window}")
    return starts, kv, row_ptr, q_tiles[: row_ptr[-1]]


def _selection(geo: Geometry, sel):
    if sel is None:
        bh = np.repeat(np.arange(geo.B * geo.heads, dtype=np.int32), geo.n_tiles)
        tiles = np.tile(np.arange(geo.n_tiles, dtype=np.int32), geo.B * geo.heads)
    else:
        bh = _i32(sel[0]).reshape(-1)
        tiles = _i32(sel[1]).reshape(-1)
    return bh, tiles


def _head_slice(t, geo: Geometry, bh: int) -> np.ndarray:
    """float64 copy of one (b, head) slice [N, d] of a [B, heads, T, H, W, d] tensor."""
    if isinstance(t, torch.Tensor):
        return _f64(t.reshape(geo.B * geo.heads, geo.n_tokens, geo.d)[bh])
    return _f64(np.asarray(t).reshape(geo.B * geo.heads, geo.n_tokens, geo.d)[bh])


def _run_by_head(geo: Geometry, tensors, offsets, sel, n_out, call, extra=None):
    """Run ``call`` once per (b, head) present in the selection, on that head's slice
    (heads are independent problems), so host memory holds one head in float64 at a time.
    ``extra(h)``, if given, returns more per-head arrays appended to the slices."""
    bh, tiles = _selection(geo, sel)
    off = _i32(offsets).reshape(geo.n_tiles, 3)
    outs = [np.zeros((len(bh), geo.tile_tokens, geo.d), np.float64) for _ in range(n_out)]
    lse = np.zeros((len(bh), geo.tile_tokens), np.float64)
    one = Geometry(1, 1, geo.d, geo.grid, geo.tile, geo.window, geo.scale)
    p = one.c_problem()
    for h in np.unique(bh):
        rows = np.nonzero(bh == h)[0]
        sl = [_head_slice(t, geo, int(h)) for t in tensors]
        if extra is not None:
            sl += list(extra(int(h)))
        sel_t = np.ascontiguousarray(tiles[rows])
        sel_b = np.zeros(len(rows), np.int32)
        part = [np.zeros((len(rows), geo.tile_tokens, geo.d), np.float64) for _ in range(n_out)]
        part_lse = np.zeros((len(rows), geo.tile_tokens), np.float64)
        rc = call(p, sl, off, len(rows), sel_b, sel_t, part, part_lse)
        if rc:
            raise RuntimeError(f"oracle call failed ({rc})")
        for o, pt in zip(outs, part):
            o[rows] = pt
        lse[rows] = part_lse
    return outs, lse


def forward_tiles(geo: Geometry, q, k, v, offsets, sel=None):
    """Forward on (bh, query tile) pairs.  Returns out[n_sel, tile_tokens, d] and
    lse[n_sel, tile_tokens] (float64), rows in each tile's raster order."""
    lib = _load()
    D = ctypes.c_double

    def call(p, sl, off, n, sb, st, part, part_lse):
        return lib.oracle_fwd(ctypes.byref(p), _ptr(sl[0], D), _ptr(sl[1], D), _ptr(sl[2], D),
                              _ptr(off, ctypes.c_int32), n, _ptr(sb, ctypes.c_int32), _ptr(st, ctypes.c_int32),
                              _ptr(part[0], D), _ptr(part_lse, D))

    (out,), lse = _run_by_head(geo, (q, k, v), offsets, sel, 1, call)
    return out, lse


def forward(geo: Geometry, q, k, v, offsets):
    """Full forward: out[B, heads, T, H, W, d] and lse[B, heads, T, H, W] in float64."""
    out_t, lse_t = forward_tiles(geo, q, k, v, offsets)
    return _scatter_forward(geo, out_t, lse_t)


def _scatter_forward(geo: Geometry, out_t, lse_t):
    """Per-tile rows ([BH * nTiles, tile_tokens, ...]) -> full tensors in token order."""
    tok = geo.tile_token_index()
    BH = geo.B * geo.heads
    out = np.zeros((BH, geo.n_tokens, geo.d), np.float64)
    lse = np.zeros((BH, geo.n_tokens), np.float64)
    out_t = out_t.reshape(BH, geo.n_tiles, geo.tile_tokens, geo.d)
    lse_t = lse_t.reshape(BH, geo.n_tiles, geo.tile_tokens)
    out[:, tok.reshape(-1)] = out_t.reshape(BH, -1, geo.d)
    lse[:, tok.reshape(-1)] = lse_t.reshape(BH, -1)
    return (out.reshape((geo.B, geo.heads) + geo.grid + (geo.d,)),
            lse.reshape((geo.B, geo.heads) + geo.grid))


def _text_slice(t, geo: Geometry, bh: int) -> np.ndarray:
    """float64 copy of one (b, head) slice [L_text, d] of a [B, heads, L_text, d] tensor."""
    a = t if isinstance(t, torch.Tensor) else torch.from_numpy(np.asarray(t))
    return _f64(a.reshape(geo.B * geo.heads, -1, geo.d)[bh])


def forward_prefix_tiles(geo: Geometry, q, k, v, offsets, k_text, v_text, sel=None):
    """Text-prefix forward of video query tokens on (bh, query tile) pairs: each attends to
    its window and to every text token (one softmax over the union).  Returns
    out[n_sel, tile_tokens, d] and lse[n_sel, tile_tokens] (float64)."""
    lib = _load()
    D = ctypes.c_double
    L_text = int(k_text.shape[2])

    def call(p, sl, off, n, sb, st, part, part_lse):
        return lib.oracle_fwd_prefix(ctypes.byref(p), _ptr(sl[0], D), _ptr(sl[1], D), _ptr(sl[2], D),
                                     _ptr(off, ctypes.c_int32), L_text, _ptr(sl[3], D), _ptr(sl[4], D), n,
                                     _ptr(sb, ctypes.c_int32), _ptr(st, ctypes.c_int32), _ptr(part[0], D),
                                     _ptr(part_lse, D))

    def text_of(h):
        return _text_slice(k_text, geo, h), _text_slice(v_text, geo, h)

    (out,), lse = _run_by_head(geo, (q, k, v), offsets, sel, 1, call, extra=text_of)
    return out, lse


def forward_prefix_text(geo: Geometry, q_text, k_text, v_text, k, v, rows=None):
    """Text-prefix forward of text query tokens: each attends to every text token and every
    video token (plain dense softmax attention over the concatenated key set, per (b, head)).
    rows: optional text token indices to compute.  Returns out[B, heads, n_rows, d] and
    lse[B, heads, n_rows] (float64)."""
    BH = geo.B * geo.heads
    L_text = int(q_text.shape[2])
    idx = np.arange(L_text) if rows is None else np.asarray(rows)
    out = np.zeros((BH, len(idx), geo.d), np.float64)
    lse = np.zeros((BH, len(idx)), np.float64)
    for h in range(BH):
        qh = _text_slice(q_text, geo, h)[idx]
        keys = np.concatenate([_text_slice(k_text, geo, h), _head_slice(k, geo, h)], axis=0)
        vals = np.concatenate([_text_slice(v_text, geo, h), _head_slice(v, geo, h)], axis=0)
        s = geo.scale * (qh @ keys.T)
        mx = s.max(axis=1, keepdims=True)
        l = mx[:, 0] + np.log(np.exp(s - mx).sum(axis=1))
        out[h] = np.exp(s - l[:, None]) @ vals
        lse[h] = l
    return (out.reshape(geo.B, geo.heads, len(idx), geo.d), lse.reshape(geo.B, geo.heads, len(idx)))


def forward_prefix(geo: Geometry, q, k, v, offsets, q_text, k_text, v_text):
    """Full text-prefix forward: (out, lse) of the video tokens as in ``forward`` and
    (out_text, lse_text) of the text tokens, float64."""
    out_t, lse_t = forward_prefix_tiles(geo, q, k, v, offsets, k_text, v_text)
    out, lse = _scatter_forward(geo, out_t, lse_t)
    out_x, lse_x = forward_prefix_text(geo, q_text, k_text, v_text, k, v)
    return out, lse, out_x, lse_x


def _prefix_key_mask(geo: Geometry, offsets, L_text: int, rows) -> np.ndarray:
    """Boolean [len(rows), N + L_text]: which keys of the unified [video; text] sequence
    query row r (r < N: video token r, else text token r - N) attends to: a video token its
    window's key tiles (the oracle's plan) and every text token; a text token everything."""
    N = geo.n_tokens
    _, kv, _, _ = plan(geo.G, geo.window, offsets)
    tile_of = np.zeros(N, np.int64)
    tile_of[geo.tile_token_index().reshape(-1)] = np.repeat(np.arange(geo.n_tiles), geo.tile_tokens)
    allowed = np.zeros((geo.n_tiles, geo.n_tiles), bool)
    allowed[np.repeat(np.arange(geo.n_tiles), kv.shape[1]), kv.reshape(-1)] = True
    rows = np.asarray(rows)
    mask = np.ones((len(rows), N + L_text), bool)
    vid = rows < N
    mask[np.nonzero(vid)[0], :N] = allowed[tile_of[rows[vid]]][:, tile_of]
    return mask


def backward_prefix(geo: Geometry, q, k, v, dout, offsets, q_text, k_text, v_text, dout_text, block: int = 512):
    """Text-prefix backward of L = sum(O * dO) over the unified sequence: the plain softmax
    attention gradients (P = exp(s - lse), D = rowsum(dO * O), dS = P (dP - D),
    dq = scale dS K, dk = scale dS^T Q, dv = P^T dO), each query row over its key set (video:
    window and every text token; text: everything), in float64, query rows in blocks of
    `block` with library matmuls.  Returns (dq, dk, dv) as [B, heads, T, H, W, d] and
    (dq_text, dk_text, dv_text) as [B, heads, L_text, d]."""
    BH, N, d = geo.B * geo.heads, geo.n_tokens, geo.d
    L = int(q_text.shape[2])
    outs = [np.zeros((BH, N + L, d), np.float64) for _ in range(3)]
    for h in range(BH):
        def cat(a, b):
            return np.concatenate([_head_slice(a, geo, h), _text_slice(b, geo, h)], axis=0)

        Q, K, V, dO = cat(q, q_text), cat(k, k_text), cat(v, v_text), cat(dout, dout_text)
        dq, dk, dv = (o[h] for o in outs)
        for r0 in range(0, N + L, block):
            rows = np.arange(r0, min(r0 + block, N + L))
            m = _prefix_key_mask(geo, offsets, L, rows)
            s = np.where(m, geo.scale * (Q[rows] @ K.T), -np.inf)
            mx = s.max(axis=1, keepdims=True)
            lse = mx + np.log(np.exp(s - mx).sum(axis=1, keepdims=True))
            P = np.exp(s - lse)
            O = P @ V
            dP = dO[rows] @ V.T
            D = (dO[rows] * O).sum(axis=1, keepdims=True)
            dS = P * (dP - D)
            dq[rows] = geo.scale * (dS @ K)
            dk += geo.scale * (dS.T @ Q[rows])
            dv += P.T @ dO[rows]
    shape_v = (geo.B, geo.heads) + geo.grid + (d,)
    shape_t = (geo.B, geo.heads, L, d)
    return (tuple(o[:, :N].reshape(shape_v) for o in outs), tuple(o[:, N:].reshape(shape_t) for o in outs))


def backward_prefix_sampled(geo: Geometry, q, k, v, dout, offsets, q_text, k_text, v_text, dout_text, h: int,
                            q_rows, qt_rows, k_rows, kt_rows):
    """Text-prefix backward of (b, head) h on selected rows only, from the definition: the
    forward of every query row of the head (video rows through the C oracle over their window
    and the text keys, text rows over every key) gives lse and O, D = rowsum(dO * O); then
    dq of the selected video query rows q_rows and text query rows qt_rows over their key sets,
    and dk, dv of the selected video key rows k_rows (over the video queries whose window
    holds the key's tile, and every text query) and text key rows kt_rows (over every query).
    Returns (dq[len(q_rows)], dq_text[len(qt_rows)], dk, dv [len(k_rows)], dk_text, dv_text
    [len(kt_rows)]), each row [d], float64."""
    N, d, sc = geo.n_tokens, geo.d, geo.scale
    one = Geometry(1, 1, d, geo.grid, geo.tile, geo.window, geo.scale)
    Q, K, V, dO = (_head_slice(t, geo, h) for t in (q, k, v, dout))
    Qt, Kt, Vt, dOt = (_text_slice(t, geo, h) for t in (q_text, k_text, v_text, dout_text))
    Lt = Qt.shape[0]
    # forward of every video row of the head (window + text keys), in token order
    sel = (np.zeros(geo.n_tiles, np.int32), np.arange(geo.n_tiles, dtype=np.int32))
    as_head = [torch.from_numpy(a).reshape((1, 1) + geo.grid + (d,)) for a in (Q, K, V)]
    out_t, lse_t = forward_prefix_tiles(one, *as_head, offsets, torch.from_numpy(Kt).reshape(1, 1, Lt, d),
                                        torch.from_numpy(Vt).reshape(1, 1, Lt, d), sel)
    tok = geo.tile_token_index().reshape(-1)
    O = np.zeros((N, d))
    lse = np.zeros(N)
    O[tok] = out_t.reshape(-1, d)
    lse[tok] = lse_t.reshape(-1)
    D = (dO * O).sum(axis=1)
    # text rows over every key (text first, then video)
    keys, vals = np.concatenate([Kt, K]), np.concatenate([Vt, V])
    st = sc * (Qt @ keys.T)
    mx = st.max(axis=1, keepdims=True)
    lse_x = mx[:, 0] + np.log(np.exp(st - mx).sum(axis=1))
    Ot = np.exp(st - lse_x[:, None]) @ vals
    Dt = (dOt * Ot).sum(axis=1)
    # key sets of the video query tiles (the oracle's plan)
    _, kv, _, _ = plan(geo.G, geo.window, offsets)
    tile_of = np.zeros(N, np.int64)
    tile_of[tok] = np.repeat(np.arange(geo.n_tiles), geo.tile_tokens)
    tiles_tok = geo.tile_token_index()

    def grad_rows(qv, dov, lsev, Dv, kk, vv):
        """dq of query rows (one row per call) over keys kk, vv: P, dS and sum dS k."""
        s = sc * (kk @ qv)
        P = np.exp(s - lsev)
        dS = P * (vv @ dov - Dv)
        return sc * (dS @ kk)

    dq = np.array([grad_rows(Q[n], dO[n], lse[n], D[n],
                             np.concatenate([K[tiles_tok[kv[tile_of[n]]].reshape(-1)], Kt]),
                             np.concatenate([V[tiles_tok[kv[tile_of[n]]].reshape(-1)], Vt])) for n in q_rows])
    dq_t = np.array([grad_rows(Qt[j], dOt[j], lse_x[j], Dt[j], keys, vals) for j in qt_rows])

    def key_grads(km, vm, qs, dos, lses, Ds):
        """dk, dv of one key over the query rows qs (with their dO, lse, D)."""
        s = sc * (qs @ km)
        P = np.exp(s - lses)
        dS = P * (dos @ vm - Ds)
        return sc * (dS @ qs), P @ dos

    dk, dv = [], []
    for m in k_rows:
        holders = np.nonzero((kv == tile_of[m]).any(axis=1))[0]  # query tiles whose window holds m
        rows = tiles_tok[holders].reshape(-1)
        qs = np.concatenate([Q[rows], Qt])
        g = key_grads(K[m], V[m], qs, np.concatenate([dO[rows], dOt]), np.concatenate([lse[rows], lse_x]),
                      np.concatenate([D[rows], Dt]))
        dk.append(g[0])
        dv.append(g[1])
    dkt, dvt = [], []
    Qall, dOall = np.concatenate([Q, Qt]), np.concatenate([dO, dOt])
    lall, Dall = np.concatenate([lse, lse_x]), np.concatenate([D, Dt])
    for j in kt_rows:
        g = key_grads(Kt[j], Vt[j], Qall, dOall, lall, Dall)
        dkt.append(g[0])
        dvt.append(g[1])
    return dq, dq_t, np.array(dk), np.array(dv), np.array(dkt), np.array(dvt)


def backward_dq_tiles(geo: Geometry, q, k, v, dout, offsets, sel=None):
    """dq on (bh, query tile) pairs: [n_sel, tile_tokens, d] float64."""
    lib = _load()
    D = ctypes.c_double

    def call(p, sl, off, n, sb, st, part, part_lse):
        return lib.oracle_bwd_dq(ctypes.byref(p), _ptr(sl[0], D), _ptr(sl[1], D), _ptr(sl[2], D), _ptr(sl[3], D),
                                 _ptr(off, ctypes.c_int32), n, _ptr(sb, ctypes.c_int32), _ptr(st, ctypes.c_int32),
                                 _ptr(part[0], D))

    (dq,), _ = _run_by_head(geo, (q, k, v, dout), offsets, sel, 1, call)
    return dq


def backward_dkdv_tiles(geo: Geometry, q, k, v, dout, offsets, sel=None):
    """dk, dv on (bh, key tile) pairs: each [n_sel, tile_tokens, d] float64, rows in the
    key tile's raster order."""
    lib = _load()
    D = ctypes.c_double

    def call(p, sl, off, n, sb, st, part, part_lse):
        return lib.oracle_bwd_dkdv(ctypes.byref(p), _ptr(sl[0], D), _ptr(sl[1], D), _ptr(sl[2], D), _ptr(sl[3], D),
                                   _ptr(off, ctypes.c_int32), n, _ptr(sb, ctypes.c_int32), _ptr(st, ctypes.c_int32),
                                   _ptr(part[0], D), _ptr(part[1], D))

    (dk, dv), _ = _run_by_head(geo, (q, k, v, dout), offsets, sel, 2, call)
    return dk, dv


def backward_head(geo: Geometry, q, k, v, dout, offsets, h: int):
    """Full backward of one (b, head) slice h: dq, dk, dv as [N, d] float64 (token order).

    The definition of the header of dsa_oracle.c, grouped by query tile: for each query tile
    i with key set K(i) (the oracle's plan), S = scale Q_i K^T, lse by max subtraction,
    P = exp(S - lse), dP = dO_i V^T, dS = P (dP - rowsum(P dP)); then dq_i = scale dS K,
    and every key row m of K(i) gains scale dS^T Q_i (dk) and P^T dO_i (dv), so dk_m and
    dv_m sum over every query token whose key set holds m.  numpy fp64 matrix products
    serve as the sums; one head is a few seconds (the C functions recompute each query
    row's softmax per key tile, which is far slower for whole heads)."""
    N, d, sc = geo.n_tokens, geo.d, geo.scale
    Q, K, V, dO = (_head_slice(t, geo, h) for t in (q, k, v, dout))
    _, kv, _, _ = plan(geo.G, geo.window, offsets)
    tiles_tok = geo.tile_token_index()
    dq, dk, dv = np.zeros((N, d)), np.zeros((N, d)), np.zeros((N, d))
    for i in range(geo.n_tiles):
        rows = tiles_tok[i]
        keys = tiles_tok[kv[i]].reshape(-1)
        s = sc * (Q[rows] @ K[keys].T)
        mx = s.max(axis=1, keepdims=True)
        lse = mx + np.log(np.exp(s - mx).sum(axis=1, keepdims=True))
        P = np.exp(s - lse)
        dP = dO[rows] @ V[keys].T
        dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
        dq[rows] = sc * (dS @ K[keys])
        # a window lists each of its tiles once, so `keys` has no repeated row
        dk[keys] += sc * (dS.T @ Q[rows])
        dv[keys] += P.T @ dO[rows]
    return dq, dk, dv


def backward(geo: Geometry, q, k, v, dout, offsets):
    """Full backward: dq, dk, dv as [B, heads, T, H, W, d] float64."""
    dq_t = backward_dq_tiles(geo, q, k, v, dout, offsets)
    dk_t, dv_t = backward_dkdv_tiles(geo, q, k, v, dout, offsets)
    tok = geo.tile_token_index().reshape(-1)
    BH = geo.B * geo.heads
    res = []
    for t in (dq_t, dk_t, dv_t):
        full = np.zeros((BH, geo.n_tokens, geo.d), np.float64)
        full[:, tok] = t.reshape(BH, -1, geo.d)
        res.append(full.reshape((geo.B, geo.heads) + geo.grid + (geo.d,)))
    return tuple(res)


# ------------------------------------------------------------------------------------------
# Key-tile lists (block-sparse form): query tile i attends to the key tiles
# kv_list[row_ptr[i]:row_ptr[i+1]] instead of its window box; see dsa_oracle.c.


def _head_lists(geo: Geometry, row_ptr, kv_list, h: int):
    """CSR of (b, head) h: row_ptr is [nTiles + 1] (one list for every head) or
    [B * heads, nTiles + 1] with absolute positions in kv_list (a list per head)."""
    rp = _i32(row_ptr)
    kl = _i32(kv_list).reshape(-1)
    if rp.ndim == 2:
        if rp.shape != (geo.B * geo.heads, geo.n_tiles + 1):
            raise ValueError("per-head row_ptr must be [B * heads, nTiles + 1]")
        rp = rp[h]
        lo, hi = int(rp[0]), int(rp[-1])
        if not 0 <= lo <= hi <= kl.shape[0]:
            raise RuntimeError("per-head row_ptr outside the list")
        rp, kl = rp - lo, kl[lo:hi]
    rp = np.ascontiguousarray(rp.reshape(-1), dtype=np.int32)
    if rp.shape[0] != geo.n_tiles + 1:
        raise ValueError("row_ptr must have nTiles + 1 entries")
    kl = np.ascontiguousarray(kl, dtype=np.int32)
    if kl.shape[0] == 0:
        kl = np.zeros(1, np.int32)  # a valid pointer for an all-empty list
    return rp, kl


def _run_by_head_lists(geo: Geometry, tensors, row_ptr, kv_list, sel, n_out, call):
    """As _run_by_head, with key-tile lists (shared by every head, or one per head)
    instead of window offsets."""
    bh, tiles = _selection(geo, sel)
    outs = [np.zeros((len(bh), geo.tile_tokens, geo.d), np.float64) for _ in range(n_out)]
    lse = np.zeros((len(bh), geo.tile_tokens), np.float64)
    one = Geometry(1, 1, geo.d, geo.grid, geo.tile, (1, 1, 1), geo.scale)
    p = one.c_problem()
    for h in np.unique(bh):
        rows = np.nonzero(bh == h)[0]
        rp, kl = _head_lists(geo, row_ptr, kv_list, int(h))
        sl = [_head_slice(t, geo, int(h)) for t in tensors]
        sel_t = np.ascontiguousarray(tiles[rows])
        sel_b = np.zeros(len(rows), np.int32)
        part = [np.zeros((len(rows), geo.tile_tokens, geo.d), np.float64) for _ in range(n_out)]
        part_lse = np.zeros((len(rows), geo.tile_tokens), np.float64)
        rc = call(p, sl, rp, kl, len(rows), sel_b, sel_t, part, part_lse)
        if rc:
            raise RuntimeError(f"oracle list call failed ({rc})")
        for o, pt in zip(outs, part):
            o[rows] = pt
        lse[rows] = part_lse
    return outs, lse


def _scatter(geo: Geometry, tiles_major):
    """[BH * nTiles, tile_tokens, ...] in (bh, tile) order -> [B, heads, T, H, W, ...]."""
    tok = geo.tile_token_index().reshape(-1)
    BH = geo.B * geo.heads
    rest = tiles_major.shape[2:]
    full = np.zeros((BH, geo.n_tokens) + rest, np.float64)
    full[:, tok] = tiles_major.reshape((BH, -1) + rest)
    return full.reshape((geo.B, geo.heads) + geo.grid + rest)


def forward_list(geo: Geometry, q, k, v, row_ptr, kv_list, sel=None):
    """Forward over key-tile lists (row_ptr [nTiles + 1] for every head, or
    [B * heads, nTiles + 1] per head).  With sel=None: out[B, heads, T, H, W, d] and
    lse[B, heads, T, H, W] (float64); with sel: per (bh, query tile) rows as forward_tiles."""
    lib = _load()
    D = ctypes.c_double
    I = ctypes.c_int32

    def call(p, sl, rp, kl, n, sb, st, part, part_lse):
        return lib.oracle_fwd_list(ctypes.byref(p), _ptr(sl[0], D), _ptr(sl[1], D), _ptr(sl[2], D), _ptr(rp, I),
                                   _ptr(kl, I), n, _ptr(sb, I), _ptr(st, I), _ptr(part[0], D), _ptr(part_lse, D))

    (out,), lse = _run_by_head_lists(geo, (q, k, v), row_ptr, kv_list, sel, 1, call)
    if sel is not None:
        return out, lse
    return _scatter(geo, out), _scatter(geo, lse)


def backward_list(geo: Geometry, q, k, v, dout, row_ptr, kv_list):
    """Backward over key-tile lists: dq, dk, dv as [B, heads, T, H, W, d] float64."""
    lib = _load()
    D = ctypes.c_double
    I = ctypes.c_int32

    def call_dq(p, sl, rp, kl, n, sb, st, part, part_lse):
        return lib.oracle_bwd_dq_list(ctypes.byref(p), _ptr(sl[0], D), _ptr(sl[1], D), _ptr(sl[2], D),
                                      _ptr(sl[3], D), _ptr(rp, I), _ptr(kl, I), n, _ptr(sb, I), _ptr(st, I),
                                      _ptr(part[0], D))

    def call_dkdv(p, sl, rp, kl, n, sb, st, part, part_lse):
        return lib.oracle_bwd_dkdv_list(ctypes.byref(p), _ptr(sl[0], D), _ptr(sl[1], D), _ptr(sl[2], D),
                                        _ptr(sl[3], D), _ptr(rp, I), _ptr(kl, I), n, _ptr(sb, I), _ptr(st, I),
                                        _ptr(part[0], D), _ptr(part[1], D))

    (dq,), _ = _run_by_head_lists(geo, (q, k, v, dout), row_ptr, kv_list, None, 1, call_dq)
    (dk, dv), _ = _run_by_head_lists(geo, (q, k, v, dout), row_ptr, kv_list, None, 2, call_dkdv)
    return _scatter(geo, dq), _scatter(geo, dk), _scatter(geo, dv)


def block_map_list(geo: Geometry, q, k, row_ptr, kv_list, sel=None):
    """Block attention mass over key-tile lists: map[bh, i, j] = mean over the query tokens
    of tile i of the attention probability on the tokens of key tile j (dsa_oracle.c).
    With sel=None: [B * heads, nTiles, nTiles]; with sel=(bh, tiles): [n_sel, nTiles]."""
    lib = _load()
    D = ctypes.c_double
    I = ctypes.c_int32
    bh, tiles = _selection(geo, sel)
    res = np.zeros((len(bh), geo.n_tiles), np.float64)
    one = Geometry(1, 1, geo.d, geo.grid, geo.tile, (1, 1, 1), geo.scale)
    p = one.c_problem()
    for h in np.unique(bh):
        rows = np.nonzero(bh == h)[0]
        rp, kl = _head_lists(geo, row_ptr, kv_list, int(h))
        sq, sk = _head_slice(q, geo, int(h)), _head_slice(k, geo, int(h))
        sel_t = np.ascontiguousarray(tiles[rows])
        sel_b = np.zeros(len(rows), np.int32)
        part = np.zeros((len(rows), geo.n_tiles), np.float64)
        rc = lib.oracle_block_map_list(ctypes.byref(p), _ptr(sq, D), _ptr(sk, D), _ptr(rp, I), _ptr(kl, I),
                                       len(rows), _ptr(sel_b, I), _ptr(sel_t, I), _ptr(part, D))
        if rc:
            raise RuntimeError(f"oracle block map failed ({rc})")
        res[rows] = part
    if sel is not None:
        return res
    return res.reshape(geo.B * geo.heads, geo.n_tiles, geo.n_tiles)


# ------------------------------------------------------------------------------------------
# Regularised least squares of the structural decomposition (the MOD-DiT page, Method
# section, Stage 1 "Sparsity Map Reconstruction"): X with (M^T M + lam I) X = M^T S_t.


def lstsq(M, lam: float, S) -> np.ndarray:
    """X [batch, p] for every row s_b of S [batch, m]: the normal equations of the page,
    solved in float64 (a library solve as the only step)."""
    M = _f64(M)
    S = _f64(S)
    G = M.T @ M + float(lam) * np.eye(M.shape[1])
    return np.linalg.solve(G, M.T @ S.T).T
