"""Seeded synthetic inputs for 3D Deformable Slide Attention (3D-DSA).

This module is shared by the fp64 oracle's tests and by the CUDA path's tests and
benchmark.  It holds the workload shapes and the seeded random draws only; it holds
none of the method's arithmetic (no window planning, no attention).

Workloads (video-latent token grids, tile-granular windows):

* ``tiny_f32``      : B=1, heads=2,  d=64,  grid 4x8x8,    tile 1x4x4, window 3x3x3, offsets 0, fp32, seed 0
* ``bf16_16x32x32`` : B=1, heads=24, d=128, grid 16x32x32, tile 4x8x8, window 3x3x3, offsets U{-1..1}
* ``bf16_480p``     : B=1, heads=12, d=128, grid 20x32x56, tile 4x8x8, window 3x3x5, offsets U{-2..2}
* ``bf16_720p``     : B=1, heads=24, d=128, grid 30x48x80, tile 6x8x8, window 3x3x3, offsets U{-2..2}
* ``adapt_480p_b2`` : the 480p shapes with B=2, plus dO; forward and backward

The sliding-tile form (a local 3D window made of whole tiles) follows "Fast Video
Generation with Sliding Tile Attention", abstract; the per-tile motion-adaptive shift
follows "MegaSlide-DiT: Memory-Centric Adaptation and Deformable Local Attention for
Efficient Video Diffusion", abstract (3D Deformable Slide Attention).

Random stream: ``torch.Generator().manual_seed(seed)`` on the CPU; draws in the order
q, k, v, (dO), offsets.  Q/K/V/dO are N(0,1) fp32 draws, rounded to bf16 (round to
nearest even) for the bf16 workloads.  Offsets are ``randint(lo, hi+1, (nTiles, 3))``
in tile units, one triple per query tile, shared by every batch entry and head.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    d: int
    grid: tuple  # (T, H, W) in tokens
    tile: tuple  # (tt, th, tw) in tokens
    window: tuple  # (wt, wh, ww) in tiles
    offset_range: tuple  # (lo, hi) inclusive, tile units
    dtype: str  # "f32" or "bf16"
    seed: int
    backward: bool = False

    @property
    def tile_grid(self):
        return tuple(g // t for g, t in zip(self.grid, self.tile))

    @property
    def n_tiles(self):
        gt, gh, gw = self.tile_grid
        return gt * gh * gw

    @property
    def n_tokens(self):
        T, H, W = self.grid
        return T * H * W

    @property
    def tile_tokens(self):
        return self.tile[0] * self.tile[1] * self.tile[2]

    @property
    def window_tiles(self):
        """Tiles per window after limiting each axis to the tile grid."""
        n = 1
        for w, g in zip(self.window, self.tile_grid):
            n *= min(w, g)
        return n

    @property
    def keys_per_query(self):
        return self.window_tiles * self.tile_tokens

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.d)

    def fwd_flops(self):
        """Effective forward FLOP: 4 * B * heads * N * keys_per_query * d."""
        return 4.0 * self.B * self.heads * self.n_tokens * self.keys_per_query * self.d

    def bwd_flops(self):
        """Effective backward FLOP: 2.5x the forward count."""
        return 2.5 * self.fwd_flops()

    def replace(self, **kw):
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 2, 64, (4, 8, 8), (1, 4, 4), (3, 3, 3), (0, 0), "f32", 0),
    "bf16_16x32x32": Workload("bf16_16x32x32", 1, 24, 128, (16, 32, 32), (4, 8, 8), (3, 3, 3), (-1, 1), "bf16", 1),
    "bf16_480p": Workload("bf16_480p", 1, 12, 128, (20, 32, 56), (4, 8, 8), (3, 3, 5), (-2, 2), "bf16", 2),
    "bf16_720p": Workload("bf16_720p", 1, 24, 128, (30, 48, 80), (6, 8, 8), (3, 3, 3), (-2, 2), "bf16", 3),
    "adapt_480p_b2": Workload("adapt_480p_b2", 2, 12, 128, (20, 32, 56), (4, 8, 8), (3, 3, 5), (-2, 2), "bf16", 4,
                              backward=True),
}


@dataclasses.dataclass
class Inputs:
    q: torch.Tensor  # [B, heads, T, H, W, d], CPU, fp32 or bf16
    k: torch.Tensor
    v: torch.Tensor
    dout: Optional[torch.Tensor]
    offsets: torch.Tensor  # [nTiles, 3] int32, tile units


def make_inputs(w: Workload, with_dout: Optional[bool] = None, seed: Optional[int] = None) -> Inputs:
    """Draw the seeded inputs of one workload on the CPU."""
    if with_dout is None:
        with_dout = w.backward
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    shape = (w.B, w.heads) + tuple(w.grid) + (w.d,)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    dout = torch.randn(shape, generator=g, dtype=torch.float32) if with_dout else None
    lo, hi = w.offset_range
    offsets = torch.randint(lo, hi + 1, (w.n_tiles, 3), generator=g, dtype=torch.int64).to(torch.int32)
    if w.dtype == "bf16":
        q, k, v = q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
        if dout is not None:
            dout = dout.to(torch.bfloat16)
    return Inputs(q, k, v, dout, offsets)


@dataclasses.dataclass
class TextInputs:
    q: torch.Tensor  # [B, heads, L_text, d], CPU, same dtype as the video tokens
    k: torch.Tensor
    v: torch.Tensor


def text_length(w: Workload) -> int:
    """Text tokens beside a video grid: about 1% of the sequence (the MOD-DiT page,
    "Token-Type-Aware Masking", puts text at roughly 1% of a unified text + video sequence)."""
    return max(1, -(-w.n_tokens // 100))


def make_text_inputs(w: Workload, L_text: int, seed: int) -> TextInputs:
    """Seeded text-token q, k, v (N(0,1) fp32 draws in that order, rounded to bf16 for bf16
    workloads), from their own generator so the video draws are unchanged."""
    g = torch.Generator().manual_seed(seed)
    shape = (w.B, w.heads, L_text, w.d)
    q, k, v = (torch.randn(shape, generator=g, dtype=torch.float32) for _ in range(3))
    if w.dtype == "bf16":
        q, k, v = q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
    return TextInputs(q, k, v)
