// Window planner of 3D Deformable Slide Attention ("MegaSlide-DiT: Memory-Centric
// Adaptation and Deformable Local Attention for Efficient Video Diffusion", abstract: a
// motion-adaptive local attention) in the tile-granular form of "Fast Video Generation
// with Sliding Tile Attention" (abstract).
//
// For query tile i and axis a, with w'_a = min(w_a, G_a):
//   start_a = clamp(i_a + offset_a - floor(w'_a / 2), 0, G_a - w'_a)
// The key tiles of the window are listed in ascending linear index (t outer, w inner).
// Optionally the inverse map is built as CSR: row j lists, ascending, the query tiles whose
// window holds key tile j (the backward pass walks it key-tile-major).
//
// The forward plan is one CTA of 1024 threads (a thread per query tile, Wt entries each);
// the inverse map spreads its containment tests over the whole grid.
#pragma once

#include <stdint.h>

namespace dsa {

struct PlanGeom {
  int G[3];   // tile grid (Gt, Gh, Gw)
  int w[3];   // effective window per axis, min(window, G)
  int n_tiles;
  int n_window_tiles;
};

__device__ __forceinline__ int plan_axis_start(int i, int off, int w, int G) {
  int s = i + off - w / 2;
  s = s < 0 ? 0 : s;
  s = s > G - w ? G - w : s;
  return s;
}

__device__ __forceinline__ bool plan_holds(const PlanGeom& g, const int32_t* starts, int i, int j) {
  const int jt = j / (g.G[1] * g.G[2]), jh = (j / g.G[2]) % g.G[1], jw = j % g.G[2];
  const int st = starts[3 * i], sh = starts[3 * i + 1], sw = starts[3 * i + 2];
  return jt >= st && jt < st + g.w[0] && jh >= sh && jh < sh + g.w[1] && jw >= sw && jw < sw + g.w[2];
}

__global__ void __launch_bounds__(1024) plan_kernel(PlanGeom g, const int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ starts, int32_t* __restrict__ kv_tiles) {
  const int n = g.n_tiles;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int it = i / (g.G[1] * g.G[2]), ih = (i / g.G[2]) % g.G[1], iw = i % g.G[2];
    const int st = plan_axis_start(it, offsets[3 * i + 0], g.w[0], g.G[0]);
    const int sh = plan_axis_start(ih, offsets[3 * i + 1], g.w[1], g.G[1]);
    const int sw = plan_axis_start(iw, offsets[3 * i + 2], g.w[2], g.G[2]);
    starts[3 * i + 0] = st;
    starts[3 * i + 1] = sh;
    starts[3 * i + 2] = sw;
    int32_t* dst = kv_tiles + static_cast<int64_t>(i) * g.n_window_tiles;
    int e = 0;
    for (int a = st; a < st + g.w[0]; ++a)
      for (int b = sh; b < sh + g.w[1]; ++b)
        for (int c = sw; c < sw + g.w[2]; ++c) dst[e++] = (a * g.G[1] + b) * g.G[2] + c;
  }
}

// The inverse map, in three launches after plan_kernel: for every key tile j the query
// tiles whose window holds j, ascending.  One warp per key tile (grid-stride over the
// warps of the whole grid) tests the query tiles 32 at a time and takes the hits from a
// ballot, so each row comes out in ascending order without a sort and the work
// (nTiles^2 / 32 warp steps) is spread over every SM.
//   kFill = false: the count of row j goes to row_ptr[j + 1];
//   kFill = true : row j is written from row_ptr[j] (after plan_scan_kernel).
template <bool kFill>
__global__ void __launch_bounds__(256) plan_inverse_kernel(PlanGeom g, const int32_t* __restrict__ starts,
                                                           int32_t* __restrict__ row_ptr,
                                                           int32_t* __restrict__ q_tiles) {
  const int n = g.n_tiles, lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t j = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; j < n; j += nwarps) {
    int pos = kFill ? row_ptr[j] : 0;
    for (int base = 0; base < n; base += 32) {
      const int i = base + lane;
      const bool hit = i < n && plan_holds(g, starts, i, static_cast<int>(j));
      const unsigned m = __ballot_sync(0xffffffffu, hit);
      if (kFill && hit) q_tiles[pos + __popc(m & ((1u << lane) - 1u))] = i;
      pos += __popc(m);
    }
    if (!kFill && lane == 0) row_ptr[j + 1] = pos;
  }
}

// Exclusive scan of the counts row_ptr[1..n] in place (row_ptr[0] = 0), one CTA of 1024
// threads, 1024 entries at a time.
__global__ void __launch_bounds__(1024) plan_scan_kernel(int n, int32_t* __restrict__ row_ptr) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  if (threadIdx.x == 0) {
    carry = 0;
    row_ptr[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < n; base += blockDim.x) {
    const int j = base + threadIdx.x;
    int x = j < n ? row_ptr[j + 1] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int t = lane < nwarps ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      if (lane < nwarps) warp_tot[lane] = t;
    }
    __syncthreads();
    x += (warp > 0 ? warp_tot[warp - 1] : 0) + carry;
    __syncthreads();
    if (j < n) row_ptr[j + 1] = x;
    if (threadIdx.x == blockDim.x - 1) carry = x;
    __syncthreads();
  }
}

// Per-(batch, head) windows as key-tile lists: head h (blockIdx.x) plans its own offsets
// offsets[h][nTiles][3] into kv_list[h * nTiles * Wt ...] (ascending key tiles per window,
// as above) with CSR offsets row_ptr[h][i] = (h * nTiles + i) * Wt, so the heads' lists
// follow one another and the flattened row_ptr is non-decreasing.
__global__ void __launch_bounds__(256) plan_heads_kernel(PlanGeom g, const int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ row_ptr, int32_t* __restrict__ kv_list) {
  const int n = g.n_tiles, h = blockIdx.x;
  const int64_t base = static_cast<int64_t>(h) * n;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int32_t* off = offsets + (base + i) * 3;
    const int it = i / (g.G[1] * g.G[2]), ih = (i / g.G[2]) % g.G[1], iw = i % g.G[2];
    const int st = plan_axis_start(it, off[0], g.w[0], g.G[0]);
    const int sh = plan_axis_start(ih, off[1], g.w[1], g.G[1]);
    const int sw = plan_axis_start(iw, off[2], g.w[2], g.G[2]);
    const int64_t first = (base + i) * g.n_window_tiles;
    row_ptr[static_cast<int64_t>(h) * (n + 1) + i] = static_cast<int32_t>(first);
    int32_t* dst = kv_list + first;
    int e = 0;
    for (int a = st; a < st + g.w[0]; ++a)
      for (int b = sh; b < sh + g.w[1]; ++b)
        for (int c = sw; c < sw + g.w[2]; ++c) dst[e++] = (a * g.G[1] + b) * g.G[2] + c;
  }
  if (threadIdx.x == 0) row_ptr[static_cast<int64_t>(h) * (n + 1) + n] = static_cast<int32_t>((base + n) * g.n_window_tiles);
}

}  // namespace dsa
