// fp32 forward of 3D Deformable Slide Attention on the CUDA cores (exact fp32 FMA).
//
// This path serves fp32 problems, whose tolerance (1e-5 against the fp64 definition)
// rules out the tensor cores' tf32 inputs.  It computes, for every query token n of query
// tile i, softmax(scale * q_n K(i)^T) V(i) over exactly the keys of the planned window
// (window rule: "MegaSlide-DiT ...", abstract; tile form: "Fast Video Generation with
// Sliding Tile Attention", abstract), with a streaming (online) softmax.
//
// Grid: (n_tiles, B * heads, row groups); block: kF32Threads threads covering
// kF32Threads / (D / 64) query rows of the tile.  A query row is owned by D / 64 adjacent threads, each holding a 64-wide slice of q and of the output
// accumulator; partial dot products are combined with one shuffle.  Keys stream through
// shared memory in chunks of kChunk tokens.
#pragma once

#include <math.h>
#include <stdint.h>

#include "dsa_device_status.cuh"

namespace dsa {

struct FwdF32Params {
  const float* q;
  const float* k;
  const float* v;
  const int32_t* kv_tiles;  // [n_tiles, Wt]
  float* out;
  float* lse;
  int T, H, W, N;
  int tt, th, tw, tile_tokens;
  int G1, G2;  // Gh, Gw
  int Wt;
  float scale;
};

__device__ __forceinline__ int64_t tile_token_index(int tile, int r, int G1, int G2, int tt, int th, int tw, int H,
                                                    int W) {
  const int ct = tile / (G1 * G2), ch = (tile / G2) % G1, cw = tile % G2;
  const int lw = r % tw, lh = (r / tw) % th, lt = r / (tw * th);
  const int64_t t = static_cast<int64_t>(ct) * tt + lt, h = static_cast<int64_t>(ch) * th + lh,
                w = static_cast<int64_t>(cw) * tw + lw;
  return (t * H + h) * W + w;
}

constexpr int kF32Threads = 256;

template <int D>
__global__ void __launch_bounds__(kF32Threads) fwd_f32_kernel(FwdF32Params p) {
  constexpr int TPR = D / 64;  // threads per query row
  constexpr int kChunk = 32;
  __shared__ float sK[kChunk][D];
  __shared__ float sV[kChunk][D];

  const int tile = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int row = blockIdx.z * (kF32Threads / TPR) + threadIdx.x / TPR;
  const int part = threadIdx.x % TPR;
  const bool active = row < p.tile_tokens;
  const int64_t base = bh * static_cast<int64_t>(p.N) * D;

  float qv[64], acc[64];
  const int64_t qtok = active ? tile_token_index(tile, row, p.G1, p.G2, p.tt, p.th, p.tw, p.H, p.W) : 0;
#pragma unroll
  for (int c = 0; c < 64; ++c) {
    qv[c] = active ? p.q[base + qtok * D + part * 64 + c] : 0.f;
    acc[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  for (int wi = 0; wi < p.Wt; ++wi) {
    const int kt = p.kv_tiles[static_cast<int64_t>(tile) * p.Wt + wi];
    for (int k0 = 0; k0 < p.tile_tokens; k0 += kChunk) {
      const int nk = min(kChunk, p.tile_tokens - k0);
      __syncthreads();
      for (int e = threadIdx.x; e < nk * D; e += blockDim.x) {
        const int kr = e / D, c = e % D;
        const int64_t tok = tile_token_index(kt, k0 + kr, p.G1, p.G2, p.tt, p.th, p.tw, p.H, p.W);
        sK[kr][c] = p.k[base + tok * D + c];
        sV[kr][c] = p.v[base + tok * D + c];
      }
      __syncthreads();
      float s[kChunk];
      float cmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        float d = 0.f;
        if (j < nk) {
#pragma unroll
          for (int c = 0; c < 64; ++c) d = fmaf(qv[c], sK[j][part * 64 + c], d);
        }
        if (TPR == 2) d += __shfl_xor_sync(0xffffffffu, d, 1);
        s[j] = j < nk ? d * p.scale : -INFINITY;
        cmax = fmaxf(cmax, s[j]);
      }
      const float m_new = fmaxf(m, cmax);
      const float alpha = expf(m - m_new);
      l *= alpha;
#pragma unroll
      for (int c = 0; c < 64; ++c) acc[c] *= alpha;
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        if (j < nk) {
          const float pj = expf(s[j] - m_new);
          l += pj;
#pragma unroll
          for (int c = 0; c < 64; ++c) acc[c] = fmaf(pj, sV[j][part * 64 + c], acc[c]);
        }
      }
      m = m_new;
    }
  }
  if (!active) return;
  const float inv = 1.f / l;
#pragma unroll
  for (int c = 0; c < 64; ++c) p.out[base + qtok * D + part * 64 + c] = acc[c] * inv;
  if (part == 0) p.lse[bh * p.N + qtok] = m + logf(l);
}

}  // namespace dsa
