// bf16 forward of 3D Deformable Slide Attention on the 5th-generation tensor cores.
//
// Operator: for every query token n of query tile i, O_n = softmax(scale * q_n K(i)^T) V(i)
// over exactly the keys of the window planned for tile i, and LSE_n = ln sum exp(...)
// ("MegaSlide-DiT: Memory-Centric Adaptation and Deformable Local Attention for Efficient
// Video Diffusion", abstract, 3D-DSA; tile-granular window form from "Fast Video
// Generation with Sliding Tile Attention", abstract).
//
// One CTA per 128-row query sub-tile (a box of tw x th x 128/(tw*th) tokens of one query
// tile), 128 threads, thread r owning query row r (TMEM lane r).  For every 128-token
// chunk of every key tile in the window:
//   TMA: K and V chunk boxes -> shared memory (128-byte swizzle, two 64-column halves)
//   tcgen05.mma: S = Q K^T into TMEM (fp32), 8 k-steps of 16
//   softmax: each thread reads its S row from TMEM, updates its running max / sum
//            (base-2 domain), writes P = exp2(S * scale * log2 e - m) as bf16 into shared
//            memory in the operand layout of the next MMA
//   tcgen05.mma: O_chunk = P V into TMEM; each thread folds it into its register
//            accumulator with the running rescale factor.
// The epilogue writes O / l as bf16 and LSE = (m + log2 l) * ln 2.
#pragma once

#include <stdint.h>

#include "sm100.cuh"

namespace dsa {

struct FwdBf16Params {
  const int32_t* kv_tiles;  // [n_tiles, Wt]
  __nv_bfloat16* out;       // [B*heads, N, 128]
  float* lse;               // [B*heads, N]
  int n_tiles, Wt;
  int S;                    // 128-row chunks per tile
  int G1, G2;               // Gh, Gw
  int tt, th, tw, tcs;      // tile shape; t-extent of one 128-token chunk
  int T, H, W, N;
  float scale_log2;         // scale * log2(e)
};

namespace fwd1 {
constexpr int kThreads = 128;
constexpr uint32_t kTileBytes = 128 * 128 * 2;  // one 128 x 128 bf16 operand
constexpr uint32_t kHalfBytes = kTileBytes / 2;  // one 128 x 64 swizzled half
constexpr uint32_t kOffQ = 0, kOffK = kTileBytes, kOffV = 2 * kTileBytes, kOffP = 3 * kTileBytes;
constexpr uint32_t kOffBar = 4 * kTileBytes;
constexpr uint32_t kSmemBytes = kOffBar + 64 + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 256;                    // S: [0,128), O: [128,256)
constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t kIdescO = idesc_bf16_f32(128, 128, 0, 1);
}  // namespace fwd1

__global__ void __launch_bounds__(fwd1::kThreads, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, FwdBf16Params p) {
  using namespace fwd1;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  uint64_t* load_bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* mma_bar = load_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(load_bar + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(load_bar + 3);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int u = blockIdx.x;
  const int sub = u % p.S;
  const int tile = (u / p.S) % p.n_tiles;
  const int bh = u / (p.S * p.n_tiles);
  const int qt = tile / (p.G1 * p.G2), qh = (tile / p.G2) % p.G1, qw = tile % p.G2;
  const int q_t0 = qt * p.tt + sub * p.tcs, q_h0 = qh * p.th, q_w0 = qw * p.tw;

  if (tid == 0) {
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    mbar_init(load_bar, 1);
    mbar_init(mma_bar, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;

  float acc[128];
#pragma unroll
  for (int c = 0; c < 128; ++c) acc[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  uint32_t load_phase = 0, mma_phase = 0;
  bool ok = true;

  const int n_chunks = p.Wt * p.S;
  for (int c = 0; c < n_chunks && ok; ++c) {
    if (tid == 0) {
      const int kt = p.kv_tiles[static_cast<int64_t>(tile) * p.Wt + c / p.S];
      const int ks = c % p.S;
      const int kt_t = kt / (p.G1 * p.G2), kt_h = (kt / p.G2) % p.G1, kt_w = kt % p.G2;
      const int t0 = kt_t * p.tt + ks * p.tcs, h0 = kt_h * p.th, w0 = kt_w * p.tw;
      mbar_arrive_expect_tx(load_bar, (c == 0 ? 3u : 2u) * kTileBytes);
      if (c == 0) {
        tma_load_5d(smem + kOffQ, &tmQ, load_bar, 0, q_w0, q_h0, q_t0, bh);
        tma_load_5d(smem + kOffQ + kHalfBytes, &tmQ, load_bar, 64, q_w0, q_h0, q_t0, bh);
      }
      tma_load_5d(smem + kOffK, &tmK, load_bar, 0, w0, h0, t0, bh);
      tma_load_5d(smem + kOffK + kHalfBytes, &tmK, load_bar, 64, w0, h0, t0, bh);
      tma_load_5d(smem + kOffV, &tmV, load_bar, 0, w0, h0, t0, bh);
      tma_load_5d(smem + kOffV + kHalfBytes, &tmV, load_bar, 64, w0, h0, t0, bh);
    }
    ok = mbar_wait(load_bar, load_phase, abort, 1);
    load_phase ^= 1;
    if (!__syncthreads_and(ok)) break;

    // S = Q K^T
    tc_fence_after();
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t koff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
        mma_ss(tS, smem_desc_sw128(sbase + kOffQ + koff, 16, 1024), smem_desc_sw128(sbase + kOffK + koff, 16, 1024),
               kIdescS, kk > 0);
      }
      mma_commit(mma_bar);
    }
    ok = mbar_wait(mma_bar, mma_phase, abort, 2);
    mma_phase ^= 1;
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();

    // online softmax on this thread's row
    uint32_t r[32];
    float cmax = -INFINITY;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      tmem_ld32_wait(tS + lane_off + g * 32, r);
#pragma unroll
      for (int j = 0; j < 32; ++j) cmax = fmaxf(cmax, __uint_as_float(r[j]));
    }
    const float m_new = fmaxf(m, cmax * p.scale_log2);
    const float alpha = ex2_approx(m - m_new);
    m = m_new;
    float psum = 0.f;
    const int rr = tid & 7;
    const uint32_t prow = sbase + kOffP + (tid >> 3) * 1024 + rr * 128;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      tmem_ld32_wait(tS + lane_off + g * 32, r);
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(r[2 * j]), p.scale_log2, -m_new));
        const float p1 = ex2_approx(fmaf(__uint_as_float(r[2 * j + 1]), p.scale_log2, -m_new));
        psum += p0 + p1;
        pk[j] = pack_bf16x2(p0, p1);
      }
      // keys 32g .. 32g+31 live in half g/2, 16-byte chunks (g%2)*4 .. +3 of the row
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int chunk = (g & 1) * 4 + q4;
        st_shared_v4(prow + (g >> 1) * kHalfBytes + ((chunk ^ rr) << 4), pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2],
                     pk[4 * q4 + 3]);
      }
    }
    l = l * alpha + psum;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // O_chunk = P V
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t poff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
        mma_ss(tO, smem_desc_sw128(sbase + kOffP + poff, 16, 1024),
               smem_desc_sw128(sbase + kOffV + kk * 2048, kHalfBytes, 1024), kIdescO, kk > 0);
      }
      mma_commit(mma_bar);
    }
    ok = mbar_wait(mma_bar, mma_phase, abort, 3);
    mma_phase ^= 1;
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      tmem_ld32_wait(tO + lane_off + g * 32, r);
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[g * 32 + j] = fmaf(acc[g * 32 + j], alpha, __uint_as_float(r[j]));
    }
    tc_fence_before();
    __syncthreads();
  }

  if (ok) {
    const int lw = tid % p.tw, lh = (tid / p.tw) % p.th, lt = tid / (p.tw * p.th);
    const int64_t tok = (static_cast<int64_t>(q_t0 + lt) * p.H + (q_h0 + lh)) * p.W + (q_w0 + lw);
    const float inv = 1.f / l;
    uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(bh) * p.N + tok) * 128);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      uint4 v;
      v.x = pack_bf16x2(acc[8 * c + 0] * inv, acc[8 * c + 1] * inv);
      v.y = pack_bf16x2(acc[8 * c + 2] * inv, acc[8 * c + 3] * inv);
      v.z = pack_bf16x2(acc[8 * c + 4] * inv, acc[8 * c + 5] * inv);
      v.w = pack_bf16x2(acc[8 * c + 6] * inv, acc[8 * c + 7] * inv);
      dst[c] = v;
    }
    p.lse[static_cast<int64_t>(bh) * p.N + tok] = (m + __log2f(l)) * 0.69314718055994531f;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace dsa
