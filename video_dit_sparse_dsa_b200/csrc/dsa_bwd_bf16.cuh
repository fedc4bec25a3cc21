// bf16 backward of 3D Deformable Slide Attention on the 5th-generation tensor cores, for
// full-parameter adaptation ("MegaSlide-DiT: Memory-Centric Adaptation and Deformable
// Local Attention for Efficient Video Diffusion", abstract).
//
// Gradients of L = sum(O * dO) for O = softmax(scale Q K^T) V restricted to each query
// tile's window.  With P = exp(scale s - LSE) and D_n = sum_c dO_nc O_nc:
//   dV_m = sum_n P_nm dO_n,   dS_nm = P_nm (dO_n . v_m - D_n),
//   dK_m = scale sum_n dS_nm q_n,   dQ_n = scale sum_m dS_nm k_m,
// where n runs over the query tokens whose window holds key m.
//
// Three kernels:
//   bwd_preprocess : D = rowsum(dO * O) (fp32) and zeroes the fp32 dQ accumulator;
//   bwd_bf16_kernel: key-major; one CTA per 128-key chunk of a key tile, walking the query
//                    tiles of the inverse plan (CSR row of the key tile).  Per 128-query
//                    chunk: S^T = K Q^T and dP^T = V dO^T on tcgen05 into TMEM; each thread
//                    (one key row) forms P^T and dS^T in registers and stores them as bf16
//                    operands; then dV += P^T dO and dK += dS^T Q accumulate in TMEM and
//                    dQ_chunk = dS K lands in TMEM, from where each thread (one query row)
//                    adds it to the fp32 accumulator in global memory;
//   bwd_dq_convert : dQ = scale * accumulator, as bf16.
#pragma once

#include <stdint.h>

#include "sm100.cuh"

namespace dsa {

struct BwdBf16Params {
  const int32_t* row_ptr;  // [n_tiles + 1] inverse plan
  const int32_t* q_tiles;  // [n_tiles * Wt]
  const float* lse;        // [BH, N]
  const float* delta;      // [BH, N]
  float* dq_acc;           // [BH, N, 128]
  __nv_bfloat16* dk;       // [BH, N, 128]
  __nv_bfloat16* dv;
  int n_tiles, S;
  int G1, G2;
  int tt, th, tw, tcs;
  int T, H, W, N;
  float scale, scale_log2;
};

namespace bwd1 {
constexpr int kThreads = 128;
constexpr uint32_t kTileBytes = 128 * 128 * 2;
constexpr uint32_t kHalfBytes = kTileBytes / 2;
constexpr uint32_t kOffK = 0, kOffV = kTileBytes, kOffQ = 2 * kTileBytes, kOffDO = 3 * kTileBytes;
constexpr uint32_t kOffP = 4 * kTileBytes, kOffDS = 5 * kTileBytes;
constexpr uint32_t kOffLse = 6 * kTileBytes;      // 128 floats (base-2 LSE)
constexpr uint32_t kOffD = kOffLse + 512;         // 128 floats
constexpr uint32_t kOffBar = kOffD + 512;
constexpr uint32_t kSmemBytes = kOffBar + 64 + 1024;
constexpr uint32_t kTmemCols = 512;  // S^T / dQ, dP^T, dV, dK
constexpr uint32_t kIdescKK = idesc_bf16_f32(128, 128, 0, 0);   // both operands K-major
constexpr uint32_t kIdescKM = idesc_bf16_f32(128, 128, 0, 1);   // B MN-major
constexpr uint32_t kIdescMM = idesc_bf16_f32(128, 128, 1, 1);   // A and B MN-major
}  // namespace bwd1

__device__ __forceinline__ int64_t chunk_row_token(int r, int t0, int h0, int w0, int th, int tw, int H, int W) {
  const int lw = r % tw, lh = (r / tw) % th, lt = r / (tw * th);
  return (static_cast<int64_t>(t0 + lt) * H + (h0 + lh)) * W + (w0 + lw);
}

__global__ void __launch_bounds__(256) bwd_preprocess(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      float* __restrict__ delta, float* __restrict__ dq_acc,
                                                      int64_t rows) {
  // 16 threads per 128-wide row, 8 elements (16 bytes) each
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 16;
  const int part = threadIdx.x % 16;
  float s = 0.f;
  if (row < rows) {
    const uint4 a = reinterpret_cast<const uint4*>(o + row * 128)[part];
    const uint4 b = reinterpret_cast<const uint4*>(dout + row * 128)[part];
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(pa[i]);
      const float2 y = __bfloat1622float2(pb[i]);
      s = fmaf(x.x, y.x, s);
      s = fmaf(x.y, y.y, s);
    }
    float4* z = reinterpret_cast<float4*>(dq_acc + row * 128) + part * 2;
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int o2 = 8; o2 > 0; o2 >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o2);
  if (row < rows && part == 0) delta[row] = s;
}

__global__ void __launch_bounds__(256) bwd_dq_convert(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq,
                                                      float scale, int64_t n8) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
  const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  uint4 v;
  v.x = pack_bf16x2(a.x * scale, a.y * scale);
  v.y = pack_bf16x2(a.z * scale, a.w * scale);
  v.z = pack_bf16x2(b.x * scale, b.y * scale);
  v.w = pack_bf16x2(b.z * scale, b.w * scale);
  reinterpret_cast<uint4*>(dq)[i] = v;
}

__global__ void __launch_bounds__(bwd1::kThreads, 1)
    bwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    BwdBf16Params p) {
  using namespace bwd1;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  float* s_lse = reinterpret_cast<float*>(smem + kOffLse);
  float* s_d = reinterpret_cast<float*>(smem + kOffD);
  uint64_t* load_bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* mma_bar = load_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(load_bar + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(load_bar + 3);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int u = blockIdx.x;
  const int ks = u % p.S;
  const int kt = (u / p.S) % p.n_tiles;
  const int bh = u / (p.S * p.n_tiles);
  const int k_t0 = (kt / (p.G1 * p.G2)) * p.tt + ks * p.tcs;
  const int k_h0 = ((kt / p.G2) % p.G1) * p.th;
  const int k_w0 = (kt % p.G2) * p.tw;
  const int row0 = p.row_ptr[kt], row1 = p.row_ptr[kt + 1];
  const int n_chunks = (row1 - row0) * p.S;

  if (tid == 0) {
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    tma_prefetch_map(&tmDO);
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
  const uint32_t tS = tmem, tDP = tmem + 128, tDV = tmem + 256, tDK = tmem + 384;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const int64_t slice = static_cast<int64_t>(bh) * p.N;

  uint32_t load_phase = 0, mma_phase = 0;
  bool ok = true;
  for (int c = 0; c < n_chunks && ok; ++c) {
    const int qi = p.q_tiles[row0 + c / p.S];
    const int qs = c % p.S;
    const int q_t0 = (qi / (p.G1 * p.G2)) * p.tt + qs * p.tcs;
    const int q_h0 = ((qi / p.G2) % p.G1) * p.th;
    const int q_w0 = (qi % p.G2) * p.tw;
    if (tid == 0) {
      mbar_arrive_expect_tx(load_bar, (c == 0 ? 4u : 2u) * kTileBytes);
      if (c == 0) {
        tma_load_5d(smem + kOffK, &tmK, load_bar, 0, k_w0, k_h0, k_t0, bh);
        tma_load_5d(smem + kOffK + kHalfBytes, &tmK, load_bar, 64, k_w0, k_h0, k_t0, bh);
        tma_load_5d(smem + kOffV, &tmV, load_bar, 0, k_w0, k_h0, k_t0, bh);
        tma_load_5d(smem + kOffV + kHalfBytes, &tmV, load_bar, 64, k_w0, k_h0, k_t0, bh);
      }
      tma_load_5d(smem + kOffQ, &tmQ, load_bar, 0, q_w0, q_h0, q_t0, bh);
      tma_load_5d(smem + kOffQ + kHalfBytes, &tmQ, load_bar, 64, q_w0, q_h0, q_t0, bh);
      tma_load_5d(smem + kOffDO, &tmDO, load_bar, 0, q_w0, q_h0, q_t0, bh);
      tma_load_5d(smem + kOffDO + kHalfBytes, &tmDO, load_bar, 64, q_w0, q_h0, q_t0, bh);
    }
    // per-query-row LSE (to base 2) and D of this chunk; thread r = query row r
    const int64_t qtok = chunk_row_token(tid, q_t0, q_h0, q_w0, p.th, p.tw, p.H, p.W);
    s_lse[tid] = p.lse[slice + qtok] * 1.4426950408889634f;
    s_d[tid] = p.delta[slice + qtok];
    ok = mbar_wait(load_bar, load_phase, abort, 11);
    load_phase ^= 1;
    if (!__syncthreads_and(ok)) break;

    // S^T = K Q^T, dP^T = V dO^T
    tc_fence_after();
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t koff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
        mma_ss(tS, smem_desc_sw128(sbase + kOffK + koff, 16, 1024), smem_desc_sw128(sbase + kOffQ + koff, 16, 1024),
               kIdescKK, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t koff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
        mma_ss(tDP, smem_desc_sw128(sbase + kOffV + koff, 16, 1024),
               smem_desc_sw128(sbase + kOffDO + koff, 16, 1024), kIdescKK, kk > 0);
      }
      mma_commit(mma_bar);
    }
    ok = mbar_wait(mma_bar, mma_phase, abort, 12);
    mma_phase ^= 1;
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();

    // thread = key row m: P^T and dS^T over the chunk's 128 query columns
    const int rr = tid & 7;
    const uint32_t prow = sbase + kOffP + (tid >> 3) * 1024 + rr * 128;
    const uint32_t dsrow = sbase + kOffDS + (tid >> 3) * 1024 + rr * 128;
#pragma unroll 1
    for (int g = 0; g < 4; ++g) {
      uint32_t sr[32], dr[32];
      tmem_ld32_wait(tS + lane_off + g * 32, sr);
      tmem_ld32_wait(tDP + lane_off + g * 32, dr);
      uint32_t pk[16], dk2[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int n0 = g * 32 + 2 * j;
        const float p0 = ex2_approx(fmaf(__uint_as_float(sr[2 * j]), p.scale_log2, -s_lse[n0]));
        const float p1 = ex2_approx(fmaf(__uint_as_float(sr[2 * j + 1]), p.scale_log2, -s_lse[n0 + 1]));
        const float d0 = p0 * (__uint_as_float(dr[2 * j]) - s_d[n0]);
        const float d1 = p1 * (__uint_as_float(dr[2 * j + 1]) - s_d[n0 + 1]);
        pk[j] = pack_bf16x2(p0, p1);
        dk2[j] = pack_bf16x2(d0, d1);
      }
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const uint32_t off = (g >> 1) * kHalfBytes + ((((g & 1) * 4 + q4) ^ rr) << 4);
        st_shared_v4(prow + off, pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        st_shared_v4(dsrow + off, dk2[4 * q4], dk2[4 * q4 + 1], dk2[4 * q4 + 2], dk2[4 * q4 + 3]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // dV += P^T dO, dK += dS^T Q, dQ_chunk = dS K
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t aoff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
        mma_ss(tDV, smem_desc_sw128(sbase + kOffP + aoff, 16, 1024),
               smem_desc_sw128(sbase + kOffDO + kk * 2048, kHalfBytes, 1024), kIdescKM, (c > 0) || (kk > 0));
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t aoff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
        mma_ss(tDK, smem_desc_sw128(sbase + kOffDS + aoff, 16, 1024),
               smem_desc_sw128(sbase + kOffQ + kk * 2048, kHalfBytes, 1024), kIdescKM, (c > 0) || (kk > 0));
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        mma_ss(tS, smem_desc_sw128(sbase + kOffDS + kk * 2048, kHalfBytes, 1024),
               smem_desc_sw128(sbase + kOffK + kk * 2048, kHalfBytes, 1024), kIdescMM, kk > 0);
      }
      mma_commit(mma_bar);
    }
    ok = mbar_wait(mma_bar, mma_phase, abort, 13);
    mma_phase ^= 1;
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();

    // thread = query row n: add its dQ row to the fp32 accumulator
    float4* dst = reinterpret_cast<float4*>(p.dq_acc + (slice + qtok) * 128);
#pragma unroll 1
    for (int g = 0; g < 4; ++g) {
      uint32_t r[32];
      tmem_ld32_wait(tS + lane_off + g * 32, r);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        atomicAdd(dst + g * 8 + j, make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                               __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
    }
    tc_fence_before();
    __syncthreads();
  }

  if (ok) {
    // thread = key row m: dV and scale * dK as bf16 (zeros for a key tile no window holds)
    const int64_t ktok = chunk_row_token(tid, k_t0, k_h0, k_w0, p.th, p.tw, p.H, p.W);
    uint4* dv_dst = reinterpret_cast<uint4*>(p.dv + (slice + ktok) * 128);
    uint4* dk_dst = reinterpret_cast<uint4*>(p.dk + (slice + ktok) * 128);
    tc_fence_after();
#pragma unroll 1
    for (int g = 0; g < 4; ++g) {
      uint32_t a[32], b[32];
      if (n_chunks > 0) {
        tmem_ld32_wait(tDV + lane_off + g * 32, a);
        tmem_ld32_wait(tDK + lane_off + g * 32, b);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) a[j] = b[j] = 0u;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 x, y;
        x.x = pack_bf16x2(__uint_as_float(a[8 * j + 0]), __uint_as_float(a[8 * j + 1]));
        x.y = pack_bf16x2(__uint_as_float(a[8 * j + 2]), __uint_as_float(a[8 * j + 3]));
        x.z = pack_bf16x2(__uint_as_float(a[8 * j + 4]), __uint_as_float(a[8 * j + 5]));
        x.w = pack_bf16x2(__uint_as_float(a[8 * j + 6]), __uint_as_float(a[8 * j + 7]));
        y.x = pack_bf16x2(__uint_as_float(b[8 * j + 0]) * p.scale, __uint_as_float(b[8 * j + 1]) * p.scale);
        y.y = pack_bf16x2(__uint_as_float(b[8 * j + 2]) * p.scale, __uint_as_float(b[8 * j + 3]) * p.scale);
        y.z = pack_bf16x2(__uint_as_float(b[8 * j + 4]) * p.scale, __uint_as_float(b[8 * j + 5]) * p.scale);
        y.w = pack_bf16x2(__uint_as_float(b[8 * j + 6]) * p.scale, __uint_as_float(b[8 * j + 7]) * p.scale);
        dv_dst[g * 4 + j] = x;
        dk_dst[g * 4 + j] = y;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace dsa
