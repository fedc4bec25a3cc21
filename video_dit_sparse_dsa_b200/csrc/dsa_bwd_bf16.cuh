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
// Kernels here:
//   bwd_preprocess      : D = rowsum(dO * O) (fp32);
//   bwd_preprocess_flat : the same for flat (text) rows, with padded LSE and D copies;
//   bwd_bf16_kernel     : key-major and persistent (described above the kernel): dK and dV,
//                         each key row summed by one CTA in a fixed order;
//   bwd_kv_combine      : the flat-key mode's per-part fp32 dK, dV summed in part order.
// dQ comes from the query-major bwd_dq_kernel (dsa_bwd_dq.cuh).  No gradient is summed with
// atomics, so the backward gives the same bits from run to run.
#pragma once

#include <stdint.h>

#include "sm100.cuh"

namespace dsa {

struct BwdBf16Params {
  const int32_t* row_ptr;  // inverse plan: [n_tiles + 1], or per (batch, head) [B*heads, n_tiles + 1]
  int rp_head_stride;      // 0 (one inverse map for every head) or n_tiles + 1
  const int32_t* q_tiles;  // [n_tiles * Wt]
  __nv_bfloat16* dk;       // [BH, N, 128]
  __nv_bfloat16* dv;
  int n_tiles;
  int KU;                  // 128-key units per tile
  int QS;                  // 64-query chunks per tile
  int n_units;             // B*heads * n_tiles * KU
  int G1, G2;
  int tt, th, tw;
  int kcs;                 // t-extent of a 128-token key chunk
  int qcs;                 // t-extent of a 64-token query chunk
  int T, H, W, N;
  float scale, scale_log2;
  // extra (text) query rows after every unit's own query chunks: flat [B*heads, Lxq, 128] Q
  // and dO, LSE and D padded to [B*heads, Lp] (Lp a multiple of 64)
  int Lxq;
  // flat-key mode: the keys are Lk rows of a flat sequence and the main query rows Nq rows
  // of another, in 64-row chunks cut into n_split parts; part j writes fp32 dK, dV at
  // dk_part / dv_part + j * part_stride (the extra queries go with part 0)
  int Lk, Nq, n_split;
  float* dk_part;
  float* dv_part;
  int64_t part_stride;
};

namespace bwd {
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kKBytes = 128 * 128 * 2;  // K or V of a 128-key unit
constexpr uint32_t kKHalf = kKBytes / 2;
constexpr uint32_t kQBytes = 64 * 128 * 2;   // Q or dO of a 64-query chunk
constexpr uint32_t kQHalf = kQBytes / 2;
constexpr uint32_t kStageBytes = 2 * kQBytes + 1024;  // Q, dO, LSE (at +0) and D (at +512) vectors
constexpr uint32_t kOffK = 0, kOffV = kKBytes;
constexpr uint32_t kOffStage = 2 * kKBytes;
// Shared-memory layout: K, V, a 4-stage ring of query chunks (Q, dO, LSE, D), 64 int32 token
// offsets within a query chunk, the barriers.
constexpr int kStages = 4;
constexpr uint32_t kOffRel = kOffStage + kStages * kStageBytes;
constexpr uint32_t kOffBar = kOffRel + 256;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory layout too large");
constexpr uint32_t kTmemCols = 512;  // dV [0,128), dK [128,256), S^T buffers [256,384), dP^T buffers [384,512)
constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, 0, 0);     // K Q^T and V dO^T
constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, 128, 0, 1);  // P^T dO, dS^T Q
// A byte offset added to a shared-memory descriptor's address field (16-byte units).
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }
// Columns (within a chunk's 64-column S^T buffer) of packed bf16 P^T and dS^T for queries
// [16kk, 16kk + 16): two threads share a key row, thread h taking queries [32h, 32h + 32)
// and writing over its own score columns [32h, 32h + 32), P^T in the first 16, dS^T in the
// next 16.
__device__ __forceinline__ uint32_t pt_col(int kk) { return 32u * (kk >> 1) + 8u * (kk & 1); }
__device__ __forceinline__ uint32_t dst_col(int kk) { return 32u * (kk >> 1) + 16u + 8u * (kk & 1); }
}  // namespace bwd

// A work unit: (batch, head), key tile and its 128-key chunk (flat-key mode: the 128-row key
// chunk kt and the part of the query chunks).
struct BwdUnit {
  int bh, kt, ku, part;
};

template <bool kFlatK>
__device__ __forceinline__ BwdUnit bwd_unit(const BwdBf16Params& p, int u) {
  BwdUnit x;
  if constexpr (kFlatK) {
    const int nk = (p.Lk + 127) / 128, per_bh = nk * p.n_split;
    x.bh = u / per_bh;
    const int rem = u % per_bh;
    x.part = rem / nk;
    x.kt = rem % nk;
    x.ku = 0;
  } else {
    x.ku = u % p.KU;
    x.kt = (u / p.KU) % p.n_tiles;
    x.bh = u / (p.KU * p.n_tiles);
    x.part = 0;
  }
  return x;
}

// The unit's 64-query chunks: nm main chunks (the query tiles of CSR row kt of the inverse
// plan from entry row0, or flat chunks from c0), then nx chunks of the extra queries.
struct BwdChunks {
  int row0, c0, nm, nx;
};

template <bool kFlatK, bool kExtra>
__device__ __forceinline__ BwdChunks bwd_chunks(const BwdBf16Params& p, const BwdUnit& x) {
  BwdChunks q;
  const int nx = kExtra ? (p.Lxq + 63) / 64 : 0;
  if constexpr (kFlatK) {
    const int nqm = (p.Nq + 63) / 64, per = (nqm + p.n_split - 1) / p.n_split;
    q.row0 = 0;
    q.c0 = x.part * per;
    q.nm = max(min(per, nqm - q.c0), 0);
    q.nx = x.part == 0 ? nx : 0;
  } else {
    const int32_t* rp = p.row_ptr + static_cast<int64_t>(x.bh) * p.rp_head_stride + x.kt;
    q.row0 = rp[0];
    q.c0 = 0;
    q.nm = (rp[1] - rp[0]) * p.QS;
    q.nx = nx;
  }
  return q;
}

// Query rows present in the unit's chunk c (a flat sequence's last chunk can be partial).
template <bool kFlatK, bool kExtra>
__device__ __forceinline__ int bwd_qvalid(const BwdBf16Params& p, const BwdChunks& q, int c) {
  if (!kFlatK && !kExtra) return 64;
  if (c < q.nm) return kFlatK ? min(p.Nq - 64 * (q.c0 + c), 64) : 64;
  return min(p.Lxq - 64 * (c - q.nm), 64);
}

__device__ __forceinline__ int64_t chunk_row_token(int r, int t0, int h0, int w0, int th, int tw, int H, int W) {
  const int lw = r % tw, lh = (r / tw) % th, lt = r / (tw * th);
  return (static_cast<int64_t>(t0 + lt) * H + (h0 + lh)) * W + (w0 + lw);
}

__global__ void __launch_bounds__(256) bwd_preprocess(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      float* __restrict__ delta, int64_t rows) {
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
  }
#pragma unroll
  for (int o2 = 8; o2 > 0; o2 >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o2);
  if (row < rows && part == 0) delta[row] = s;
}

// bwd_preprocess for flat rows ([B*heads, L, 128]) whose LSE and D are read by 64-row TMA
// boxes: D and a copy of the LSE go to [B*heads, Lp] arrays (Lp a multiple of 64, so every
// box starts 16-byte aligned) with zeros past L.
__global__ void __launch_bounds__(256) bwd_preprocess_flat(const __nv_bfloat16* __restrict__ o,
                                                           const __nv_bfloat16* __restrict__ dout,
                                                           const float* __restrict__ lse, float* __restrict__ delta_pad,
                                                           float* __restrict__ lse_pad, int L, int Lp, int64_t BH) {
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 16;
  const int part = threadIdx.x % 16;
  const bool in = r < BH * Lp;
  const int64_t bh = in ? r / Lp : 0;
  const int i = in ? static_cast<int>(r % Lp) : L;
  const bool live = in && i < L;
  const int64_t row = bh * L + i;
  float s = 0.f;
  if (live) {
    const uint4 a = reinterpret_cast<const uint4*>(o + row * 128)[part];
    const uint4 b = reinterpret_cast<const uint4*>(dout + row * 128)[part];
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 x = __bfloat1622float2(pa[k]);
      const float2 y = __bfloat1622float2(pb[k]);
      s = fmaf(x.x, y.x, s);
      s = fmaf(x.y, y.y, s);
    }
  }
#pragma unroll
  for (int o2 = 8; o2 > 0; o2 >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o2);
  if (in && part == 0) {
    delta_pad[r] = s;
    lse_pad[r] = live ? lse[row] : 0.f;
  }
}

// dK = scale * sum of the parts' dK, dV = sum of their dV (fp32 parts of flat keys), bf16.
__global__ void __launch_bounds__(256) bwd_kv_combine(const float* __restrict__ dk_part,
                                                      const float* __restrict__ dv_part, int n_parts,
                                                      int64_t part_stride, float scale, int64_t n4,
                                                      __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
  for (int j = 0; j < n_parts; ++j) {
    const float4 x = reinterpret_cast<const float4*>(dk_part + j * part_stride)[i];
    const float4 y = reinterpret_cast<const float4*>(dv_part + j * part_stride)[i];
    a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
    b.x += y.x; b.y += y.y; b.z += y.z; b.w += y.w;
  }
  reinterpret_cast<uint2*>(dk)[i] = make_uint2(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale));
  reinterpret_cast<uint2*>(dv)[i] = make_uint2(pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
}

// Persistent, warp-specialised backward; one CTA per SM, one 128-key chunk of a key tile
// per work unit.  The unit walks the 64-query chunks of every query tile whose window
// holds its key tile (the CSR row of the inverse plan).  Roles:
//   warp 8      TMA producer: K and V of the unit, then per query chunk Q, dO, LSE and D
//               through a 4-stage ring;
//   warp 9      MMA issuer, per chunk c (buffer b = c % 2):
//                 S^T_b = K Q_c^T, dP^T_b = V dO_c^T                 (TMEM, 64 columns each)
//                 dV += P^T dO_c, dK += dS^T Q_c (P^T and dS^T read from TMEM)
//               so the scores of chunk c+1 are ready while chunk c's elementwise work runs;
//   warps 0-7   two threads per key row (lane of warps w and w + 4), thread h taking queries
//               [32h, 32h + 32) of every chunk: P^T = exp2(S^T * scale * log2 e - LSE_n *
//               log2 e), dS^T = P^T (dP^T - D_n), both back into TMEM as bf16 over the
//               thread's own score columns (the dV and dK products read them there); at the
//               end of a unit warps 0-3 write dV and warps 4-7 scale * dK as bf16.
// Barriers advance at most one phase ahead of their waiters (each refill of a buffer waits
// for the previous consumer), so waiting by phase parity is unambiguous.
//
// kFlatK: the keys and the main queries are flat sequences (rank-3 / rank-2 maps); rows past
// the end of either load as zeros and get P = dS = 0, and their gradients are not written.
// kExtra: extra queries (p.Lxq of them, flat maps tmQx, tmDOx, tmLsex, tmDx) follow every
// unit's own.
template <bool kFlatK, bool kExtra>
__global__ void __launch_bounds__(bwd::kThreads, 1)
    bwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmLse, const __grid_constant__ CUtensorMap tmD,
                    const __grid_constant__ CUtensorMap tmQx, const __grid_constant__ CUtensorMap tmDOx,
                    const __grid_constant__ CUtensorMap tmLsex, const __grid_constant__ CUtensorMap tmDx,
                    BwdBf16Params p) {
  using namespace bwd;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  int32_t* rel = reinterpret_cast<int32_t*>(smem + kOffRel);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_free = bars + 1;
  uint64_t* ld_full = bars + 2;               // [kStages]
  uint64_t* ld_empty = bars + 2 + kStages;    // [kStages]
  uint64_t* s_full = bars + 2 + 2 * kStages;  // [2]
  uint64_t* p_full = s_full + 2;              // [2]
  uint64_t* dkv_full = s_full + 4;
  uint64_t* dkv_free = s_full + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 6);
  volatile int* abort = reinterpret_cast<volatile int*>(s_full + 7);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    tma_prefetch_map(&tmDO);
    tma_prefetch_map(&tmLse);
    tma_prefetch_map(&tmD);
    if (kExtra && p.Lxq > 0) {
      tma_prefetch_map(&tmQx);
      tma_prefetch_map(&tmDOx);
      tma_prefetch_map(&tmLsex);
      tma_prefetch_map(&tmDx);
    }
    mbar_init(kv_full, 1);
    mbar_init(kv_free, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(ld_full + s, 1);
      mbar_init(ld_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(p_full + b, 8);  // the warps that write P^T and dS^T
    }
    mbar_init(dkv_full, 1);
    mbar_init(dkv_free, 8);  // the warps that read dK and dV out
    *abort = 0;
    fence_mbar_init();
  }
  if (!kFlatK && tid < 64) {
    // token offset of row n of a 64-query chunk box, relative to the box origin
    const int lw = tid % p.tw, lh = (tid / p.tw) % p.th, lt = tid / (p.tw * p.th);
    rel[tid] = (lt * p.H + lh) * p.W + lw;
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tDV = tmem, tDK = tmem + 128, tS = tmem + 256, tDP = tmem + 384;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int ld = 0, uc = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
        const BwdUnit x = bwd_unit<kFlatK>(p, u);
        const BwdChunks qc = bwd_chunks<kFlatK, kExtra>(p, x);
        const int bh = x.bh, n = qc.nm + qc.nx;
        if (n == 0) continue;
        ok = mbar_wait(kv_free, (uc & 1) ^ 1, abort, 50);
        if (!ok) break;
        ++uc;
        mbar_arrive_expect_tx(kv_full, 2 * kKBytes);
        if constexpr (kFlatK) {  // rows past Lk load as zeros
          tma_load_3d(smem + kOffK, &tmK, kv_full, 0, 128 * x.kt, bh);
          tma_load_3d(smem + kOffK + kKHalf, &tmK, kv_full, 64, 128 * x.kt, bh);
          tma_load_3d(smem + kOffV, &tmV, kv_full, 0, 128 * x.kt, bh);
          tma_load_3d(smem + kOffV + kKHalf, &tmV, kv_full, 64, 128 * x.kt, bh);
        } else {
          const int k_t0 = (x.kt / (p.G1 * p.G2)) * p.tt + x.ku * p.kcs;
          const int k_h0 = ((x.kt / p.G2) % p.G1) * p.th, k_w0 = (x.kt % p.G2) * p.tw;
          tma_load_5d(smem + kOffK, &tmK, kv_full, 0, k_w0, k_h0, k_t0, bh);
          tma_load_5d(smem + kOffK + kKHalf, &tmK, kv_full, 64, k_w0, k_h0, k_t0, bh);
          tma_load_5d(smem + kOffV, &tmV, kv_full, 0, k_w0, k_h0, k_t0, bh);
          tma_load_5d(smem + kOffV + kKHalf, &tmV, kv_full, 64, k_w0, k_h0, k_t0, bh);
        }
        for (int c = 0; c < n && ok; ++c, ++ld) {
          const int st = ld % kStages;
          ok = mbar_wait(ld_empty + st, ((ld / kStages) & 1) ^ 1, abort, 51);
          if (!ok) break;
          uint8_t* dst = smem + kOffStage + st * kStageBytes;
          mbar_arrive_expect_tx(ld_full + st, 2 * kQBytes + 512);
          if ((kExtra && c >= qc.nm) || kFlatK) {  // flat rows (past the end: zeros)
            const bool extra = c >= qc.nm;
            const int row = extra ? 64 * (c - qc.nm) : 64 * (qc.c0 + c);
            const CUtensorMap* mq = extra ? &tmQx : &tmQ;
            const CUtensorMap* mdo = extra ? &tmDOx : &tmDO;
            tma_load_3d(dst, mq, ld_full + st, 0, row, bh);
            tma_load_3d(dst + kQHalf, mq, ld_full + st, 64, row, bh);
            tma_load_3d(dst + kQBytes, mdo, ld_full + st, 0, row, bh);
            tma_load_3d(dst + kQBytes + kQHalf, mdo, ld_full + st, 64, row, bh);
            tma_load_2d(dst + 2 * kQBytes, extra ? &tmLsex : &tmLse, ld_full + st, row, bh);
            tma_load_2d(dst + 2 * kQBytes + 512, extra ? &tmDx : &tmD, ld_full + st, row, bh);
          } else {
            const int qi = p.q_tiles[qc.row0 + c / p.QS], qs = c % p.QS;
            const int q_t0 = (qi / (p.G1 * p.G2)) * p.tt + qs * p.qcs;
            const int q_h0 = ((qi / p.G2) % p.G1) * p.th, q_w0 = (qi % p.G2) * p.tw;
            tma_load_5d(dst, &tmQ, ld_full + st, 0, q_w0, q_h0, q_t0, bh);
            tma_load_5d(dst + kQHalf, &tmQ, ld_full + st, 64, q_w0, q_h0, q_t0, bh);
            tma_load_5d(dst + kQBytes, &tmDO, ld_full + st, 0, q_w0, q_h0, q_t0, bh);
            tma_load_5d(dst + kQBytes + kQHalf, &tmDO, ld_full + st, 64, q_w0, q_h0, q_t0, bh);
            tma_load_4d(dst + 2 * kQBytes, &tmLse, ld_full + st, q_w0, q_h0, q_t0, bh);
            tma_load_4d(dst + 2 * kQBytes + 512, &tmD, ld_full + st, q_w0, q_h0, q_t0, bh);
          }
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer (whole warp)
    {
      const uint64_t dK = smem_desc_sw128(sbase + kOffK, 16, 1024);            // K, K-major
      const uint64_t dV = smem_desc_sw128(sbase + kOffV, 16, 1024);            // V, K-major
      const uint64_t dQk = smem_desc_sw128(sbase + kOffStage, 16, 1024);       // stage 0 Q, K-major
      const uint64_t dQm = smem_desc_sw128(sbase + kOffStage, kQHalf, 1024);   // stage 0 Q, MN-major
      int ld = 0, uc = 0, sc = 0, pc = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
        const BwdChunks qc = bwd_chunks<kFlatK, kExtra>(p, bwd_unit<kFlatK>(p, u));
        const int n = qc.nm + qc.nx;
        if (n == 0) continue;
        ok = __all_sync(0xffffffffu, mbar_wait(kv_full, uc & 1, abort, 60));
        if (!ok) break;
        const int ld0 = ld;
        ld += n;
        // S^T and dP^T of chunk c (ring entry ld0 + c) into buffer sc % 2; the first two
        // chunks here, chunk c + 2 after chunk c's gradient products
        for (int c = 0; c < n + 2 && ok; ++c) {
          if (c >= 2) {
            const int cc = c - 2;  // gradient products of chunk cc
            const int b = pc & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(p_full + b, (pc >> 1) & 1, abort, 63));
            ++pc;
            if (ok && cc == 0) ok = __all_sync(0xffffffffu, mbar_wait(dkv_free, (uc & 1) ^ 1, abort, 64));
            if (!ok) break;
            tc_fence_after();
            const uint32_t so = ((ld0 + cc) % kStages) * kStageBytes;
            const uint64_t q_m = desc_add(dQm, so), do_m = desc_add(dQm, so + kQBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // dV += P^T dO
              mma_ts_warp(tDV, tS + b * 64 + pt_col(kk), desc_add(do_m, kk * 2048), kIdescAcc, (cc > 0) || (kk > 0));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // dK += dS^T Q (dS^T from TMEM, beside P^T)
              mma_ts_warp(tDK, tS + b * 64 + dst_col(kk), desc_add(q_m, kk * 2048), kIdescAcc,
                          (cc > 0) || (kk > 0));
            mma_commit_warp(ld_empty + (ld0 + cc) % kStages);
          }
          if (c < n) {
            const int l = ld0 + c, b = sc & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(ld_full + l % kStages, (l / kStages) & 1, abort, 61));
            if (!ok) break;
            tc_fence_after();
            const uint32_t so = (l % kStages) * kStageBytes;
            const uint64_t q_k = desc_add(dQk, so), do_k = desc_add(dQk, so + kQBytes);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t ko = (kk >> 2) * kKHalf + (kk & 3) * 32, qo = (kk >> 2) * kQHalf + (kk & 3) * 32;
              mma_ss_warp(tS + b * 64, desc_add(dK, ko), desc_add(q_k, qo), kIdescS, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t ko = (kk >> 2) * kKHalf + (kk & 3) * 32, qo = (kk >> 2) * kQHalf + (kk & 3) * 32;
              mma_ss_warp(tDP + b * 64, desc_add(dV, ko), desc_add(do_k, qo), kIdescS, kk > 0);
            }
            mma_commit_warp(s_full + b);
            ++sc;
          }
        }
        if (!ok) break;
        mma_commit_warp(dkv_full);
        mma_commit_warp(kv_free);
        ++uc;
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ P^T, dS^T and dK / dV out
    // Two threads per key row (lane of warps w and w + 4): thread h takes queries [32h, 32h + 32)
    // of every chunk.  At the end of a unit warps 0-3 write dV and warps 4-7 scale * dK.
    const int h = warp >> 2;
    const int m = 32 * (warp & 3) + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float kLog2e = 1.4426950408889634f;
    int cc = 0, ld = 0, uc = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      const BwdUnit x = bwd_unit<kFlatK>(p, u);
      const BwdChunks qc = bwd_chunks<kFlatK, kExtra>(p, x);
      const int n = qc.nm + qc.nx;
      // flat keys: this thread's key row may lie past the end (zeros, no gradient)
      const bool k_ok = !kFlatK || 128 * x.kt + m < p.Lk;
      for (int c = 0; c < n; ++c, ++cc, ++ld) {
        const int nvq = bwd_qvalid<kFlatK, kExtra>(p, qc, c) - 32 * h;  // valid queries of this half
        const bool masked = !k_ok || nvq < 32;  // P = dS = 0 for missing keys and queries
        const int b = cc & 1;
        ok = mbar_wait(s_full + b, (cc >> 1) & 1, abort, 70);
        if (ok) ok = mbar_wait(ld_full + ld % kStages, (ld / kStages) & 1, abort, 71);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const float4* lse4 =
            reinterpret_cast<const float4*>(smem + kOffStage + (ld % kStages) * kStageBytes + 2 * kQBytes) + 8 * h;
        const float4* dd4 = lse4 + 32;  // D at +512 bytes
        uint32_t sr[32], dr[32];
        tmem_ld32_wait(tS + lane_off + b * 64 + 32 * h, sr);
        tmem_ld32_wait(tDP + lane_off + b * 64 + 32 * h, dr);
        uint32_t pk[16], dk2[16];
#pragma unroll
        for (int g = 0; g < 8; ++g) {  // queries 32h + 4g .. 32h + 4g + 3
          const float4 lv = lse4[g], dv = dd4[g];
          const float nl[4] = {-lv.x * kLog2e, -lv.y * kLog2e, -lv.z * kLog2e, -lv.w * kLog2e};
          const float dq4[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int n0 = 4 * g + 2 * e;
            float p0 = ex2_approx(fmaf(__uint_as_float(sr[n0]), p.scale_log2, nl[2 * e]));
            float p1 = ex2_approx(fmaf(__uint_as_float(sr[n0 + 1]), p.scale_log2, nl[2 * e + 1]));
            if (masked) {
              if (!k_ok || n0 >= nvq) p0 = 0.f;
              if (!k_ok || n0 + 1 >= nvq) p1 = 0.f;
            }
            pk[2 * g + e] = pack_bf16x2(p0, p1);
            dk2[2 * g + e] = pack_bf16x2(p0 * (__uint_as_float(dr[n0]) - dq4[2 * e]),
                                         p1 * (__uint_as_float(dr[n0 + 1]) - dq4[2 * e + 1]));
          }
        }
        tmem_st16(tS + lane_off + b * 64 + 32 * h, pk);        // P^T over this thread's own score columns
        tmem_st16(tS + lane_off + b * 64 + 32 * h + 16, dk2);  // dS^T beside it
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + b);
      }
      if (!ok) break;
      // dV (warps 0-3) or scale * dK (warps 4-7) of the unit's 128 keys; zeros for a key tile
      // no window holds.  Flat keys: fp32 partial sums of this part (unscaled dK), rows past
      // Lk not written.
      int64_t ktok;
      bool k_row_ok = true;
      if constexpr (kFlatK) {
        ktok = 128 * static_cast<int64_t>(x.kt) + m;
        k_row_ok = ktok < p.Lk;
        if (!k_row_ok) ktok = 0;
      } else {
        const int k_t0 = (x.kt / (p.G1 * p.G2)) * p.tt + x.ku * p.kcs;
        const int k_h0 = ((x.kt / p.G2) % p.G1) * p.th, k_w0 = (x.kt % p.G2) * p.tw;
        ktok = chunk_row_token(m, k_t0, k_h0, k_w0, p.th, p.tw, p.H, p.W);
      }
      const int64_t slice = static_cast<int64_t>(x.bh) * p.N;
      __nv_bfloat16* outp = h ? p.dk : p.dv;
      const float sc_out = h ? p.scale : 1.f;
      uint4* dst = reinterpret_cast<uint4*>(outp + (slice + ktok) * 128);
      float4* dstp = nullptr;
      if constexpr (kFlatK) {
        const int64_t o = static_cast<int64_t>(x.part) * p.part_stride + (static_cast<int64_t>(x.bh) * p.Lk + ktok) * 128;
        dstp = reinterpret_cast<float4*>((h ? p.dk_part : p.dv_part) + o);
      }
      if (n > 0) {
        ok = mbar_wait(dkv_full, uc & 1, abort, 81);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
#pragma unroll 1
      for (int g = 0; g < 4; ++g) {
        uint32_t a[32];
        if (n > 0) {
          tmem_ld32_wait((h ? tDK : tDV) + lane_off + g * 32, a);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) a[j] = 0u;
        }
        if constexpr (kFlatK) {
          if (k_row_ok) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dstp[g * 8 + j] = make_float4(__uint_as_float(a[4 * j]), __uint_as_float(a[4 * j + 1]),
                                            __uint_as_float(a[4 * j + 2]), __uint_as_float(a[4 * j + 3]));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 y;
            y.x = pack_bf16x2(__uint_as_float(a[8 * j + 0]) * sc_out, __uint_as_float(a[8 * j + 1]) * sc_out);
            y.y = pack_bf16x2(__uint_as_float(a[8 * j + 2]) * sc_out, __uint_as_float(a[8 * j + 3]) * sc_out);
            y.z = pack_bf16x2(__uint_as_float(a[8 * j + 4]) * sc_out, __uint_as_float(a[8 * j + 5]) * sc_out);
            y.w = pack_bf16x2(__uint_as_float(a[8 * j + 6]) * sc_out, __uint_as_float(a[8 * j + 7]) * sc_out);
            dst[g * 4 + j] = y;
          }
        }
      }
      if (n > 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dkv_free);
        ++uc;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace dsa
