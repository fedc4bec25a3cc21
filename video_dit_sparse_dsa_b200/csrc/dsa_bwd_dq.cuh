// dQ of the 3D-DSA backward, query-major and deterministic ("MegaSlide-DiT: Memory-Centric
// Adaptation and Deformable Local Attention for Efficient Video Diffusion", abstract:
// full-parameter adaptation needs the gradients of the attention inputs).
//
// For query token n with key set K(i) of its tile i:
//   P_nm = exp(scale q_n.k_m - LSE_n),  dS_nm = P_nm (dO_n.v_m - D_n),  dQ_n = scale sum_m dS_nm k_m,
// with LSE the forward's and D_n = dO_n.O_n (bwd_preprocess).  A work unit is one 128-row
// query chunk of one query tile of one (batch, head); it walks its window's keys 128 at a
// time ("steps"), recomputes S = Q K^T and dP = dO V^T on the tensor cores, forms dS in
// registers and accumulates dQ += dS K in TMEM.  Each dQ row is summed by one CTA in the
// fixed order of the unit's key list and written once as bf16: no atomics, and the result is
// identical from run to run.  (The key-major kernel computes dK and dV; together the two
// passes are the whole backward.)
//
// Persistent and warp-specialised, one CTA per SM, 384 threads:
//   warp 8      TMA producer of Q and dO (once per unit) and of K (a 3-stage ring: a K
//               chunk is read by the score product of its step and by the dQ product, which
//               is issued one step later);
//   warp 10     TMA producer of V (2-stage ring, read by the dP product only);
//   warp 9      MMA issuer (a converged warp; one elected lane issues), per step t:
//                 S(t+1) = Q K(t+1)^T and dP(t+1) = dO V(t+1)^T once the elementwise warps
//                 hold S(t) and dP(t) in registers, then dQ += dS(t) K(t) with dS from TMEM;
//   warp 11     idle (its warpgroup's registers go to the elementwise warpgroups);
//   warps 0-7   elementwise: warpgroup i (warps 4i..4i+3) takes keys [64i, 64i+64) of every
//               step, one thread per query row: P = 2^(S scale log2 e - LSE log2 e),
//               dS = P (dP - D), packed to bf16 into TMEM; at the end of a unit each writes
//               half of the row's 128 channels of dQ = scale * accumulator.
// TMEM (512 columns): regions A [0,128), B [128,256), C [256,384) and the dQ accumulator
// [384,512).  A step of parity e puts S in A (e = 0) or C (e = 1) and dP in B; the dS of
// keys [64i, 64i+64) goes to columns [64i, 64i+32) of S's region, over the S columns the
// same threads have already loaded.  So S(t+1) never lands on the dS(t) the dQ product
// still reads, and dP(t+1) only needs the elementwise warps to have loaded dP(t).
// Units are ordered head, tile, chunk, as in the forward (the chunks of a tile read the
// same keys at the same time).
#pragma once

#include <stdint.h>

#include "sm100.cuh"

namespace dsa {

struct BwdDqParams {
  const int32_t* kv_tiles;  // window form: [n_tiles, Wt]; list form: the caller's list [nnz]
  const int32_t* row_ptr;   // list form: CSR offsets into kv_tiles; null: window form
  int rp_head_stride;       // list form: 0 (one list for every head) or n_tiles + 1
  int nnz;
  const float* lse;         // [B*heads, N] natural log (the forward's)
  const float* delta;       // [B*heads, N] D = rowsum(dO * O)
  __nv_bfloat16* dq;        // [B*heads, N, 128]
  int n_tiles, Wt;
  int S;                    // 128-row chunks per tile (query chunks and key chunks alike)
  int n_units;              // B*heads * n_tiles * S
  int G1, G2;
  int tt, th, tw, tcs;      // tile shape; t-extent of a 128-token chunk
  int T, H, W, N;
  float scale, scale_log2;
};

namespace bdq {
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;  // Q, dO, K
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10;
constexpr int kRegsElem = 216;
constexpr int kRegsAux = 72;
constexpr int kRegsAtLaunch = (2 * 128 * kRegsElem + 128 * kRegsAux) / kThreads;  // 168
static_assert(kRegsAtLaunch * kThreads == 2 * 128 * kRegsElem + 128 * kRegsAux, "split must use the launch registers");
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t kTileBytes = 128 * 128 * 2;  // 128 tokens x 128 channels, bf16
constexpr uint32_t kHalfBytes = kTileBytes / 2;
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffDO = kTileBytes;
constexpr uint32_t kOffK = 2 * kTileBytes;
constexpr uint32_t kOffV = kOffK + kKStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kVStages * kTileBytes;
constexpr uint32_t kSmemUsed = kOffBar + 256;
constexpr uint32_t kSmemBytes = 227 * 1024;
static_assert(kSmemUsed + 1023 <= kSmemBytes, "shared memory layout too large for any base alignment");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColB = 128, kColDQ = 384;
constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);   // Q K^T, dO V^T: both K-major
constexpr uint32_t kIdescDQ = idesc_bf16_f32(128, 128, 0, 1);  // dS (TMEM) K: K as the MN-major B
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }
__device__ __forceinline__ uint32_t col_s(int e) { return e ? 256u : 0u; }

// S = A B^T over 128 channels for a K-major 128-row A and B (8 k-steps of 16 in two
// 64-channel halves).
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t o = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
    mma_ss_warp(d_tmem, desc_add(a_desc, o), desc_add(b_desc, o), kIdescS, kk > 0);
  }
}

// dQ (+)= dS K over one 128-key step: dS of keys [16kk, 16kk+16) at TMEM columns
// 8kk (kk < 4) and 64 + 8(kk - 4) (kk >= 4) of its region; K an MN-major tile, 16 keys =
// 2048 bytes per k-step.
__device__ __forceinline__ void issue_dq(uint32_t d_tmem, uint32_t ds_tmem, uint64_t k_desc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts_warp(d_tmem, ds_tmem + (kk >> 2) * 64 + (kk & 3) * 8, desc_add(k_desc, kk * 2048), kIdescDQ,
                accumulate || kk > 0);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int site) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, site));
}

struct Unit {
  int bh, tile, sub;
};

__device__ __forceinline__ Unit decode(const BwdDqParams& p, int u) {
  Unit x;
  const int per_bh = p.S * p.n_tiles;
  x.bh = u / per_bh;
  const int rem = u % per_bh;
  x.tile = rem / p.S;
  x.sub = rem % p.S;
  return x;
}

// Key tiles of query tile `tile` (window plan or the caller's list, every index clamped
// into the list: an invalid list gives wrong numbers, never an access outside it).
__device__ __forceinline__ const int32_t* unit_keys(const BwdDqParams& p, int bh, int tile, int& n_list) {
  if (p.row_ptr == nullptr) {
    n_list = p.Wt;
    return p.kv_tiles + static_cast<int64_t>(tile) * p.Wt;
  }
  const int32_t* rp = p.row_ptr + static_cast<int64_t>(bh) * p.rp_head_stride;
  const int a = min(max(rp[tile], 0), p.nnz), b = min(max(rp[tile + 1], a), p.nnz);
  n_list = b - a;
  return p.kv_tiles + a;
}

// Token index of row r of 128-row chunk `sub` of tile `tile`.
__device__ __forceinline__ int64_t chunk_token(const BwdDqParams& p, int tile, int sub, int r) {
  const int qt = tile / (p.G1 * p.G2), qh = (tile / p.G2) % p.G1, qw = tile % p.G2;
  const int lw = r % p.tw, lh = (r / p.tw) % p.th, lt = r / (p.tw * p.th);
  const int t0 = qt * p.tt + sub * p.tcs;
  return (static_cast<int64_t>(t0 + lt) * p.H + (qh * p.th + lh)) * p.W + (qw * p.tw + lw);
}
}  // namespace bdq

__global__ void __launch_bounds__(bdq::kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO, BwdDqParams p) {
  using namespace bdq;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  if (pad + kSmemUsed > kSmemBytes) {  // uniform over the CTA: nothing has started yet
    if (threadIdx.x == 0) device_report(DSA_DEV_BOUNDS, 3);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* qd_full = bars + 0;
  uint64_t* qd_empty = bars + 1;
  uint64_t* k_full = bars + 2;               // [kKStages]
  uint64_t* k_empty = k_full + kKStages;     // [kKStages]
  uint64_t* v_full = k_empty + kKStages;     // [kVStages]
  uint64_t* v_empty = v_full + kVStages;     // [kVStages]
  uint64_t* s_full = v_empty + kVStages;     // [2] S and dP of a step of parity e ready
  uint64_t* s_read = s_full + 2;             // [2] ... loaded by the elementwise warps (8)
  uint64_t* ds_full = s_full + 4;            // [2] dS of a step of parity e written (8)
  uint64_t* dq_done = s_full + 6;            // every dQ product of a unit done
  uint64_t* dq_free = s_full + 7;            // dQ read out (8)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 8);
  volatile int* abort = reinterpret_cast<volatile int*>(s_full + 9);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    tma_prefetch_map(&tmDO);
    mbar_init(qd_full, 1);
    mbar_init(qd_empty, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int e = 0; e < 2; ++e) {
      mbar_init(s_full + e, 1);
      mbar_init(s_read + e, 8);
      mbar_init(ds_full + e, 8);
    }
    mbar_init(dq_done, 1);
    mbar_init(dq_free, 8);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kProducerWarp) {
    setmaxnreg_dec<kRegsAux>();
    if (warp == kProducerWarp || warp == kVProducerWarp) {
      // ------------------------------------------------------------------ TMA producers
      if (lane == 0) {
        const bool is_k = warp == kProducerWarp;
        int ld = 0, uc = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
          const Unit x = decode(p, u);
          int n_list = 0;
          const int32_t* kv = unit_keys(p, x.bh, x.tile, n_list);
          const int n_steps = n_list * p.S;
          if (n_steps == 0) continue;  // no keys: the elementwise warps write dQ = 0
          if (is_k) {
            ok = mbar_wait(qd_empty, (uc & 1) ^ 1, abort, 110);
            if (!ok) break;
            const int qt = x.tile / (p.G1 * p.G2), qh = (x.tile / p.G2) % p.G1, qw = x.tile % p.G2;
            const int t0 = qt * p.tt + x.sub * p.tcs;
            mbar_arrive_expect_tx(qd_full, 2 * kTileBytes);
            tma_load_5d(smem + kOffQ, &tmQ, qd_full, 0, qw * p.tw, qh * p.th, t0, x.bh);
            tma_load_5d(smem + kOffQ + kHalfBytes, &tmQ, qd_full, 64, qw * p.tw, qh * p.th, t0, x.bh);
            tma_load_5d(smem + kOffDO, &tmDO, qd_full, 0, qw * p.tw, qh * p.th, t0, x.bh);
            tma_load_5d(smem + kOffDO + kHalfBytes, &tmDO, qd_full, 64, qw * p.tw, qh * p.th, t0, x.bh);
          }
          ++uc;
          const int n_st = is_k ? kKStages : kVStages;
          for (int j = 0; j < n_steps && ok; ++j, ++ld) {
            const int st = ld % n_st;
            ok = mbar_wait((is_k ? k_empty : v_empty) + st, ((ld / n_st) & 1) ^ 1, abort, is_k ? 111 : 112);
            if (!ok) break;
            const int kt = min(max(kv[j / p.S], 0), p.n_tiles - 1), ks = j % p.S;
            const int t0 = (kt / (p.G1 * p.G2)) * p.tt + ks * p.tcs;
            const int h0 = ((kt / p.G2) % p.G1) * p.th, w0 = (kt % p.G2) * p.tw;
            uint64_t* full = (is_k ? k_full : v_full) + st;
            uint8_t* dst = smem + (is_k ? kOffK : kOffV) + st * kTileBytes;
            mbar_arrive_expect_tx(full, kTileBytes);
            tma_load_5d(dst, is_k ? &tmK : &tmV, full, 0, w0, h0, t0, x.bh);
            tma_load_5d(dst + kHalfBytes, is_k ? &tmK : &tmV, full, 64, w0, h0, t0, x.bh);
          }
        }
      }
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------------------ MMA issuer (whole warp)
      const uint64_t dQd = smem_desc_sw128(sbase + kOffQ, 16, 1024);
      const uint64_t dDO = smem_desc_sw128(sbase + kOffDO, 16, 1024);
      const uint64_t dKk = smem_desc_sw128(sbase + kOffK, 16, 1024);          // K stage 0, K-major
      const uint64_t dKm = smem_desc_sw128(sbase + kOffK, kHalfBytes, 1024);  // K stage 0, MN-major
      const uint64_t dVk = smem_desc_sw128(sbase + kOffV, 16, 1024);          // V stage 0, K-major
      int ks = 0, kd = 0, vs = 0;  // K stages taken by the score and by the dQ products, V stages
      int uc = 0, g = 0;           // units with keys, steps before the current unit
      int rc0 = 0, rc1 = 0;        // phases of s_read[0 / 1] consumed (ds_full alike)
      bool ok = true;
      // S and dP of one step into the region of parity e; the V stage is released when they are done
      auto issue_step = [&](int e) -> bool {
        if (!warp_wait(k_full + ks % kKStages, (ks / kKStages) & 1, abort, 121)) return false;
        if (!warp_wait(v_full + vs % kVStages, (vs / kVStages) & 1, abort, 122)) return false;
        tc_fence_after();
        issue_qk(tmem + col_s(e), dQd, desc_add(dKk, (ks % kKStages) * kTileBytes));
        issue_qk(tmem + kColB, dDO, desc_add(dVk, (vs % kVStages) * kTileBytes));
        mma_commit_warp(s_full + e);
        mma_commit_warp(v_empty + vs % kVStages);
        ++ks;
        ++vs;
        return true;
      };
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
        int n_list = 0;
        const Unit x = decode(p, u);
        unit_keys(p, x.bh, x.tile, n_list);
        const int n_steps = n_list * p.S;
        if (n_steps == 0) continue;
        ok = warp_wait(qd_full, uc & 1, abort, 120);
        if (ok) ok = issue_step(g & 1);
        if (!ok) break;
        if (n_steps == 1) mma_commit_warp(qd_empty);
        for (int t = 0; t < n_steps && ok; ++t) {
          const int e = (g + t) & 1;
          const int ph = (e == 0 ? rc0++ : rc1++) & 1;
          ok = warp_wait(s_read + e, ph, abort, 123);
          if (!ok) break;
          if (t + 1 < n_steps) {
            // the elementwise warps hold S(t) and dP(t): S(t+1) goes to the other region, dP(t+1) to B
            ok = issue_step(e ^ 1);
            if (!ok) break;
            if (t + 2 == n_steps) mma_commit_warp(qd_empty);  // every product reading Q and dO issued
          }
          ok = warp_wait(ds_full + e, ph, abort, 124);
          if (ok && t == 0) ok = warp_wait(dq_free, (uc & 1) ^ 1, abort, 125);
          if (!ok) break;
          tc_fence_after();
          issue_dq(tmem + kColDQ, tmem + col_s(e), desc_add(dKm, (kd % kKStages) * kTileBytes), t > 0);
          mma_commit_warp(k_empty + kd % kKStages);
          ++kd;
        }
        if (!ok) break;
        mma_commit_warp(dq_done);
        g += n_steps;
        ++uc;
      }
    }
  } else {
    setmaxnreg_inc<kRegsElem>();
    // ------------------------------------------------------------------ elementwise (P, dS) and dQ out
    // Every barrier is waited on at most one phase behind its completions: s_full alternates
    // with the step parity and each phase needs the previous step's s_read; dq_done completes
    // once per unit and the next completion needs this warpgroup's dq_free arrival.
    const int i = warp >> 2;
    const int r = tid & 127;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float kLog2e = 1.4426950408889634f;
    int sc0 = 0, sc1 = 0, g = 0, uc = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      const Unit x = decode(p, u);
      int n_list = 0;
      unit_keys(p, x.bh, x.tile, n_list);
      const int n_steps = n_list * p.S;
      const int64_t row = static_cast<int64_t>(x.bh) * p.N + chunk_token(p, x.tile, x.sub, r);
      uint4* dst = reinterpret_cast<uint4*>(p.dq + row * 128) + 8 * i;
      if (n_steps == 0) {  // no keys: no gradient
#pragma unroll
        for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
        continue;
      }
      const float neg_lse2 = -p.lse[row] * kLog2e, dd = p.delta[row];
      for (int t = 0; t < n_steps; ++t) {
        const int e = (g + t) & 1;
        ok = warp_wait(s_full + e, (e == 0 ? sc0++ : sc1++) & 1, abort, 130);
        if (!ok) break;
        tc_fence_after();
        uint32_t s[64], dp[64];
        tmem_ld64_wait(tmem + col_s(e) + 64 * i + lane_off, s);
        tmem_ld64_wait(tmem + kColB + 64 * i + lane_off, dp);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_read + e);  // dP(t+1) may now go into B
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          float x0, x1;
          ffma2(x0, x1, __uint_as_float(s[c]), __uint_as_float(s[c + 1]), p.scale_log2, p.scale_log2, neg_lse2,
                neg_lse2);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          s[c >> 1] = pack_bf16x2(p0 * (__uint_as_float(dp[c]) - dd), p1 * (__uint_as_float(dp[c + 1]) - dd));
        }
        {
          uint32_t w[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) w[c] = s[c];
          tmem_st32(tmem + col_s(e) + 64 * i + lane_off, w);  // over this thread's own S columns
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full + e);
      }
      if (!ok) break;
      // epilogue: dQ = scale * accumulator, channels [64i, 64i + 64) of the row
      ok = warp_wait(dq_done, uc & 1, abort, 131);
      if (!ok) break;
      tc_fence_after();
      uint32_t a[32], b[32];
      tmem_ld32_wait(tmem + kColDQ + 64 * i + lane_off, a);
      tmem_ld32_wait(tmem + kColDQ + 64 * i + 32 + lane_off, b);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_free);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(a[8 * c + 0]) * p.scale, __uint_as_float(a[8 * c + 1]) * p.scale);
        v.y = pack_bf16x2(__uint_as_float(a[8 * c + 2]) * p.scale, __uint_as_float(a[8 * c + 3]) * p.scale);
        v.z = pack_bf16x2(__uint_as_float(a[8 * c + 4]) * p.scale, __uint_as_float(a[8 * c + 5]) * p.scale);
        v.w = pack_bf16x2(__uint_as_float(a[8 * c + 6]) * p.scale, __uint_as_float(a[8 * c + 7]) * p.scale);
        dst[c] = v;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(b[8 * c + 0]) * p.scale, __uint_as_float(b[8 * c + 1]) * p.scale);
        v.y = pack_bf16x2(__uint_as_float(b[8 * c + 2]) * p.scale, __uint_as_float(b[8 * c + 3]) * p.scale);
        v.z = pack_bf16x2(__uint_as_float(b[8 * c + 4]) * p.scale, __uint_as_float(b[8 * c + 5]) * p.scale);
        v.w = pack_bf16x2(__uint_as_float(b[8 * c + 6]) * p.scale, __uint_as_float(b[8 * c + 7]) * p.scale);
        dst[4 + c] = v;
      }
      g += n_steps;
      ++uc;
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
