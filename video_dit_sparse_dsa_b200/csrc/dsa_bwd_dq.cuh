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
//   warp 8      TMA producer of K (128-key chunks, a 4-entry ring: a K chunk is read by the
//               score product of its step, issued a step early, and by the dQ product of
//               its step);
//   warp 10     TMA producer of V (128-key chunks, 3-entry ring, read by the dP product only);
//   warp 9      MMA issuer (a converged warp; one elected lane issues), per step t: once
//               the elementwise warps hold S(t) in registers, S(t+1) = Q K(t+1)^T; once
//               they have written dS(t), dQ += dS(t) K(t), then dP(t+1) = dO V(t+1)^T; Q
//               and dO are read from TMEM.  So the next scores run during the elementwise
//               work of step t and only dP(t+1) waits for dS(t);
//   warp 11     idle (its warpgroup's registers go to the elementwise warpgroups);
//   warps 0-7   elementwise: two threads per query row (lane of warps w and w + 4).  At the
//               start of a unit thread 0 of a row loads the row of Q, thread 1 that of dO,
//               from global memory into TMEM (no shared-memory staging: its 64 KB go to
//               deeper K and V rings).  Per step thread h takes keys
//               [64h, 64h + 64): P = 2^(S scale log2 e - LSE log2 e) as soon as S is in (the
//               score buffer is then released), then with dP: dS = P (dP - D), packed to
//               bf16 into TMEM over its own dP columns; at the end of a unit each writes
//               half of the row's 128 channels of dQ = scale * accumulator.
// Steps of 128 keys rather than 64: each step costs a fixed round of barrier hand-offs
// between the elementwise warps and the MMA warp (arrive, wake, issue, commit, wake), about
// 1300 clocks with no work at all, which 64-key steps paid twice as often.
// Every product takes its A operand (Q, dO or dS) from TMEM, so shared memory holds only the
// K and V rings and carries their operand reads and fills: 160 KB per 128-key step against
// 1536 cycles of products, inside its bandwidth.
// TMEM (512 columns): Q [0,64) and dO [64,128) as packed bf16 pairs, the scores [128,256),
// dP (then dS) [256,384), the dQ accumulator [384,512).  S(t + 1) overwrites the scores
// once every elementwise warp has loaded S(t) (s_read); dP(t + 1) overwrites dS(t) after the
// dQ product of step t, which reads it, is issued (products run in issue order).  A unit's
// Q and dO are overwritten only after the elementwise warps have seen the unit's last
// scores and dP, i.e. after its last score products.
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
  const __nv_bfloat16* q;   // the queries' rows: [B*heads, N, 128] (flat mode: [B*heads, Lq, 128])
  const __nv_bfloat16* dout;  // dO, laid out as q
  const float* lse;         // [B*heads, N] natural log (the forward's)
  const float* delta;       // [B*heads, N] D = rowsum(dO * O)
  __nv_bfloat16* dq;        // [B*heads, N, 128]
  int n_tiles, Wt;
  int S;                    // 128-row chunks per tile (the unit is one of them)
  int KS;                   // 128-key chunks per tile (a step is one of them)
  int n_units;              // B*heads * n_tiles * S
  int G1, G2;
  int tt, th, tw;
  int tcs;                  // t-extent of a 128-token query chunk
  int kcs;                  // t-extent of a 128-token key chunk
  int T, H, W, N;
  float scale, scale_log2;
  // extra (text) keys after every unit's own: Lx rows of flat [B*heads, Lx, 128] K and V
  // (0: none); the tail of their last 128-row chunk is masked
  int Lx;
  // flat mode: the query rows are Lq rows of a flat [B*heads, Lq, 128] sequence (lse, delta
  // [B*heads, Lq]) and the keys Lk rows of another, in 128-row chunks cut into n_split parts
  // (the extra keys go with part 0); part j writes fp32 scale * dQ to dq_part + j * part_stride
  int Lq, Lk, n_split;
  float* dq_part;
  int64_t part_stride;
  int ld_rows;              // flat mode: rows per (batch, head) of lse and delta (>= Lq)
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
constexpr int kKStages = 4;
constexpr int kVStages = 3;
constexpr uint32_t kKTileBytes = 128 * 128 * 2;  // 128 keys x 128 channels
constexpr uint32_t kKHalfBytes = kKTileBytes / 2;
constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kOffK + kKStages * kKTileBytes;
constexpr uint32_t kOffBar = kOffV + kVStages * kKTileBytes;
constexpr uint32_t kSmemUsed = kOffBar + 512;
constexpr uint32_t kSmemBytes = 227 * 1024;
static_assert(kSmemUsed + 1023 <= kSmemBytes, "shared memory layout too large for any base alignment");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0, kColDO = 64, kColS = 128, kColDP = 256, kColDQ = 384;
constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);   // Q K^T, dO V^T: both K-major, 128 keys
constexpr uint32_t kIdescDQ = idesc_bf16_f32(128, 128, 0, 1);  // dS (TMEM) K: K as the MN-major B
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

// D = A B^T over 128 channels for A (128 rows) in TMEM as packed bf16 pairs, 8 columns per
// 16 channels, and a K-major B of 128 rows in shared memory (two 64-channel halves of
// 16 KB): 8 k-steps of 16 channels.
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts_warp(d_tmem, a_tmem + 8 * kk, desc_add(b_desc, (kk >> 2) * kKHalfBytes + (kk & 3) * 32), kIdescS, kk > 0);
}

// dQ (+)= dS K over one 128-key step: dS of keys [16kk, 16kk + 16) at TMEM columns
// 64 (kk >> 2) + 8 (kk & 3) of the dP buffer (thread h wrote keys [64h, 64h + 64) over its
// own dP columns); K an MN-major tile, 16 keys = 2048 bytes per k-step.
__device__ __forceinline__ void issue_dq(uint32_t d_tmem, uint32_t ds_tmem, uint64_t k_desc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts_warp(d_tmem, ds_tmem + 64 * (kk >> 2) + 8 * (kk & 3), desc_add(k_desc, kk * 2048), kIdescDQ,
                accumulate || kk > 0);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int site) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, site));
}

struct Unit {
  int bh, tile, sub;
};

// Window / list form: units run (batch*head, tile, chunk).  Flat form: (batch*head, part,
// query chunk), so the query chunks that read the same keys are neighbours; tile = the query
// chunk, sub = the part.
template <bool kFlat>
__device__ __forceinline__ Unit decode(const BwdDqParams& p, int u) {
  Unit x;
  if constexpr (kFlat) {
    const int nq = (p.Lq + 127) / 128, per_bh = nq * p.n_split;
    x.bh = u / per_bh;
    const int rem = u % per_bh;
    x.sub = rem / nq;
    x.tile = rem % nq;
  } else {
    const int per_bh = p.S * p.n_tiles;
    x.bh = u / per_bh;
    const int rem = u % per_bh;
    x.tile = rem / p.S;
    x.sub = rem % p.S;
  }
  return x;
}

// The unit's 128-key chunks: nm main chunks from main chunk c0 (the listed tiles' chunks, or
// rows of the flat key sequence), then nx chunks of the extra keys.
struct Chunks {
  int c0, nm, nx;
};

template <bool kFlat, bool kExtra>
__device__ __forceinline__ Chunks unit_chunks(const BwdDqParams& p, const Unit& x, int n_list) {
  Chunks k;
  const int nx = kExtra ? (p.Lx + 127) / 128 : 0;
  if constexpr (kFlat) {
    const int n_main = (p.Lk + 127) / 128, per = (n_main + p.n_split - 1) / p.n_split;
    k.c0 = x.sub * per;
    k.nm = max(min(per, n_main - k.c0), 0);
    k.nx = x.sub == 0 ? nx : 0;
  } else {
    k.c0 = 0;
    k.nm = n_list * p.KS;
    k.nx = nx;
  }
  return k;
}

// Keys present in local chunk j: the last chunk of a flat sequence and of the extra keys can
// be partial.
template <bool kFlat, bool kExtra>
__device__ __forceinline__ int chunk_valid(const BwdDqParams& p, const Chunks& k, int j) {
  if (!kFlat && !kExtra) return 128;
  if (j < k.nm) return kFlat ? min(p.Lk - 128 * (k.c0 + j), 128) : 128;
  return min(p.Lx - 128 * (j - k.nm), 128);
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

// kFlat: flat query rows over flat key rows in parts (rank-3 maps; rows past the end load as
// zeros, keys past the end are masked, rows past the end are not written).  kExtra: the
// extra keys (maps tmKx, tmVx) follow every unit's own.
template <bool kFlat, bool kExtra>
__global__ void __launch_bounds__(bdq::kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmKx, const __grid_constant__ CUtensorMap tmVx, BwdDqParams p) {
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
  uint64_t* k_full = bars + 0;               // [kKStages]
  uint64_t* k_empty = k_full + kKStages;     // [kKStages]
  uint64_t* v_full = k_empty + kKStages;     // [kVStages]
  uint64_t* v_empty = v_full + kVStages;     // [kVStages]
  uint64_t* s_full = v_empty + kVStages;     // S of a step ready
  uint64_t* dp_full = s_full + 1;            // dP of a step ready
  uint64_t* s_read = s_full + 2;             // S of a step loaded (8)
  uint64_t* ds_full = s_full + 3;            // dS of a step written (8)
  uint64_t* dq_done = s_full + 4;            // every dQ product of a unit done
  uint64_t* dq_free = s_full + 5;            // dQ read out (8)
  uint64_t* qa_full = s_full + 6;            // the unit's Q and dO are in TMEM (8)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 7);
  volatile int* abort = reinterpret_cast<volatile int*>(s_full + 8);
  static_assert(2 * kKStages + 2 * kVStages + 9 <= 512 / 8, "barriers must fit their 512 bytes");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    if (kExtra && p.Lx > 0) {
      tma_prefetch_map(&tmKx);
      tma_prefetch_map(&tmVx);
    }
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(s_read, 8);
    mbar_init(ds_full, 8);
    mbar_init(dq_done, 1);
    mbar_init(dq_free, 8);
    mbar_init(qa_full, 8);
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
        int ld = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
          const Unit x = decode<kFlat>(p, u);
          int n_list = 0;
          const int32_t* kv = kFlat ? nullptr : unit_keys(p, x.bh, x.tile, n_list);
          const Chunks ck = unit_chunks<kFlat, kExtra>(p, x, n_list);
          const int n_steps = ck.nm + ck.nx;
          if (n_steps == 0) continue;  // no keys: the elementwise warps write dQ = 0
          const int n_st = is_k ? kKStages : kVStages;
          for (int j = 0; j < n_steps && ok; ++j, ++ld) {
            const int st = ld % n_st;
            ok = mbar_wait((is_k ? k_empty : v_empty) + st, ((ld / n_st) & 1) ^ 1, abort, is_k ? 111 : 112);
            if (!ok) break;
            uint64_t* full = (is_k ? k_full : v_full) + st;
            uint8_t* dst = smem + (is_k ? kOffK : kOffV) + st * kKTileBytes;
            mbar_arrive_expect_tx(full, kKTileBytes);
            if (kExtra && j >= ck.nm) {  // extra keys (rows past Lx load as zeros and are masked)
              const CUtensorMap* m = is_k ? &tmKx : &tmVx;
              tma_load_3d(dst, m, full, 0, 128 * (j - ck.nm), x.bh);
              tma_load_3d(dst + kKHalfBytes, m, full, 64, 128 * (j - ck.nm), x.bh);
            } else if (kFlat) {  // flat key rows (past Lk: zeros, masked)
              const CUtensorMap* m = is_k ? &tmK : &tmV;
              tma_load_3d(dst, m, full, 0, 128 * (ck.c0 + j), x.bh);
              tma_load_3d(dst + kKHalfBytes, m, full, 64, 128 * (ck.c0 + j), x.bh);
            } else {
              const int kt = min(max(kv[j / p.KS], 0), p.n_tiles - 1), ks = j % p.KS;
              const int t0 = (kt / (p.G1 * p.G2)) * p.tt + ks * p.kcs;
              const int h0 = ((kt / p.G2) % p.G1) * p.th, w0 = (kt % p.G2) * p.tw;
              tma_load_5d(dst, is_k ? &tmK : &tmV, full, 0, w0, h0, t0, x.bh);
              tma_load_5d(dst + kKHalfBytes, is_k ? &tmK : &tmV, full, 64, w0, h0, t0, x.bh);
            }
          }
        }
      }
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------------------ MMA issuer (whole warp)
      const uint64_t dKk = smem_desc_sw128(sbase + kOffK, 16, 1024);           // K stage 0, K-major
      const uint64_t dKm = smem_desc_sw128(sbase + kOffK, kKHalfBytes, 1024);  // K stage 0, MN-major
      const uint64_t dVk = smem_desc_sw128(sbase + kOffV, 16, 1024);           // V stage 0, K-major
      int ks = 0, kd = 0, vs = 0;  // K stages taken by the score and by the dQ products, V stages
      int uc = 0, g = 0;           // units with keys, steps before the current unit
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
        int n_list = 0;
        const Unit x = decode<kFlat>(p, u);
        if constexpr (!kFlat) unit_keys(p, x.bh, x.tile, n_list);
        const int n_steps = unit_chunks<kFlat, kExtra>(p, x, n_list).nm + unit_chunks<kFlat, kExtra>(p, x, n_list).nx;
        if (n_steps == 0) continue;
        ok = warp_wait(qa_full, uc & 1, abort, 120);
        if (!ok) break;
        tc_fence_after();
        // S(G) of global step G, once S(G - 1) has been loaded
        auto issue_s = [&](int G) -> bool {
          if (G >= 1 && !warp_wait(s_read, (G - 1) & 1, abort, 126)) return false;
          if (!warp_wait(k_full + ks % kKStages, (ks / kKStages) & 1, abort, 121)) return false;
          tc_fence_after();
          issue_qk(tmem + kColS, tmem + kColQ, desc_add(dKk, (ks % kKStages) * kKTileBytes));
          mma_commit_warp(s_full);
          ++ks;
          return true;
        };
        // dP(G) (after the dQ product that read dS(G - 1) from its columns)
        auto issue_dp = [&](int G) -> bool {
          if (!warp_wait(v_full + vs % kVStages, (vs / kVStages) & 1, abort, 122)) return false;
          tc_fence_after();
          issue_qk(tmem + kColDP, tmem + kColDO, desc_add(dVk, (vs % kVStages) * kKTileBytes));
          mma_commit_warp(dp_full);
          mma_commit_warp(v_empty + vs % kVStages);
          ++vs;
          return true;
        };
        // dQ += dS(G) K(G), once dS(G) is written (the unit's first: once dQ was read out)
        auto issue_dq_step = [&](int G, bool first) -> bool {
          if (!warp_wait(ds_full, G & 1, abort, 124)) return false;
          if (first && !warp_wait(dq_free, (uc & 1) ^ 1, abort, 125)) return false;
          tc_fence_after();
          issue_dq(tmem + kColDQ, tmem + kColDP, desc_add(dKm, (kd % kKStages) * kKTileBytes), !first);
          mma_commit_warp(k_empty + kd % kKStages);
          ++kd;
          return true;
        };
        ok = issue_s(g);
        if (ok) ok = issue_dp(g);
        for (int t = 0; t < n_steps && ok; ++t) {
          if (t + 1 < n_steps) ok = issue_s(g + t + 1);
          if (ok) ok = issue_dq_step(g + t, t == 0);
          if (ok && t + 1 < n_steps) ok = issue_dp(g + t + 1);
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
    // s_full and dp_full complete once per step; a step's S needs this warp's s_read arrival
    // for the step before and its dP the dQ product of the step before (which needs this
    // warp's ds_full arrival), so a wait by parity is never more than one phase behind.
    // dq_done completes once per unit and the next completion needs this warpgroup's dq_free
    // arrival.
    const int h = warp >> 2;
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float kLog2e = 1.4426950408889634f;
    int g = 0, uc = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      const Unit x = decode<kFlat>(p, u);
      int n_list = 0;
      if constexpr (!kFlat) unit_keys(p, x.bh, x.tile, n_list);
      const Chunks ck = unit_chunks<kFlat, kExtra>(p, x, n_list);
      const int n_steps = ck.nm + ck.nx;
      // the row: a token of the tile (window / list form) or of the flat query sequence (rows
      // past Lq of the last chunk have no gradient; their Q and dO load as zeros)
      const int64_t qrow = kFlat ? 128 * static_cast<int64_t>(x.tile) + r : chunk_token(p, x.tile, x.sub, r);
      const bool row_ok = !kFlat || qrow < p.Lq;
      const int64_t row = static_cast<int64_t>(x.bh) * (kFlat ? p.Lq : p.N) + (row_ok ? qrow : 0);
      uint4* dst = reinterpret_cast<uint4*>(p.dq + row * 128) + 8 * h;
      float4* dstp = kFlat ? reinterpret_cast<float4*>(p.dq_part + x.sub * p.part_stride + row * 128) + 16 * h : nullptr;
      if (n_steps == 0) {  // no keys: no gradient
        if (row_ok) {
          if constexpr (kFlat) {
#pragma unroll
            for (int c = 0; c < 16; ++c) dstp[c] = make_float4(0.f, 0.f, 0.f, 0.f);
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        continue;
      }
      const int64_t lrow = kFlat ? static_cast<int64_t>(x.bh) * p.ld_rows + qrow : row;
      const float neg_lse2 = row_ok ? -p.lse[lrow] * kLog2e : 0.f, dd = row_ok ? p.delta[lrow] : 0.f;
      {
        // the unit's row of Q (h = 0) or dO (h = 1), 256 bytes from global memory, into TMEM as
        // packed bf16 pairs (rows past Lq of a flat chunk: zeros).  The previous unit's
        // products have all completed: this warp has seen its last scores and dP.
        const uint4* srcq = reinterpret_cast<const uint4*>((h ? p.dout : p.q) + row * 128);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t w[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v4 = row_ok ? srcq[8 * half + c] : make_uint4(0u, 0u, 0u, 0u);
            w[4 * c] = v4.x;
            w[4 * c + 1] = v4.y;
            w[4 * c + 2] = v4.z;
            w[4 * c + 3] = v4.w;
          }
          tmem_st32(tmem + (h ? kColDO : kColQ) + 32 * half + lane_off, w);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(qa_full);
      }
      for (int t = 0; t < n_steps; ++t) {
        const int ph = (g + t) & 1;
        ok = warp_wait(s_full, ph, abort, 130);
        if (!ok) break;
        tc_fence_after();
        float pf[64];
        {
          uint32_t s[64];
          tmem_ld64_wait(tmem + kColS + 64 * h + lane_off, s);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_read);  // the scores may take S(t + 1)
          // keys of this thread's 64 columns present in the chunk (a flat sequence's or the
          // extra keys' last chunk may be partial): the others get P = dS = 0
          const int nv = chunk_valid<kFlat, kExtra>(p, ck, t) - 64 * h;
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            float x0, x1;
            ffma2(x0, x1, __uint_as_float(s[c]), __uint_as_float(s[c + 1]), p.scale_log2, p.scale_log2, neg_lse2,
                  neg_lse2);
            pf[c] = ex2_approx(x0);
            pf[c + 1] = ex2_approx(x1);
            if (kFlat || kExtra) {
              if (c >= nv) pf[c] = 0.f;
              if (c + 1 >= nv) pf[c + 1] = 0.f;
            }
          }
        }
        ok = warp_wait(dp_full, ph, abort, 133);
        if (!ok) break;
        tc_fence_after();
        uint32_t dp[64];
        tmem_ld64_wait(tmem + kColDP + 64 * h + lane_off, dp);
        uint32_t w[32];
#pragma unroll
        for (int c = 0; c < 64; c += 2) {  // dS = P (dP - D), paired fp32 arithmetic
          float a0, a1, d0, d1;
          fadd2(a0, a1, __uint_as_float(dp[c]), __uint_as_float(dp[c + 1]), -dd, -dd);
          ffma2(d0, d1, a0, a1, pf[c], pf[c + 1], 0.f, 0.f);
          w[c >> 1] = pack_bf16x2(d0, d1);
        }
        tmem_st32(tmem + kColDP + 64 * h + lane_off, w);  // over this thread's own dP columns
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
      }
      if (!ok) break;
      // epilogue: dQ = scale * accumulator, channels [64h, 64h + 64) of the row
      ok = warp_wait(dq_done, uc & 1, abort, 131);
      if (!ok) break;
      tc_fence_after();
      uint32_t a[32], c2[32];
      tmem_ld32_wait(tmem + kColDQ + 64 * h + lane_off, a);
      tmem_ld32_wait(tmem + kColDQ + 64 * h + 32 + lane_off, c2);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_free);
      if constexpr (kFlat) {  // this part's fp32 share of scale * dQ
        if (row_ok) {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dstp[c] = make_float4(__uint_as_float(a[4 * c]) * p.scale, __uint_as_float(a[4 * c + 1]) * p.scale,
                                  __uint_as_float(a[4 * c + 2]) * p.scale, __uint_as_float(a[4 * c + 3]) * p.scale);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dstp[8 + c] = make_float4(__uint_as_float(c2[4 * c]) * p.scale, __uint_as_float(c2[4 * c + 1]) * p.scale,
                                      __uint_as_float(c2[4 * c + 2]) * p.scale, __uint_as_float(c2[4 * c + 3]) * p.scale);
        }
      } else {
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
          v.x = pack_bf16x2(__uint_as_float(c2[8 * c + 0]) * p.scale, __uint_as_float(c2[8 * c + 1]) * p.scale);
          v.y = pack_bf16x2(__uint_as_float(c2[8 * c + 2]) * p.scale, __uint_as_float(c2[8 * c + 3]) * p.scale);
          v.z = pack_bf16x2(__uint_as_float(c2[8 * c + 4]) * p.scale, __uint_as_float(c2[8 * c + 5]) * p.scale);
          v.w = pack_bf16x2(__uint_as_float(c2[8 * c + 6]) * p.scale, __uint_as_float(c2[8 * c + 7]) * p.scale);
          dst[4 + c] = v;
        }
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

// dQ = the sum of the parts' fp32 shares (in part order), as bf16: n8 groups of 8 channels.
__global__ void __launch_bounds__(256) dq_parts_combine(const float* __restrict__ part, int n_parts,
                                                        int64_t part_stride, int64_t n8,
                                                        __nv_bfloat16* __restrict__ dq) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
  for (int j = 0; j < n_parts; ++j) {
    const float4 x = reinterpret_cast<const float4*>(part + j * part_stride)[2 * i];
    const float4 y = reinterpret_cast<const float4*>(part + j * part_stride)[2 * i + 1];
    a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
    b.x += y.x; b.y += y.y; b.z += y.z; b.w += y.w;
  }
  uint4 v;
  v.x = pack_bf16x2(a.x, a.y);
  v.y = pack_bf16x2(a.z, a.w);
  v.z = pack_bf16x2(b.x, b.y);
  v.w = pack_bf16x2(b.z, b.w);
  reinterpret_cast<uint4*>(dq)[i] = v;
}

}  // namespace dsa
