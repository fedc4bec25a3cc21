// bf16 forward of 3D Deformable Slide Attention on CTA pairs: the window form (and the
// window form with extra text keys) run as one tcgen05 product per pair of SMs.
//
// Operator: as in the single-CTA forward (dsa_fwd_bf16.cuh): for every query token n of
// query tile i, O_n = softmax(scale * q_n K(i)^T) V(i) over exactly the keys of the window
// planned for tile i, and LSE_n = ln sum exp(...) ("MegaSlide-DiT: Memory-Centric
// Adaptation and Deformable Local Attention for Efficient Video Diffusion", abstract, 3D-DSA;
// tile-granular window form from "Fast Video Generation with Sliding Tile Attention",
// abstract).
//
// Why pairs.  The single-CTA forward reads every 256-key step's K and V (128 KB) for 128
// query rows, and its shared memory carries the fills plus the MMA operand reads (Q, K for
// the scores, V for P.V): 288 KB per step, about 2250 clocks at 128 bytes per clock against
// 2048 clocks of products.  Here a cluster of two CTAs on the two SMs of a pair holds two
// 128-row query chunks of one query tile (so one window: tiles of an even number of
// chunks) and runs every product as one M = 256 tcgen05.mma.cta_group::2: the S product
// takes the 256 keys of a step as N, 128 from each CTA's shared memory (CTA r loads chunk
// 2t + r of the step), and the P.V product takes the 128 channels as N, 64 from each CTA
// (CTA r loads channel half r of every V chunk).  Each CTA so loads 64 KB per step for its
// 128 rows instead of 128 KB, and its shared memory carries 160 KB per step instead of
// 288 KB.  (Tiles of an odd number of chunks run on the single-CTA kernel.)  Measured, the
// L2-to-SM bytes and the MMA operand reads halve as designed while the tensor pipe stays at
// the single-CTA kernel's occupancy: the softmax warps' latency chain sets the step, and the
// pair gains a few percent.
//
// Roles (per CTA, 12 warps as in the single-CTA kernel): warp 8 loads Q (its own chunk) and
// its K halves, warp 10 its V halves, warps 0-7 run the softmax of its own 128 rows; the
// even CTA's warp 9 issues every product of the pair.  The loads of both CTAs count their
// bytes on the even CTA's full barriers; the products' commits arrive on the barrier at the
// same offset in both CTAs (s_full, o_done, o_final, and the empty barriers both producers
// wait on); the softmax warps of both CTAs arrive on the even CTA's s_read, p_full and
// o_free (16 arrivals each).  The TMEM regions, the step schedule (S(t+1) issued as soon
// as every softmax warp holds S(t), then O += P(t) V(t)), the lazy rescale and the
// epilogue are those of the single-CTA kernel, so a row's arithmetic is the same.
//
// A step of one chunk (an odd chunk count) still runs the N = 256 score product: its keys
// are the even CTA's; the 128 columns from the odd CTA's stage are never read (the softmax
// of a one-chunk step takes columns 0-127 only), and the P.V product takes 128 keys.
#pragma once

#include "dsa_fwd_bf16.cuh"

namespace dsa {

namespace fwdp {
constexpr int kThreads = fwd::kThreads;
constexpr int kKStages = 3;                              // this CTA's 128 keys of a step
constexpr int kVStages = 4;                              // this CTA's 64 channels of a 128-key chunk
constexpr uint32_t kQBytes = fwd::kTileBytes;            // 128 rows x 128 channels
constexpr uint32_t kKStageBytes = fwd::kTileBytes;       // channel half h at h * 16 KB
constexpr uint32_t kVEntryBytes = fwd::kHalfBytes;       // 128 keys x 64 channels
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kQBytes;
constexpr uint32_t kOffV = kOffK + kKStages * kKStageBytes;
constexpr uint32_t kOffBar = kOffV + kVStages * kVEntryBytes;
constexpr uint32_t kOffX = kOffBar + 256;
constexpr uint32_t kSmemUsed = kOffX + 2 * 2 * 128 * 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // room for the 1024-byte alignment of the base
static_assert(kSmemBytes <= 227 * 1024, "shared memory layout too large");
constexpr uint32_t kIdescS = idesc_bf16_f32(256, 256, 0, 0);   // Q, K both K-major (smem)
constexpr uint32_t kIdescPV = idesc_bf16_f32(256, 128, 0, 1);  // P from TMEM, V MN-major (smem)
constexpr uint16_t kBoth = 3;                                  // commit to both CTAs of the pair

// The cluster's it-th pair unit (p.n_units / 2 of them: the launcher keeps p.n_units within
// int32): units run (batch * head)-major, then query tile, then the tile's pairs of chunks
// (2j, 2j + 1), strided over the clusters, so neighbouring clusters take neighbouring tiles
// of one head, whose windows overlap in L2; CTA `rank` takes chunk 2j + rank.
__device__ __forceinline__ bool next_pair(const FwdBf16Params& p, int it, uint32_t rank, fwd::Unit& x) {
  const int u = static_cast<int>(cluster_id_x() + static_cast<uint32_t>(it) * cluster_count_x());
  if (u >= p.n_units / 2) return false;
  const int half = p.S / 2, per_bh = half * p.n_tiles;
  x.bh = u / per_bh;
  const int rem = u % per_bh;
  x.tile = rem / half;
  x.sub = 2 * (rem % half) + static_cast<int>(rank);
  return true;
}

// S = Q K^T over the 128 channels for 256 keys: 8 k-steps of 16 channels.  Q (this CTA's
// rows) and a K stage (this CTA's 128 keys) both hold channel half h at h * 16 KB.
__device__ __forceinline__ void issue_scores_pair(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc) {
  fwd::opaque(q_desc);
  fwd::opaque(k_desc);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t o = (kk >> 2) * fwd::kHalfBytes + (kk & 3) * 32;
    mma_ss_pair_warp(d_tmem, fwd::desc_add(q_desc, o), fwd::desc_add(k_desc, o), kIdescS, kk > 0);
  }
}

// O (+)= P V over one 128-key chunk: P from TMEM (8 columns of packed bf16 per 16 keys), V
// this CTA's 64 channels, MN-major, 16 keys = 2048 bytes per k-step.
__device__ __forceinline__ void issue_pv_pair(uint32_t d_tmem, uint32_t p_tmem, uint64_t v_desc, bool accumulate) {
  fwd::opaque(v_desc);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts_pair_warp(d_tmem, p_tmem + kk * 8, fwd::desc_add(v_desc, kk * 2048), kIdescPV, accumulate || kk > 0);
}

__device__ __forceinline__ bool warp_wait_cl(uint64_t* bar, uint32_t parity, volatile int* abort, int site) {
  return __all_sync(0xffffffffu, mbar_wait_cluster(bar, parity, abort, site));
}

// Waits for a barrier phase whatever the abort flag says, for at most 100 ms: used once at
// the end, so that no product is still writing the pair's TMEM when it is released.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_cluster(bar, parity))
    if (globaltimer_ns() - t0 > 100000000ull) break;
}
}  // namespace fwdp

// The window form (p.row_ptr null) with p.S even; kExtra: p.Lx extra (text) keys after
// every unit's window (maps tmKx, tmVx).
template <bool kExtra>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(fwdp::kThreads, 1)
    fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKx,
                    const __grid_constant__ CUtensorMap tmVx, FwdBf16Params p) {
  using namespace fwdp;
  using fwd::col_p;
  using fwd::col_s;
  using fwd::desc_add;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  if (pad + kSmemUsed > kSmemBytes) {  // the same in both CTAs: both leave before any cluster step
    if (threadIdx.x == 0) device_report(DSA_DEV_BOUNDS, 60);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;            // [kKStages]
  uint64_t* k_empty = k_full + kKStages;  // [kKStages]
  uint64_t* v_full = k_empty + kKStages;  // [kVStages]
  uint64_t* v_empty = v_full + kVStages;  // [kVStages]
  uint64_t* s_full = v_empty + kVStages;  // [2]
  uint64_t* p_full = s_full + 2;          // [2] (16 warps)
  uint64_t* s_read = s_full + 4;          // [2] (16 warps)
  uint64_t* o_done = s_full + 6;
  uint64_t* o_free = s_full + 7;          // (16 warps)
  uint64_t* o_final = s_full + 8;
  uint64_t* drain = s_full + 9;           // every product issued has completed (even CTA)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 10);
  volatile int* abort = reinterpret_cast<volatile int*>(s_full + 11);
  static_assert(2 + 2 * kKStages + 2 * kVStages + 12 <= 256 / 8, "barriers must fit their 256 bytes");
  float* xbuf = reinterpret_cast<float*>(smem + kOffX);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool lead = rank == 0;

  if (tid == 0) {
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    if (kExtra && p.Lx > 0) {
      tma_prefetch_map(&tmKx);
      tma_prefetch_map(&tmVx);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
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
      mbar_init(p_full + e, 16);
      mbar_init(s_read + e, 16);
    }
    mbar_init(o_done, 1);
    mbar_init(o_free, 16);
    mbar_init(o_final, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == fwd::kMmaWarp) {
    tmem_alloc_pair(tmem_slot, fwd::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before either arrives on the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // (the even CTA's barriers are addressed as mapa_shared(..., 0) where they are used)

  if (warp >= fwd::kProducerWarp) {
    setmaxnreg_dec<fwd::kRegsAux>();
    if (warp == fwd::kProducerWarp || warp == fwd::kVProducerWarp) {
      // ------------------------------------------------------------------ TMA producers (both CTAs)
      if (lane == 0) {
        const bool is_k = warp == fwd::kProducerWarp;
        int ld = 0, uc = 0;
        bool ok = true;
        fwd::Unit x;
        for (int it = 0; ok && next_pair(p, it, rank, x); ++it) {
          int n_list = 0;
          const int32_t* kv = fwd::unit_keys(p, x.bh, x.tile, n_list);
          const fwd::Chunks ck = fwd::unit_chunks<false, kExtra>(p, x, n_list);
          const int n_chunks = ck.nm + ck.nx, n_steps = (n_chunks + 1) / 2;
          if (n_chunks == 0) continue;
          if (is_k) {
            ok = mbar_wait(q_empty, (uc & 1) ^ 1, abort, 61);
            if (!ok) break;
            if (lead) mbar_arrive_expect_tx(q_full, 2 * kQBytes);
            const int qt = x.tile / (p.G1 * p.G2), qh = (x.tile / p.G2) % p.G1, qw = x.tile % p.G2;
            const int tq0 = qt * p.tt + x.sub * p.tcs;
            const uint32_t qbar = mapa_shared(smem_u32(q_full), 0);
            tma_load_5d_pair(smem + kOffQ, &tmQ, qbar, 0, qw * p.tw, qh * p.th, tq0, x.bh);
            tma_load_5d_pair(smem + kOffQ + fwd::kHalfBytes, &tmQ, qbar, 64, qw * p.tw, qh * p.th, tq0, x.bh);
          }
          ++uc;
          // K: one stage per step, this CTA's chunk 2j + rank (both channel halves);
          // V: one entry per chunk, this CTA's channel half
          const int n_loads = is_k ? n_steps : n_chunks;
          const int n_st = is_k ? kKStages : kVStages;
          for (int j = 0; j < n_loads && ok; ++j, ++ld) {
            const int st = ld % n_st;
            ok = mbar_wait((is_k ? k_empty : v_empty) + st, ((ld / n_st) & 1) ^ 1, abort, is_k ? 62 : 63);
            if (!ok) break;
            const bool two = 2 * j + 1 < n_chunks;  // a K step of two chunks
            if (lead)
              mbar_arrive_expect_tx((is_k ? k_full : v_full) + st,
                                    is_k ? (two ? 2 : 1) * kKStageBytes : 2 * kVEntryBytes);
            if (is_k && !two && !lead) continue;  // a one-chunk step's keys are the even CTA's
            const int jc = is_k ? 2 * j + static_cast<int>(rank) : j;  // the unit's chunk
            const uint32_t bar = mapa_shared(smem_u32((is_k ? k_full : v_full) + st), 0);
            uint8_t* dst = is_k ? smem + kOffK + st * kKStageBytes : smem + kOffV + st * kVEntryBytes;
            if (kExtra && jc >= ck.nm) {  // extra keys (rows past Lx load as zeros and are masked)
              const int row = 128 * (jc - ck.nm);
              if (is_k) {
                tma_load_3d_pair(dst, &tmKx, bar, 0, row, x.bh);
                tma_load_3d_pair(dst + fwd::kHalfBytes, &tmKx, bar, 64, row, x.bh);
              } else {
                tma_load_3d_pair(dst, &tmVx, bar, 64 * static_cast<int>(rank), row, x.bh);
              }
              continue;
            }
            const int c = ck.c0 + jc;
            const int kt = min(max(kv[c / p.S], 0), p.n_tiles - 1), ks = c % p.S;
            const int t0 = (kt / (p.G1 * p.G2)) * p.tt + ks * p.tcs;
            const int h0 = ((kt / p.G2) % p.G1) * p.th, w0 = (kt % p.G2) * p.tw;
            if (is_k) {
              tma_load_5d_pair(dst, &tmK, bar, 0, w0, h0, t0, x.bh);
              tma_load_5d_pair(dst + fwd::kHalfBytes, &tmK, bar, 64, w0, h0, t0, x.bh);
            } else {
              tma_load_5d_pair(dst, &tmV, bar, 64 * static_cast<int>(rank), w0, h0, t0, x.bh);
            }
          }
        }
      }
    } else if (warp == fwd::kMmaWarp && lead) {
      // ------------------------------------------------------------------ MMA issuer of the pair
      const uint64_t dQ = smem_desc_sw128(sbase + kOffQ, 16, 1024);
      const uint64_t dK = smem_desc_sw128(sbase + kOffK, 16, 1024);             // stage 0, K-major
      const uint64_t dV = smem_desc_sw128(sbase + kOffV, kVEntryBytes, 1024);   // entry 0, MN-major
      int ks = 0, vs = 0, uc = 0, g = 0, pc0 = 0, pc1 = 0;
      bool ok = true;
      fwd::Unit xm;
      for (int it = 0; ok && next_pair(p, it, rank, xm); ++it) {
        int n_list = 0;
        fwd::unit_keys(p, xm.bh, xm.tile, n_list);
        const fwd::Chunks ck = fwd::unit_chunks<false, kExtra>(p, xm, n_list);
        const int n_chunks = ck.nm + ck.nx, n_steps = (n_chunks + 1) / 2;
        if (n_chunks == 0) continue;
        ok = warp_wait_cl(q_full, uc & 1, abort, 64);
        if (ok) ok = warp_wait_cl(k_full + ks % kKStages, (ks / kKStages) & 1, abort, 65);
        if (!ok) break;
        tc_fence_after();
        issue_scores_pair(tmem + col_s(g & 1), dQ, desc_add(dK, (ks % kKStages) * kKStageBytes));
        mma_commit_pair_warp(s_full + (g & 1), kBoth);
        mma_commit_pair_warp(k_empty + ks % kKStages, kBoth);
        ++ks;
        if (n_steps == 1) mma_commit_pair_warp(q_empty, kBoth);
        for (int t = 0; t < n_steps && ok; ++t) {
          const int e = (g + t) & 1;
          const int ph = (e == 0 ? pc0++ : pc1++) & 1;
          ok = warp_wait_cl(s_read + e, ph, abort, 66);
          if (!ok) break;
          if (t + 1 < n_steps) {
            ok = warp_wait_cl(k_full + ks % kKStages, (ks / kKStages) & 1, abort, 67);
            if (!ok) break;
            tc_fence_after();
            issue_scores_pair(tmem + col_s(e ^ 1), dQ, desc_add(dK, (ks % kKStages) * kKStageBytes));
            mma_commit_pair_warp(s_full + (e ^ 1), kBoth);
            mma_commit_pair_warp(k_empty + ks % kKStages, kBoth);
            ++ks;
            if (t + 2 == n_steps) mma_commit_pair_warp(q_empty, kBoth);
          }
          ok = warp_wait_cl(p_full + e, ph, abort, 68);
          if (ok && t == 0) ok = warp_wait_cl(o_free, (uc & 1) ^ 1, abort, 69);
          const int nb = 2 * t + 1 < n_chunks ? 2 : 1;
          for (int b = 0; b < nb && ok; ++b, ++vs) {
            ok = warp_wait_cl(v_full + vs % kVStages, (vs / kVStages) & 1, abort, 70);
            if (!ok) break;
            tc_fence_after();
            issue_pv_pair(tmem + fwd::kColO, tmem + col_p(e) + 64 * b, desc_add(dV, (vs % kVStages) * kVEntryBytes),
                          t > 0 || b > 0);
            mma_commit_pair_warp(v_empty + vs % kVStages, kBoth);
          }
          if (!ok) break;
          mma_commit_pair_warp(o_done, kBoth);
        }
        if (!ok) break;
        mma_commit_pair_warp(o_final, kBoth);
        g += n_steps;
        ++uc;
      }
      // every product issued has completed before the pair's TMEM is released
      mma_commit_pair_warp(drain, 1);
      drain_wait(drain, 0);
    }
  } else {
    setmaxnreg_inc<fwd::kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax (both CTAs, own rows)
    // As in the single-CTA kernel; the arrivals that release the products go to the even
    // CTA's barriers.  A softmax warp never leaves the unit loop early, even after a failed
    // wait, so its partner warp finds it at every named barrier.
    const int i = warp >> 2;
    const int r = tid & 127;
    const int bar_id = 1 + (warp & 3);
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + fwd::kColO + 64 * i + lane_off;
    int sc0 = 0, sc1 = 0, g = 0, uc = 0, xe = 0;
    bool ok = true;
    fwd::Unit x;
    for (int it = 0; next_pair(p, it, rank, x); ++it) {
      int n_list = 0;
      fwd::unit_keys(p, x.bh, x.tile, n_list);
      const fwd::Chunks ck = fwd::unit_chunks<false, kExtra>(p, x, n_list);
      const int n_chunks = ck.nm + ck.nx, n_steps = (n_chunks + 1) / 2;
      if (n_chunks == 0) {  // no keys: O = 0 and LSE = -inf (as the single-CTA kernel)
        const int64_t tok = fwd::chunk_token(p, x.tile, x.sub, r);
        uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(x.bh) * p.N + tok) * 128) + 8 * i;
#pragma unroll
        for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
        if (i == 0) p.lse[static_cast<int64_t>(x.bh) * p.N + tok] = -INFINITY;
        continue;
      }
      float m_used = -INFINITY, l = 0.f;
      for (int t = 0; t < n_steps; ++t) {
        const int e = (g + t) & 1;
        if (ok) ok = fwd::warp_wait(s_full + e, (e == 0 ? sc0++ : sc1++) & 1, abort, 72);
        if (ok) tc_fence_after();
        float alpha;
        bool need;
        const bool full = 2 * t + 1 < n_chunks;
        const int nvalid = full ? fwd::chunk_valid<false, kExtra>(p, ck, 2 * t + i)
                                : min(max(fwd::chunk_valid<false, kExtra>(p, ck, 2 * t) - 64 * i, 0), 64);
        if (full)
          need = fwd::softmax_step<128, true>(ok, tmem + col_s(e) + 128 * i + lane_off,
                                              tmem + col_p(e) + 64 * i + lane_off, mapa_shared(smem_u32(s_read + e), 0),
                                              p.scale_log2,
                                              m_used, l, alpha, xbuf, xe, i, r, bar_id, nvalid);
        else
          need = fwd::softmax_step<64, true>(ok, tmem + col_s(e) + 64 * i + lane_off,
                                             tmem + col_p(e) + 32 * i + lane_off, mapa_shared(smem_u32(s_read + e), 0),
                                             p.scale_log2,
                                             m_used, l, alpha, xbuf, xe, i, r, bar_id, nvalid);
        if (ok && t > 0 && __any_sync(0xffffffffu, need)) {
          ok = fwd::warp_wait(o_done, (g + t - 1) & 1, abort, 73);
          if (ok) {
            tc_fence_after();
            fwd::rescale_o(tO, 2, alpha);
          }
        }
        if (ok) {
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(p_full + e), 0));
        }
      }
      // epilogue: O / l as bf16 (channels [64i, 64i + 64)), LSE = (m + log2 l) ln 2
      if (ok) ok = fwd::warp_wait(o_final, uc & 1, abort, 74);
      const float l_all = l + fwd::pair_exchange(xbuf, xe, i, r, bar_id, l);
      if (ok) {
        tc_fence_after();
        const int64_t tok = fwd::chunk_token(p, x.tile, x.sub, r);
        fwd::store_o(tO, 2, 1.f / l_all,
                     reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(x.bh) * p.N + tok) * 128) + 8 * i);
        if (i == 0)
          p.lse[static_cast<int64_t>(x.bh) * p.N + tok] = (m_used + __log2f(l_all)) * 0.69314718055994531f;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(o_free), 0));
      }
      g += n_steps;
      ++uc;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort && tid == 0) {
    // after a failed wait, give loads already issued time to land before the CTA leaves
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {
    }
  }
  __syncthreads();
  cluster_sync();  // no CTA leaves while the other may still arrive on its barriers or run products into its TMEM
  if (warp == fwd::kMmaWarp) {
    __syncwarp();
    tmem_dealloc_pair(tmem, fwd::kTmemCols);
  }
}

}  // namespace dsa
