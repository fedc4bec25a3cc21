// bf16 forward of 3D Deformable Slide Attention on the 5th-generation tensor cores.
//
// Operator: for every query token n of query tile i, O_n = softmax(scale * q_n K(i)^T) V(i)
// over exactly the keys of the window planned for tile i, and LSE_n = ln sum exp(...)
// ("MegaSlide-DiT: Memory-Centric Adaptation and Deformable Local Attention for Efficient
// Video Diffusion", abstract, 3D-DSA; tile-granular window form from "Fast Video
// Generation with Sliding Tile Attention", abstract).
//
// Persistent, warp-specialised kernel, one CTA per SM.  A work unit takes 128-row query
// chunks of one query tile of one (batch, head): two chunks ("slots") that share every
// K/V chunk of the tile's window, or, for the last chunk of a tile with an odd number of
// chunks, one chunk alone.  Roles:
//   warp 8      TMA producer: Q of the unit, then K and V chunks through a 5-stage ring;
//   warp 9      MMA issuer (a converged warp; one elected lane issues):
//                 two slots: S_i = Q_i K^T into score buffer i, O_i += P_i V with P_i read
//                 from TMEM (the scores' own columns), order S0 S1 | PV0 S0' PV1 S1' | ...;
//                 one slot:  S(j) into buffer j % 2, so S(j+1) is computed while the
//                 softmax of S(j) runs; O_0 += P(j) V;
//   warps 0-3   softmax of slot 0 (and of single-slot units), warps 4-7 softmax of slot 1:
//               one thread per query row reads its S row from TMEM, keeps a running max m
//               and sum l (base 2), writes P = exp2(S * scale * log2 e - m) as bf16 back
//               into TMEM, and at the end of a unit normalises its O row and writes O, LSE.
// The running max is only moved when it grows by more than 8 (a factor 256): P stays
// <= 256, which bf16 and the fp32 accumulators hold exactly as well, and the O rescale
// (a TMEM read-modify-write of the row) happens a few times per row instead of per chunk.
// The result is exact: O = sum P V / sum P with the same reference max in both sums.
//
// Units are ordered (batch*head, pass, tile): pass p takes chunks 2p and 2p+1 of every
// tile, so consecutive units work on neighbouring tiles of one head (their windows
// overlap in L2), and the persistent CTAs' strided walk mixes paired and single units.
//
// TMEM (512 columns): score buffers 0 [0,128) and 1 [128,256), O0 [256,384), O1 [384,512).
// Shared memory: Q0, Q1 (32 KB each), 5 K/V stages (32 KB each), barriers.
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
  int n_pass;               // units per tile, ceil(S / 2)
  int n_units;              // B*heads * n_pass * n_tiles
  int G1, G2;               // Gh, Gw
  int tt, th, tw, tcs;      // tile shape; t-extent of one 128-token chunk
  int T, H, W, N;
  float scale_log2;         // scale * log2(e)
};

namespace fwd {
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kStages = 5;
constexpr uint32_t kTileBytes = 128 * 128 * 2;
constexpr uint32_t kHalfBytes = kTileBytes / 2;
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKV = 2 * kTileBytes;
constexpr uint32_t kOffBar = kOffKV + kStages * kTileBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);   // Q, K both K-major (smem)
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 0, 1);  // P from TMEM, V MN-major (smem)
constexpr float kRescaleThreshold = 8.0f;                      // log2 units
constexpr int kPolyEvery = 4;  // one 16-column group in 4 takes 2^x from the FMA-pipe polynomial

struct Unit {
  int bh, tile, sub0;
  bool two;  // two slots (chunks sub0, sub0 + 1) or one
};

__device__ __forceinline__ Unit decode(const FwdBf16Params& p, int u) {
  Unit x;
  const int per_bh = p.n_pass * p.n_tiles;
  x.bh = u / per_bh;
  const int rem = u % per_bh;
  x.sub0 = 2 * (rem / p.n_tiles);
  x.tile = rem % p.n_tiles;
  x.two = x.sub0 + 1 < p.S;
  return x;
}

// Shared-memory descriptors are built once; a byte offset is added in 16-byte units to
// the address field (all addresses stay below 256 KB, so the 14-bit field cannot carry).
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

// S = Q K^T over the 128 channels: 8 k-steps of 16 within the two 64-channel halves.
__device__ __forceinline__ void issue_scores(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
    mma_ss_warp(d_tmem, desc_add(q_desc, off), desc_add(k_desc, off), kIdescS, kk > 0);
  }
}

// O (+)= P V over 128 keys: P from TMEM (8 columns of packed bf16 per 16 keys), V
// MN-major with 16 keys = two 8-row groups = 2048 bytes per k-step.
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint64_t v_desc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts_warp(d_tmem, p_tmem + kk * 8, desc_add(v_desc, kk * 2048), kIdescPV, accumulate || kk > 0);
}

// Waits (whole warp) for `count` consecutive ring entries from `base` to be full.
__device__ __forceinline__ bool wait_entries(uint64_t* full, int base, int count, volatile int* abort, int site) {
  bool ok = true;
  for (int t = 0; t < count && ok; ++t) ok = mbar_wait(full + (base + t) % kStages, ((base + t) / kStages) & 1, abort, site);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void release_entries(uint64_t* empty, int base, int count) {
  for (int t = 0; t < count; ++t) mma_commit_warp(empty + (base + t) % kStages);
}

// Barrier wait by a whole warp, with a warp-uniform result.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int site) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, site));
}
}  // namespace fwd

__global__ void __launch_bounds__(fwd::kThreads, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, FwdBf16Params p) {
  using namespace fwd;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;              // [kStages]
  uint64_t* kv_empty = bars + 2 + kStages;   // [kStages]
  // scores ready / P ready, indexed 0: buffer 0, 1: buffer 1 of a two-slot unit, 2: buffer 1
  // of a single-slot unit (warpgroup 0's odd chunks) -- a separate barrier, so that the
  // phases warpgroup 1 waits for are its own chunks only
  uint64_t* s_full = bars + 2 + 2 * kStages; // [3]
  uint64_t* p_full = s_full + 3;             // [3]
  uint64_t* o_done = s_full + 6;             // [2]
  uint64_t* o_free = s_full + 8;             // [2]
  uint64_t* o_final = s_full + 10;           // [2] every product of a unit into O_i done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 12);
  volatile int* abort = reinterpret_cast<volatile int*>(s_full + 13);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_chunks = p.Wt * p.S;

  if (tid == 0) {
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 4);  // one arrival per softmax warp
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(o_done + i, 1);
      mbar_init(o_free + i, 4);
      mbar_init(o_final + i, 1);
    }
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

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int kv_load = 0, uc = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++uc) {
        const Unit x = decode(p, u);
        const int qt = x.tile / (p.G1 * p.G2), qh = (x.tile / p.G2) % p.G1, qw = x.tile % p.G2;
        ok = mbar_wait(q_empty, (uc & 1) ^ 1, abort, 20);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, (x.two ? 2u : 1u) * kTileBytes);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          if (i == 1 && !x.two) break;
          const int t0 = qt * p.tt + (x.sub0 + i) * p.tcs;
          uint8_t* dst = smem + kOffQ + i * kTileBytes;
          tma_load_5d(dst, &tmQ, q_full, 0, qw * p.tw, qh * p.th, t0, x.bh);
          tma_load_5d(dst + kHalfBytes, &tmQ, q_full, 64, qw * p.tw, qh * p.th, t0, x.bh);
        }
        const int32_t* kv = p.kv_tiles + static_cast<int64_t>(x.tile) * p.Wt;
        for (int j = 0; j < n_chunks && ok; ++j) {
          const int kt = kv[j / p.S], ks = j % p.S;
          const int t0 = (kt / (p.G1 * p.G2)) * p.tt + ks * p.tcs;
          const int h0 = ((kt / p.G2) % p.G1) * p.th, w0 = (kt % p.G2) * p.tw;
          for (int which = 0; which < 2; ++which, ++kv_load) {
            const int st = kv_load % kStages;
            ok = mbar_wait(kv_empty + st, ((kv_load / kStages) & 1) ^ 1, abort, 21);
            if (!ok) break;
            mbar_arrive_expect_tx(kv_full + st, kTileBytes);
            uint8_t* dst = smem + kOffKV + st * kTileBytes;
            const CUtensorMap* map = which == 0 ? &tmK : &tmV;
            tma_load_5d(dst, map, kv_full + st, 0, w0, h0, t0, x.bh);
            tma_load_5d(dst + kHalfBytes, map, kv_full + st, 64, w0, h0, t0, x.bh);
          }
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer (whole warp)
    const uint64_t dQ0 = smem_desc_sw128(sbase + kOffQ, 16, 1024);
    const uint64_t dQ1 = desc_add(dQ0, kTileBytes);
    const uint64_t dK = smem_desc_sw128(sbase + kOffKV, 16, 1024);          // stage 0, K-major
    const uint64_t dV = smem_desc_sw128(sbase + kOffKV, kHalfBytes, 1024);  // stage 0, MN-major
    int kv_use = 0, uc = 0;
    int pb0 = 0, pb1 = 0, pb2 = 0;  // P consumed per ready-barrier
    int us0 = 0, us1 = 0;  // units that used O0 / O1
    bool ok = true;
    for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++uc) {
      const Unit x = decode(p, u);
      ok = warp_wait(q_full, uc & 1, abort, 30);
      if (!ok) break;
      // K(j) is ring entry base + 2j, V(j) is base + 2j + 1
      const int base = kv_use;
      kv_use += 2 * n_chunks;
      if (x.two) {
        ok = wait_entries(kv_full, base, 1, abort, 31);
        if (!ok) break;
        tc_fence_after();
        issue_scores(tmem, dQ0, desc_add(dK, (base % kStages) * kTileBytes));
        mma_commit_warp(s_full);
        issue_scores(tmem + 128, dQ1, desc_add(dK, (base % kStages) * kTileBytes));
        mma_commit_warp(s_full + 1);
        release_entries(kv_empty, base, 1);
        if (n_chunks == 1) mma_commit_warp(q_empty);
        for (int j = 0; j < n_chunks && ok; ++j) {
          const int v_idx = base + 2 * j + 1, k_idx = base + 2 * j + 2;
          const bool more = j + 1 < n_chunks;
          ok = wait_entries(kv_full, v_idx, 1, abort, 32);
          if (!ok) break;
          // slot 0: O0 += P0 V, then S0 = Q0 K'
          ok = warp_wait(p_full, pb0++ & 1, abort, 33);
          if (ok && j == 0) ok = warp_wait(o_free, (us0 & 1) ^ 1, abort, 34);
          if (!ok) break;
          tc_fence_after();
          issue_pv(tmem + 256, tmem, desc_add(dV, (v_idx % kStages) * kTileBytes), j > 0);
          mma_commit_warp(o_done);
          if (more) {
            ok = wait_entries(kv_full, k_idx, 1, abort, 35);
            if (!ok) break;
            tc_fence_after();
            issue_scores(tmem, dQ0, desc_add(dK, (k_idx % kStages) * kTileBytes));
            mma_commit_warp(s_full);
          }
          // slot 1
          ok = warp_wait(p_full + 1, pb1++ & 1, abort, 33);
          if (ok && j == 0) ok = warp_wait(o_free + 1, (us1 & 1) ^ 1, abort, 34);
          if (!ok) break;
          tc_fence_after();
          issue_pv(tmem + 384, tmem + 128, desc_add(dV, (v_idx % kStages) * kTileBytes), j > 0);
          mma_commit_warp(o_done + 1);
          if (more) {
            issue_scores(tmem + 128, dQ1, desc_add(dK, (k_idx % kStages) * kTileBytes));
            mma_commit_warp(s_full + 1);
            release_entries(kv_empty, k_idx, 1);
          }
          release_entries(kv_empty, v_idx, 1);
          if (j + 2 == n_chunks) mma_commit_warp(q_empty);  // every score of this unit issued
        }
        if (!ok) break;
        mma_commit_warp(o_final);
        mma_commit_warp(o_final + 1);
        ++us0;
        ++us1;
      } else {
        // one slot: scores alternate between the two buffers, O0 accumulates
        const int pre = n_chunks < 2 ? n_chunks : 2;
        for (int j = 0; j < pre && ok; ++j) {
          ok = wait_entries(kv_full, base + 2 * j, 1, abort, 31);
          if (!ok) break;
          tc_fence_after();
          const int b = j;  // buffer of chunk j
          issue_scores(tmem + b * 128, dQ0, desc_add(dK, ((base + 2 * j) % kStages) * kTileBytes));
          mma_commit_warp(s_full + 2 * b);
          release_entries(kv_empty, base + 2 * j, 1);
        }
        if (ok && n_chunks <= 2) mma_commit_warp(q_empty);
        for (int j = 0; j < n_chunks && ok; ++j) {
          const int b = j & 1;
          const int v_idx = base + 2 * j + 1, k_idx = base + 2 * j + 4;
          ok = wait_entries(kv_full, v_idx, 1, abort, 32);
          if (ok) ok = warp_wait(p_full + 2 * b, (b == 0 ? pb0++ : pb2++) & 1, abort, 33);
          if (ok && j == 0) ok = warp_wait(o_free, (us0 & 1) ^ 1, abort, 34);
          if (!ok) break;
          tc_fence_after();
          issue_pv(tmem + 256, tmem + b * 128, desc_add(dV, (v_idx % kStages) * kTileBytes), j > 0);
          mma_commit_warp(o_done);
          if (j + 2 < n_chunks) {
            // S(j+2) reuses buffer b; in issue order it follows the product that reads P(j)
            ok = wait_entries(kv_full, k_idx, 1, abort, 35);
            if (!ok) break;
            tc_fence_after();
            issue_scores(tmem + b * 128, dQ0, desc_add(dK, (k_idx % kStages) * kTileBytes));
            mma_commit_warp(s_full + 2 * b);
            release_entries(kv_empty, k_idx, 1);
          }
          release_entries(kv_empty, v_idx, 1);
          if (j + 3 == n_chunks) mma_commit_warp(q_empty);
        }
        if (!ok) break;
        mma_commit_warp(o_final);
        ++us0;
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax (slot i)
    const int i = warp >> 2;
    const int r = tid & 127;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + 256 + i * 128 + lane_off;
    int sc0 = 0, sc1 = 0, sc2 = 0;  // phases waited per ready-barrier
    int pv_base = 0, uf = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      const Unit x = decode(p, u);
      if (!x.two && i == 1) continue;
      const int sub = x.sub0 + i;
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < n_chunks; ++j) {
        const int b = x.two ? i : (j & 1);                   // score buffer of this chunk
        const int rb = x.two ? i : 2 * (j & 1);              // its ready-barrier index
        const uint32_t tS = tmem + b * 128 + lane_off;
        ok = mbar_wait(s_full + rb, (rb == 0 ? sc0++ : (rb == 1 ? sc1++ : sc2++)) & 1, abort, 40);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        uint32_t s[128];
        tmem_ld128_wait(tS, s);
        // row max: 8 independent chains of 3-input max
        float mxs[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          mxs[e] = __uint_as_float(s[e]);
#pragma unroll
          for (int c = 8 + e; c < 128; c += 16)
            mxs[e] = max3f(mxs[e], __uint_as_float(s[c]), __uint_as_float(s[c + 8]));
        }
        const float mx = max3f(max3f(mxs[0], mxs[1], mxs[2]), max3f(mxs[3], mxs[4], mxs[5]), fmaxf(mxs[6], mxs[7]));
        const float m_new = fmaxf(m_used, mx * p.scale_log2);
        const bool need = m_new > m_used + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx(m_used - m_new);
          m_used = m_new;
        }
        l *= alpha;
        const float neg_m = -m_used;
        // P = 2^(s * scale * log2 e - m): paired fp32 arithmetic; one column group in
        // kPolyEvery goes to the FMA-pipe polynomial to unload the MUFU unit
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float x0, x1, p0, p1;
            ffma2(x0, x1, __uint_as_float(s[16 * g + 2 * e]), __uint_as_float(s[16 * g + 2 * e + 1]), p.scale_log2,
                  p.scale_log2, neg_m, neg_m);
            if (kPolyEvery > 0 && (g % kPolyEvery) == kPolyEvery - 1) {
              exp2_poly2(x0, x1, p0, p1);
            } else {
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            fadd2(sa[e & 3], sb[e & 3], sa[e & 3], sb[e & 3], p0, p1);
            pk[e] = pack_bf16x2(p0, p1);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) s[8 * g + e] = pk[e];  // packed P of columns 16g..16g+15
        }
        l += ((sa[0] + sb[0]) + (sa[1] + sb[1])) + ((sa[2] + sb[2]) + (sa[3] + sb[3]));
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = s[16 * g + e];
          tmem_st16(tS + 16 * g, w);
        }
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // O_i holds sum P V up to chunk j-1 with the old reference max: rescale it
          ok = mbar_wait(o_done + i, (pv_base + j - 1) & 1, abort, 41);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int g = 0; g < 4; ++g) {
            uint32_t o[32];
            tmem_ld32_wait(tO + 32 * g, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + 32 * g, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + rb);
      }
      if (!ok) break;
      // epilogue: O / l as bf16, LSE = (m + log2 l) ln 2.  o_final completes once per unit
      // (after the unit's last product into O_i), so its parity is never ambiguous.
      ok = mbar_wait(o_final + i, uf & 1, abort, 42);
      ++uf;
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      pv_base += n_chunks;
      const int qt = x.tile / (p.G1 * p.G2), qh = (x.tile / p.G2) % p.G1, qw = x.tile % p.G2;
      const int t0 = qt * p.tt + sub * p.tcs;
      const int lw = r % p.tw, lh = (r / p.tw) % p.th, lt = r / (p.tw * p.th);
      const int64_t tok = (static_cast<int64_t>(t0 + lt) * p.H + (qh * p.th + lh)) * p.W + (qw * p.tw + lw);
      const float inv = 1.f / l;
      uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(x.bh) * p.N + tok) * 128);
#pragma unroll 1
      for (int g = 0; g < 4; ++g) {
        uint32_t o[32];
        tmem_ld32_wait(tO + 32 * g, o);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv);
          v.y = pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv);
          v.z = pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv);
          v.w = pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv);
          dst[4 * g + c] = v;
        }
      }
      p.lse[static_cast<int64_t>(x.bh) * p.N + tok] = (m_used + __log2f(l)) * 0.69314718055994531f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free + i);
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
