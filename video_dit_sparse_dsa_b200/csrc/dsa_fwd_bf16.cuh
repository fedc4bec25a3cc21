// bf16 forward of 3D Deformable Slide Attention on the 5th-generation tensor cores.
//
// Operator: for every query token n of query tile i, O_n = softmax(scale * q_n K(i)^T) V(i)
// over exactly the keys of the window planned for tile i, and LSE_n = ln sum exp(...)
// ("MegaSlide-DiT: Memory-Centric Adaptation and Deformable Local Attention for Efficient
// Video Diffusion", abstract, 3D-DSA; tile-granular window form from "Fast Video
// Generation with Sliding Tile Attention", abstract).
//
// Persistent, warp-specialised kernel, one CTA per SM.  A work unit is one 128-row query
// chunk of one query tile of one (batch, head); its window's keys are taken 256 at a time
// (a "step": two 128-token K/V chunks; an odd last chunk makes a 128-key half step), so
// the score product is one M=128, N=256 tcgen05.mma per 16 channels, the shape that keeps
// the tensor pipe full (an N=128 product costs nearly as many cycles as an N=256 one).
// Roles:
//   warp 8      TMA producer of Q (once per unit) and K: per step one 64 KB stage (two
//               chunks) of a 2-stage ring, so K of step t+1 is loaded while step t runs;
//   warp 10     TMA producer of V: one 32 KB chunk per entry of a 2-entry ring, each
//               entry released as soon as the half of the product that reads it is done;
//   warp 9      MMA issuer (a converged warp; one elected lane issues), per step t:
//               S(t+1) = Q K(t+1)^T as soon as the softmax warps have loaded the scores
//               of step t into registers, then O += P(t) V(t) with P read from TMEM, so
//               the next scores are computed while the softmax of step t runs;
//   warp 11     idle (the four warps 8-11 form the third warpgroup, whose registers the
//               softmax warpgroups take over through setmaxnreg);
//   warps 0-7   softmax: warpgroup i (warps 4i..4i+3) takes keys [128i, 128i+128) of
//               every step (half steps: [64i, 64i+64)), one thread per query row.  The
//               two threads of a row (same lane of warps w and w+4) agree on the step's
//               row max through shared memory (a 64-thread named barrier per warp pair),
//               write P = exp2(S * scale * log2 e - m) as bf16 into TMEM, keep partial
//               row sums, and at the end add them and each write half of the channels of
//               O / l, and LSE.
// The running max is only moved when it grows by more than 8 (a factor 256): P stays
// <= 256, which bf16 and the fp32 accumulators hold exactly as well, and the O rescale
// (a TMEM read-modify-write of the row) happens a few times per row instead of per step.
// The result is exact: O = sum P V / sum P with the same reference max in both sums.
//
// TMEM (512 columns): three 128-column regions R0, R1, R2 and O in [384, 512).  Steps
// alternate: an even step's scores fill R0 R1 and its P (256 keys, bf16 pairs) goes to R0;
// an odd step's scores fill R1 R2 and its P goes to R2.  So the scores of step t+1 never
// land on P(t), and only need the softmax warps to have loaded the scores of step t (R1)
// and the product of step t-1 (issued earlier, executed in order) to have read P(t-1).
// Shared memory: Q (32 KB), 2 K stages (64 KB each), 2 V entries (32 KB each), barriers,
// the exchange buffer.
// Units are ordered (batch*head, chunk, tile): consecutive units are neighbouring tiles of
// one head, whose windows overlap in L2.
#pragma once

#include <stdint.h>

#include "sm100.cuh"

namespace dsa {

struct FwdBf16Params {
  const int32_t* kv_tiles;  // window form: [n_tiles, Wt]; list form: the caller's list [nnz]
  const int32_t* row_ptr;   // list form: CSR offsets into kv_tiles; null: window form
  int rp_head_stride;       // list form: 0 (one list for every head) or n_tiles + 1 (one per head)
  int nnz;                  // list form: entries of the list
  __nv_bfloat16* out;       // [B*heads, N, 128]
  float* lse;               // [B*heads, N]
  int n_tiles, Wt;
  int S;                    // 128-row chunks per tile
  int n_units;              // B*heads * S * n_tiles
  int G1, G2;               // Gh, Gw
  int tt, th, tw, tcs;      // tile shape; t-extent of one 128-token chunk
  int T, H, W, N;
  float scale_log2;         // scale * log2(e)
  // block-map mode only: the forward's LSE for the same lists and the map it adds into,
  // [B*heads, n_tiles, n_tiles] (zeroed by the caller)
  const float* lse_in;
  float* bmap;
  // flat mode only: dense attention of Lq query rows over Lk key rows of flat
  // [B*heads, L, 128] tensors (out, lse as [B*heads, Lq, 128] and [B*heads, Lq])
  int Lq, Lk;
  // extra (text) keys appended to every unit's keys in the forward and flat modes: Lx rows
  // of a flat [B*heads, Lx, 128] pair of tensors (0: none)
  int Lx;
  // flat mode only: the main key chunks are cut into n_split parts, one unit each; part j
  // writes out + j * part_out and lse + j * part_lse (the extra keys go with part 0)
  int n_split;
  int64_t part_out, part_lse;
};

namespace fwd {
constexpr int kThreads = 384;      // 3 warpgroups: softmax, softmax, producers + MMA (+ 1 idle warp)
constexpr int kProducerWarp = 8;   // Q and K
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10;
constexpr int kRegsSoftmax = 216;  // per-thread register budgets after setmaxnreg
constexpr int kRegsAux = 72;
constexpr int kRegsAtLaunch = (2 * 128 * kRegsSoftmax + 128 * kRegsAux) / kThreads;  // 168
static_assert(kRegsAtLaunch * kThreads == 2 * 128 * kRegsSoftmax + 128 * kRegsAux, "split must use the launch registers");
static_assert(kRegsAtLaunch <= 65536 / kThreads / 8 * 8, "one CTA per SM must fit");
constexpr int kKStages = 2;        // 256-key K stages
constexpr int kVStages = 2;        // 128-key V entries
constexpr uint32_t kTileBytes = 128 * 128 * 2;  // 128 tokens x 128 channels
constexpr uint32_t kHalfBytes = kTileBytes / 2; // 64 channels
constexpr uint32_t kStageBytes = 2 * kTileBytes;
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kTileBytes;
constexpr uint32_t kOffV = kOffK + kKStages * kStageBytes;
constexpr uint32_t kOffBar = kOffV + kVStages * kTileBytes;
constexpr uint32_t kOffX = kOffBar + 256;                // float [2 buffers][2 warpgroups][128 rows]
constexpr uint32_t kSmemUsed = kOffX + 2 * 2 * 128 * 4;  // from the 1024-aligned base
// The whole opt-in shared memory of a CTA: the part above kSmemUsed is the room the
// base's alignment may take; the kernel checks that it sufficed (it does whenever the
// dynamic shared memory starts 1024-aligned, as it does on sm_100).
constexpr uint32_t kSmemBytes = 227 * 1024;
static_assert(kSmemUsed <= kSmemBytes, "shared memory layout too large");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 384;
constexpr uint32_t kIdescS256 = idesc_bf16_f32(128, 256, 0, 0);  // Q, K both K-major (smem)
constexpr uint32_t kIdescS128 = idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 0, 1);    // P from TMEM, V MN-major (smem)
constexpr float kRescaleThreshold = 8.0f;                        // log2 units
// 16-column groups (bit g of a step's 8 groups; a half step uses the low 4) whose 2^x is
// taken from the FMA-pipe polynomial instead of the MUFU unit, which takes 16 per clock per
// SM and would otherwise bound the softmax
constexpr uint32_t kPolyMask = 0x88u;
// the block-map pass's share of 2^x on the FMA pipe: column pairs (bit e of the 8 pairs of
// every 16-column group) 1, 4 and 7, spread through each group so that the two softmax warps
// of a sub-partition keep the MUFU unit and the FMA pipe busy side by side (measured on the
// dense 16x32x32 map: 3/8 spread 2.04-2.12 ms; 2/8 spread 2.09; 4/8 2.24; 5/8 2.23-2.31;
// 2/8 as whole groups 2.16; the pass has no bf16 pack, so it takes a larger share than the
// forward)
constexpr uint32_t kPolyMaskMap = 0x92u;
// list positions of a query tile's row the block-map pass keeps totals for, one total per
// position and softmax warp (the V ring's shared memory, which the pass does not use)
constexpr int kMapCap = 1024;
static_assert(4 * 8 * kMapCap + 4 * kMapCap <= kVStages * kTileBytes, "map totals must fit in the V ring");

// TMEM columns of the scores and of P for a step of parity e.
__device__ __forceinline__ uint32_t col_s(int e) { return e ? 128u : 0u; }
__device__ __forceinline__ uint32_t col_p(int e) { return e ? 256u : 0u; }

// Kernel modes: the window / key-tile-list forward, its block-map pass, dense attention
// between flat token sequences (text tokens), and the window forward with extra (text)
// keys after every unit's own.
constexpr int kModeFwd = 0, kModeMap = 1, kModeFlat = 2, kModeFwdX = 3;

struct Unit {
  int bh, tile, sub;  // flat mode: tile = query chunk, sub = part of the key chunks
};

// Key tiles of query tile `tile` and their count: the window's Wt tiles, or the tile's
// row of the caller's list with every index clamped into the list (an invalid list gives
// wrong numbers and a device error from the list check, never an access outside it).
__device__ __forceinline__ const int32_t* unit_keys(const FwdBf16Params& p, int bh, int tile, int& n_list) {
  if (p.row_ptr == nullptr) {
    n_list = p.Wt;
    return p.kv_tiles + static_cast<int64_t>(tile) * p.Wt;
  }
  const int32_t* rp = p.row_ptr + static_cast<int64_t>(bh) * p.rp_head_stride;
  const int a = min(max(rp[tile], 0), p.nnz), b = min(max(rp[tile + 1], a), p.nnz);
  n_list = b - a;
  return p.kv_tiles + a;
}

// Flat mode: units run (batch, head), then part of the key chunks, then query chunk, so
// the query chunks that read the same keys are neighbours.
__device__ __forceinline__ Unit decode_flat(const FwdBf16Params& p, int u) {
  const int nq = (p.Lq + 127) / 128, per_bh = nq * p.n_split;
  Unit x;
  x.bh = u / per_bh;
  const int rem = u % per_bh;
  x.sub = rem / nq;  // part
  x.tile = rem % nq;
  return x;
}

// Key chunks of a unit: nm main chunks from main chunk c0 (the tiles' 128-row chunks, or
// rows of the flat key sequence), then nx chunks of the extra keys.
struct Chunks {
  int c0, nm, nx;
};

template <bool kFlat, bool kExtra>
__device__ __forceinline__ Chunks unit_chunks(const FwdBf16Params& p, const Unit& x, int n_list) {
  Chunks k;
  const int nx = kExtra ? (p.Lx + 127) / 128 : 0;
  if constexpr (kFlat) {
    const int n_main = (p.Lk + 127) / 128, per = (n_main + p.n_split - 1) / p.n_split;
    k.c0 = x.sub * per;
    k.nm = max(min(per, n_main - k.c0), 0);
    k.nx = x.sub == 0 ? nx : 0;
  } else {
    k.c0 = 0;
    k.nm = n_list * p.S;
    k.nx = nx;
  }
  return k;
}

// Keys present in local chunk j of a unit: the last chunk of a flat sequence and of the
// extra keys can be partial.
template <bool kFlat, bool kExtra>
__device__ __forceinline__ int chunk_valid(const FwdBf16Params& p, const Chunks& k, int j) {
  if (!kFlat && !kExtra) return 128;
  if (j < k.nm) return kFlat ? min(p.Lk - 128 * (k.c0 + j), 128) : 128;
  return min(p.Lx - 128 * (j - k.nm), 128);
}

// Units run head-major, then tile, then the tile's 128-row chunks: the chunks of a tile
// (same key set) are neighbouring units, so the persistent CTAs take them at the same time
// and each key tile is read from DRAM about once per head.
__device__ __forceinline__ Unit decode(const FwdBf16Params& p, int u) {
  Unit x;
  const int per_bh = p.S * p.n_tiles;
  x.bh = u / per_bh;
  const int rem = u % per_bh;
  x.tile = rem / p.S;
  x.sub = rem % p.S;
  return x;
}

// The CTA's it-th work unit.  The forward and flat modes stride over the unit sequence; the
// block-map mode takes every chunk of a query tile in one CTA (tiles strided over the grid,
// a tile's chunks in order), so that one CTA owns each row of the map and sums it in a fixed
// order.
template <int kMode>
__device__ __forceinline__ bool next_unit(const FwdBf16Params& p, int it, Unit& x) {
  if constexpr (kMode == kModeMap) {
    const int64_t tu = blockIdx.x + static_cast<int64_t>(it / p.S) * gridDim.x;
    if (tu >= p.n_units / p.S) return false;
    x.bh = static_cast<int>(tu / p.n_tiles);
    x.tile = static_cast<int>(tu % p.n_tiles);
    x.sub = it % p.S;
    return true;
  } else {
    const int64_t u = blockIdx.x + static_cast<int64_t>(it) * gridDim.x;
    if (u >= p.n_units) return false;
    x = kMode == kModeFlat ? decode_flat(p, static_cast<int>(u)) : decode(p, static_cast<int>(u));
    return true;
  }
}

// Shared-memory descriptors are built once; a byte offset is added in 16-byte units to
// the address field (all addresses stay below 256 KB, so the 14-bit field cannot carry).
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

// Makes a value opaque to the compiler at this point, so that descriptor arithmetic
// derived from it is done where it is used instead of being hoisted out of the loops and
// held in registers (the MMA warp runs under a small setmaxnreg budget).
__device__ __forceinline__ void opaque(uint64_t& v) { asm volatile("" : "+l"(v)); }

// S = Q K^T over the 128 channels: 8 k-steps of 16 within the two 64-channel halves.  A K
// stage holds channel half h of chunk b at h * 32 KB + b * 16 KB, so the 256 keys of a
// step are one K-major operand of 256 rows per channel half.
__device__ __forceinline__ void issue_scores(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc, bool full) {
  opaque(q_desc);
  opaque(k_desc);
  const uint32_t idesc = full ? kIdescS256 : kIdescS128;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ss_warp(d_tmem, desc_add(q_desc, (kk >> 2) * kHalfBytes + (kk & 3) * 32),
                desc_add(k_desc, (kk >> 2) * kTileBytes + (kk & 3) * 32), idesc, kk > 0);
}

// O (+)= P V over one 128-key chunk: P from TMEM, 8 columns of packed bf16 per 16 keys; V
// an MN-major tile, 16 keys = 2048 bytes per k-step.
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint64_t v_desc, bool accumulate) {
  opaque(v_desc);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts_warp(d_tmem, p_tmem + kk * 8, desc_add(v_desc, kk * 2048), kIdescPV, accumulate || kk > 0);
}

// Barrier wait by a whole warp, with a warp-uniform result.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int site) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, site));
}

// Exchange of one float per row between the two threads of a row (same lane of warps w
// and w + 4).  Double-buffered by exchange count, so a value is never overwritten before
// the partner has read it: the next write to a buffer follows the partner's next barrier,
// which follows its read.  The tcgen05 fences order each thread's earlier TMEM reads
// before the partner's later TMEM writes (P lands partly on the partner's score columns).
__device__ __forceinline__ float pair_exchange(float* xbuf, int& xe, int i, int r, int bar_id, float v) {
  float* b = xbuf + (xe & 1) * 256;
  ++xe;
  b[i * 128 + r] = v;
  tc_fence_before();
  named_bar_sync(bar_id, 64);
  tc_fence_after();
  return b[(i ^ 1) * 128 + r];
}

// The softmax of one step for this thread's NC score columns at tS (NC = 128: a full step,
// NC = 64: a half step): agrees on the row max with the partner thread, writes packed bf16
// P (NC/2 columns) at tP, updates m_used and l, and returns whether the reference max
// moved; it arrives on the mbarrier at `loaded` (a shared::cta address, or with kCluster a
// shared::cluster one, possibly the peer CTA's) as soon as its scores are in registers.  Columns from
// nvalid on hold no key (the tail of a flat key sequence) and get probability 0 (alpha: the factor the old O and l take).  With !ok (an earlier wait failed; TMEM
// stays allocated, so the load is harmless) the thread still takes part in the exchange,
// so its partner never waits for it, and does nothing else.  The load is unconditional: a
// load under `ok` with the exchange between it and the use makes the compiler keep far
// more registers live.
template <int NC, bool kCluster = false>
__device__ __forceinline__ bool softmax_step(bool ok, uint32_t tS, uint32_t tP, uint32_t loaded, float scale_log2,
                                             float& m_used, float& l, float& alpha, float* xbuf, int& xe, int i,
                                             int r, int bar_id, int nvalid = NC) {
  uint32_t s[NC];
  if constexpr (NC == 128)
    tmem_ld128_wait(tS, s);
  else
    tmem_ld64_wait(tS, s);
  if (nvalid < NC) {  // columns past the end of a flat key sequence: no key, score -inf
#pragma unroll
    for (int c = 0; c < NC; ++c)
      if (c >= nvalid) s[c] = 0xff800000u;
  }
  if (ok) {  // the scores are in registers: their TMEM columns may be overwritten
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
      if constexpr (kCluster)
        mbar_arrive_cluster(loaded);
      else
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(loaded) : "memory");
    }
  }
  // row max: 8 independent chains over columns e, e + 8, ..., e + NC - 8
  float mxs[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    mxs[e] = fmaxf(__uint_as_float(s[e]), __uint_as_float(s[NC - 8 + e]));
#pragma unroll
    for (int c = 8 + e; c < NC - 8; c += 16)
      mxs[e] = max3f(mxs[e], __uint_as_float(s[c]), __uint_as_float(s[c + 8]));
  }
  float mx = max3f(max3f(mxs[0], mxs[1], mxs[2]), max3f(mxs[3], mxs[4], mxs[5]), fmaxf(mxs[6], mxs[7]));
  mx = fmaxf(mx, pair_exchange(xbuf, xe, i, r, bar_id, ok ? mx : -INFINITY));
  alpha = 1.f;
  if (!ok) return false;
  const float m_new = fmaxf(m_used, mx * scale_log2);
  const bool need = m_new > m_used + kRescaleThreshold;
  if (need) {
    alpha = ex2_approx(m_used - m_new);
    m_used = m_new;
  }
  l *= alpha;
  const float neg_m = -m_used;
  // P = 2^(s * scale * log2 e - m): paired fp32 arithmetic; the kPolyMask column groups
  // go to the FMA-pipe polynomial to unload the MUFU unit
  float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int g = 0; g < NC / 16; ++g) {
    uint32_t pk[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float x0, x1, p0, p1;
      ffma2(x0, x1, __uint_as_float(s[16 * g + 2 * e]), __uint_as_float(s[16 * g + 2 * e + 1]), scale_log2,
            scale_log2, neg_m, neg_m);
      if ((kPolyMask >> g) & 1u) {
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
  for (int h = 0; h < NC / 64; ++h) {
    uint32_t w[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) w[e] = s[32 * h + e];
    tmem_st32(tP + 32 * h, w);
  }
  return need;
}

// Token index of row r of 128-row chunk `sub` of query tile `tile`.
__device__ __forceinline__ int64_t chunk_token(const FwdBf16Params& p, int tile, int sub, int r) {
  const int qt = tile / (p.G1 * p.G2), qh = (tile / p.G2) % p.G1, qw = tile % p.G2;
  const int lw = r % p.tw, lh = (r / p.tw) % p.th, lt = r / (p.tw * p.th);
  const int t0 = qt * p.tt + sub * p.tcs;
  return (static_cast<int64_t>(t0 + lt) * p.H + (qh * p.th + lh)) * p.W + (qw * p.tw + lw);
}

// O row columns [0, 32 * groups) of this thread's lane times alpha (TMEM read-modify-write).
__device__ __forceinline__ void rescale_o(uint32_t tO, int groups, float alpha) {
#pragma unroll 1
  for (int g = 0; g < groups; ++g) {
    uint32_t o[32];
    tmem_ld32_wait(tO + 32 * g, o);
#pragma unroll
    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
    tmem_st32(tO + 32 * g, o);
  }
}

// Writes O row columns [0, 32 * groups) from tO, times inv, as bf16 to dst (only where
// `write`: the TMEM loads are warp-collective and run on every lane regardless).
__device__ __forceinline__ void store_o(uint32_t tO, int groups, float inv, uint4* dst, bool write = true) {
#pragma unroll 1
  for (int g = 0; g < groups; ++g) {
    uint32_t o[32];
    tmem_ld32_wait(tO + 32 * g, o);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint4 v;
      v.x = pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv);
      v.y = pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv);
      v.z = pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv);
      v.w = pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv);
      if (write) dst[4 * g + c] = v;
    }
  }
}
}  // namespace fwd

// kMode = kModeFwd: the forward (O, LSE).  kModeMap: the block attention mass of the same
// units against a given LSE, bmap[bh][query tile][key tile] += (1 / tile tokens) *
// sum over the unit's rows and the key tile's keys of exp(scale q.k - lse) -- the scores are
// recomputed with the same products and ring, without V, P.V, the row max or the epilogue.
// kModeFlat: dense attention between flat sequences (rank-3 tensor maps [128, L, B*heads]):
// every query chunk over every key chunk, the tail of the last key chunk masked.
// kModeFwdX: kModeFwd with p.Lx extra (text) keys after every unit's own (maps tmKx, tmVx).
template <int kMode>
__global__ void __launch_bounds__(fwd::kThreads, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKx,
                    const __grid_constant__ CUtensorMap tmVx, FwdBf16Params p) {
  using namespace fwd;
  constexpr bool kMap = kMode == kModeMap, kFlat = kMode == kModeFlat;
  constexpr bool kExtra = kFlat || kMode == kModeFwdX;  // extra keys possible (p.Lx > 0)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  if (pad + kSmemUsed > kSmemBytes) {  // uniform over the CTA: nothing has started yet
    if (threadIdx.x == 0) device_report(DSA_DEV_BOUNDS, 1);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;               // [kKStages]
  uint64_t* k_empty = k_full + kKStages;     // [kKStages]
  uint64_t* v_full = k_empty + kKStages;     // [kVStages]
  uint64_t* v_empty = v_full + kVStages;     // [kVStages]
  uint64_t* s_full = v_empty + kVStages;     // [2] scores of a step of parity e ready
  uint64_t* p_full = s_full + 2;             // [2] P of a step of parity e written (8 warps)
  uint64_t* s_read = s_full + 4;             // [2] scores of a step of parity e loaded (8 warps)
  uint64_t* o_done = s_full + 6;             // a product into O done
  uint64_t* o_free = s_full + 7;             // O read out (8 warps)
  uint64_t* o_final = s_full + 8;            // every product of a unit done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 9);
  volatile int* abort = reinterpret_cast<volatile int*>(s_full + 10);
  float* xbuf = reinterpret_cast<float*>(smem + kOffX);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

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
      mbar_init(p_full + e, 8);
      mbar_init(s_read + e, 8);
    }
    mbar_init(o_done, 1);
    mbar_init(o_free, 8);
    mbar_init(o_final, 1);
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
    if (warp == kProducerWarp || (warp == kVProducerWarp && !kMap)) {
      // ------------------------------------------------------------------ TMA producers
      if (lane == 0) {
        const bool is_k = warp == kProducerWarp;
        int ld = 0, uc = 0;  // ring entries loaded, units with keys
        bool ok = true;
        Unit x;
        for (int it = 0; ok && next_unit<kMode>(p, it, x); ++it) {
          int n_list = 0;
          const int32_t* kv = kFlat ? nullptr : unit_keys(p, x.bh, x.tile, n_list);
          const Chunks ck = unit_chunks<kFlat, kExtra>(p, x, n_list);
          const int n_chunks = ck.nm + ck.nx, n_steps = (n_chunks + 1) / 2;
          if (n_chunks == 0) continue;  // nothing to load: the softmax warps write O = 0
          if (is_k) {
            ok = mbar_wait(q_empty, (uc & 1) ^ 1, abort, 20);
            if (!ok) break;
            mbar_arrive_expect_tx(q_full, kTileBytes);
            if constexpr (kFlat) {
              tma_load_3d(smem + kOffQ, &tmQ, q_full, 0, 128 * x.tile, x.bh);
              tma_load_3d(smem + kOffQ + kHalfBytes, &tmQ, q_full, 64, 128 * x.tile, x.bh);
            } else {
              const int qt = x.tile / (p.G1 * p.G2), qh = (x.tile / p.G2) % p.G1, qw = x.tile % p.G2;
              const int tq0 = qt * p.tt + x.sub * p.tcs;
              tma_load_5d(smem + kOffQ, &tmQ, q_full, 0, qw * p.tw, qh * p.th, tq0, x.bh);
              tma_load_5d(smem + kOffQ + kHalfBytes, &tmQ, q_full, 64, qw * p.tw, qh * p.th, tq0, x.bh);
            }
          }
          ++uc;
          // K: one stage per step, chunk b's channel half h at h * 32 KB + b * 16 KB;
          // V: one entry per chunk
          const int n_loads = is_k ? n_steps : n_chunks;
          for (int j = 0; j < n_loads && ok; ++j, ++ld) {
            const int n_st = is_k ? kKStages : kVStages;
            const int st = ld % n_st;
            ok = mbar_wait((is_k ? k_empty : v_empty) + st, ((ld / n_st) & 1) ^ 1, abort, is_k ? 21 : 22);
            if (!ok) break;
            const int nb = is_k ? (2 * j + 1 < n_chunks ? 2 : 1) : 1;
            uint64_t* full = (is_k ? k_full : v_full) + st;
            mbar_arrive_expect_tx(full, nb * kTileBytes);
            for (int b = 0; b < nb; ++b) {
              const int jc = is_k ? 2 * j + b : j;  // the unit's chunk
              if (kExtra && jc >= ck.nm) {  // extra keys (rows past Lx load as zeros and are masked)
                const int row = 128 * (jc - ck.nm);
                if (is_k) {
                  uint8_t* dst = smem + kOffK + st * kStageBytes + b * kHalfBytes;
                  tma_load_3d(dst, &tmKx, full, 0, row, x.bh);
                  tma_load_3d(dst + kTileBytes, &tmKx, full, 64, row, x.bh);
                } else {
                  uint8_t* dst = smem + kOffV + st * kTileBytes;
                  tma_load_3d(dst, &tmVx, full, 0, row, x.bh);
                  tma_load_3d(dst + kHalfBytes, &tmVx, full, 64, row, x.bh);
                }
                continue;
              }
              const int c = ck.c0 + jc;
              if constexpr (kFlat) {  // rows past Lk load as zeros (and are masked)
                if (is_k) {
                  uint8_t* dst = smem + kOffK + st * kStageBytes + b * kHalfBytes;
                  tma_load_3d(dst, &tmK, full, 0, 128 * c, x.bh);
                  tma_load_3d(dst + kTileBytes, &tmK, full, 64, 128 * c, x.bh);
                } else {
                  uint8_t* dst = smem + kOffV + st * kTileBytes;
                  tma_load_3d(dst, &tmV, full, 0, 128 * c, x.bh);
                  tma_load_3d(dst + kHalfBytes, &tmV, full, 64, 128 * c, x.bh);
                }
                continue;
              }
              const int kt = min(max(kv[c / p.S], 0), p.n_tiles - 1), ks = c % p.S;
              const int t0 = (kt / (p.G1 * p.G2)) * p.tt + ks * p.tcs;
              const int h0 = ((kt / p.G2) % p.G1) * p.th, w0 = (kt % p.G2) * p.tw;
              if (is_k) {
                uint8_t* dst = smem + kOffK + st * kStageBytes + b * kHalfBytes;
                tma_load_5d(dst, &tmK, full, 0, w0, h0, t0, x.bh);
                tma_load_5d(dst + kTileBytes, &tmK, full, 64, w0, h0, t0, x.bh);
              } else {
                uint8_t* dst = smem + kOffV + st * kTileBytes;
                tma_load_5d(dst, &tmV, full, 0, w0, h0, t0, x.bh);
                tma_load_5d(dst + kHalfBytes, &tmV, full, 64, w0, h0, t0, x.bh);
              }
            }
          }
        }
      }
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------------------ MMA issuer (whole warp)
      const uint64_t dQ = smem_desc_sw128(sbase + kOffQ, 16, 1024);
      const uint64_t dK = smem_desc_sw128(sbase + kOffK, 16, 1024);          // stage 0, K-major
      const uint64_t dV = smem_desc_sw128(sbase + kOffV, kHalfBytes, 1024);  // entry 0, MN-major
      int ks = 0, vs = 0;             // K stages and V entries consumed
      int uc = 0, g = 0;              // units and steps so far
      int pc0 = 0, pc1 = 0;           // phases of p_full[0 / 1] and s_read[0 / 1] consumed
      bool ok = true;
      Unit xm;
      for (int it = 0; ok && next_unit<kMode>(p, it, xm); ++it) {
        int n_list = 0;
        if constexpr (!kFlat) unit_keys(p, xm.bh, xm.tile, n_list);
        const Chunks ck = unit_chunks<kFlat, kExtra>(p, xm, n_list);
        const int n_chunks = ck.nm + ck.nx, n_steps = (n_chunks + 1) / 2;
        if (n_chunks == 0) continue;
        ok = warp_wait(q_full, uc & 1, abort, 30);
        if (ok) ok = warp_wait(k_full + ks % kKStages, (ks / kKStages) & 1, abort, 31);
        if (!ok) break;
        tc_fence_after();
        issue_scores(tmem + col_s(g & 1), dQ, desc_add(dK, (ks % kKStages) * kStageBytes), n_chunks > 1);
        mma_commit_warp(s_full + (g & 1));
        mma_commit_warp(k_empty + ks % kKStages);
        ++ks;
        if (n_steps == 1) mma_commit_warp(q_empty);
        for (int t = 0; t < n_steps && ok; ++t) {
          const int e = (g + t) & 1;
          const int ph = (e == 0 ? pc0++ : pc1++) & 1;
          ok = warp_wait(s_read + e, ph, abort, 36);
          if (!ok) break;
          if (t + 1 < n_steps) {
            // the softmax warps hold the scores of step t: those of step t+1 may go in
            ok = warp_wait(k_full + ks % kKStages, (ks / kKStages) & 1, abort, 35);
            if (!ok) break;
            tc_fence_after();
            issue_scores(tmem + col_s(e ^ 1), dQ, desc_add(dK, (ks % kKStages) * kStageBytes), 2 * t + 3 < n_chunks);
            mma_commit_warp(s_full + (e ^ 1));
            mma_commit_warp(k_empty + ks % kKStages);
            ++ks;
            if (t + 2 == n_steps) mma_commit_warp(q_empty);  // every score of this unit issued
          }
          if constexpr (kMap) continue;  // scores only
          ok = warp_wait(p_full + e, ph, abort, 33);
          if (ok && t == 0) ok = warp_wait(o_free, (uc & 1) ^ 1, abort, 34);
          const int nb = 2 * t + 1 < n_chunks ? 2 : 1;
          for (int b = 0; b < nb && ok; ++b, ++vs) {
            ok = warp_wait(v_full + vs % kVStages, (vs / kVStages) & 1, abort, 32);
            if (!ok) break;
            tc_fence_after();
            issue_pv(tmem + kColO, tmem + col_p(e) + 64 * b, desc_add(dV, (vs % kVStages) * kTileBytes), t > 0 || b > 0);
            mma_commit_warp(v_empty + vs % kVStages);
          }
          if (!ok) break;
          mma_commit_warp(o_done);
        }
        if (!ok) break;
        if constexpr (!kMap) mma_commit_warp(o_final);
        g += n_steps;
        ++uc;
      }
    }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    if constexpr (kMap) {
      // ---------------------------------------------------------------- block attention mass
      // One CTA owns every chunk of a query tile (next_unit), so the tile's row of the map is
      // summed here in a fixed order and written once: per step each warp sums its 32 rows x
      // 128 keys and adds the sum to its own total for the list position (only that warp
      // writes that total, in step order); at the tile's end the eight warps' totals of each
      // position are added in warp order, and those of every position listing a key tile (in
      // list order, so a tile listed twice counts twice) are written to the map.  The named
      // barriers are taken by every map warp, even after a failed wait, so none waits for a
      // warp that has left.
      const int i = warp >> 2;
      const int r = tid & 127;
      const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const float inv_rows = 1.f / static_cast<float>(p.S * 128);
      float* acc = reinterpret_cast<float*>(smem + kOffV);                        // [8][kMapCap]
      int32_t* kvs = reinterpret_cast<int32_t*>(smem + kOffV + 4 * 8 * kMapCap);  // [kMapCap]
      float* my_acc = acc + warp * kMapCap;
      int sc0 = 0, sc1 = 0, g = 0;
      bool ok = true;
      Unit x;
      for (int it = 0; next_unit<kMode>(p, it, x); ++it) {
        int n_list;
        const int32_t* kv = unit_keys(p, x.bh, x.tile, n_list);
        const int n_chunks = n_list * p.S, n_steps = (n_chunks + 1) / 2;
        const bool fits = n_list <= kMapCap;
        if (x.sub == 0) {  // a new query tile: its totals start at zero
          named_bar_sync(5, 256);  // the previous tile's row has been written
          if (fits) {
            for (int e = tid; e < 8 * n_list; e += 256) acc[(e / n_list) * kMapCap + e % n_list] = 0.f;
            for (int e = tid; e < n_list; e += 256) kvs[e] = min(max(kv[e], 0), p.n_tiles - 1);
          } else if (tid == 0) {
            device_report(DSA_DEV_BOUNDS, 48);  // a list row longer than the map pass takes
          }
          named_bar_sync(5, 256);
        }
        const int64_t tok = chunk_token(p, x.tile, x.sub, r);
        const float neg_lse = -p.lse_in[static_cast<int64_t>(x.bh) * p.N + tok] * 1.4426950408889634f;
        for (int t = 0; t < n_steps; ++t) {
          const int e = (g + t) & 1;
          if (ok) ok = warp_wait(s_full + e, (e == 0 ? sc0++ : sc1++) & 1, abort, 49);
          if (!ok) continue;
          tc_fence_after();
          const bool full = 2 * t + 1 < n_chunks;
          uint32_t sv[128];
          if (full) {
            tmem_ld128_wait(tmem + col_s(e) + 128 * i + lane_off, sv);
          } else {
            uint32_t (&half)[64] = *reinterpret_cast<uint32_t(*)[64]>(sv);
            tmem_ld64_wait(tmem + col_s(e) + 64 * i + lane_off, half);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_read + e);  // the scores' columns may be overwritten
          const int nc = full ? 128 : 64;
          float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < 128; c += 2) {
            if (c < nc) {
              float x0, x1;
              ffma2(x0, x1, __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]), p.scale_log2, p.scale_log2, neg_lse,
                    neg_lse);
              float p0, p1;
              if ((kPolyMaskMap >> ((c >> 1) & 7)) & 1u) {  // a share of 2^x on the FMA pipe
                exp2_poly2(x0, x1, p0, p1);
              } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              fadd2(sa[(c >> 1) & 3], sb[(c >> 1) & 3], sa[(c >> 1) & 3], sb[(c >> 1) & 3], p0, p1);
            }
          }
          float sum = ((sa[0] + sb[0]) + (sa[1] + sb[1])) + ((sa[2] + sb[2]) + (sa[3] + sb[3]));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          // this warp's keys: chunk 2t + i of a full step, or half i of the single chunk 2t
          const int c = full ? 2 * t + i : 2 * t;
          if (lane == 0 && fits) my_acc[c / p.S] += sum;
        }
        g += n_steps;
        if (x.sub == p.S - 1) {
          named_bar_sync(5, 256);  // every warp's totals of the tile are complete
          float* mrow = p.bmap + (static_cast<int64_t>(x.bh) * p.n_tiles + x.tile) * p.n_tiles;
          if (fits) {
            for (int e = tid; e < n_list; e += 256) {
              const int kt = kvs[e];
              bool first = true;
              for (int f = 0; f < e && first; ++f) first = kvs[f] != kt;
              if (!first) continue;  // counted with the tile's first occurrence
              float s = 0.f;
              for (int f = e; f < n_list; ++f) {
                if (kvs[f] != kt) continue;
                float tf = 0.f;
#pragma unroll
                for (int w = 0; w < 8; ++w) tf += acc[w * kMapCap + f];
                s += tf;
              }
              mrow[kt] = s * inv_rows;
            }
          }
        }
      }
    } else {
    // ------------------------------------------------------------------ softmax
    // Every barrier is waited on at most one phase behind its count of completions: the
    // score and P barriers alternate with the step parity and each of their phases needs
    // the previous one consumed; o_done completes once per step and o_final once per unit,
    // and the next completion needs this warpgroup's own arrival.  A softmax warp never
    // leaves the unit loop early, even after a failed wait, so its partner warp finds it
    // at every named barrier.
    const int i = warp >> 2;
    const int r = tid & 127;
    const int bar_id = 1 + (warp & 3);
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + kColO + 64 * i + lane_off;  // this warpgroup's 64 channels of O
    int sc0 = 0, sc1 = 0;  // phases of s_full[0 / 1] waited
    int g = 0;             // steps before the current unit (products into O, step parity)
    int uc = 0;            // units with keys before the current one
    int xe = 0;            // pair exchanges so far
    bool ok = true;
    Unit x;
    for (int it = 0; next_unit<kMode>(p, it, x); ++it) {
      int n_list = 0;
      if constexpr (!kFlat) unit_keys(p, x.bh, x.tile, n_list);
      const Chunks ck = unit_chunks<kFlat, kExtra>(p, x, n_list);
      const int n_chunks = ck.nm + ck.nx, n_steps = (n_chunks + 1) / 2;
      // flat mode: part x.sub of the key chunks writes its own partial output
      const int64_t po = kFlat ? static_cast<int64_t>(x.sub) * p.part_out : 0;
      const int64_t pl = kFlat ? static_cast<int64_t>(x.sub) * p.part_lse : 0;
      if (n_chunks == 0) {
        // no keys: O = 0 and LSE = ln 0 = -inf (the softmax of an empty set has no value;
        // this is the limit the oracle and the list form define)
        const int64_t rows = kFlat ? p.Lq : p.N;
        const int64_t tok = kFlat ? 128 * static_cast<int64_t>(x.tile) + r : chunk_token(p, x.tile, x.sub, r);
        if (tok < rows) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + po + (static_cast<int64_t>(x.bh) * rows + tok) * 128) + 8 * i;
#pragma unroll
          for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
          if (i == 0) p.lse[pl + static_cast<int64_t>(x.bh) * rows + tok] = -INFINITY;
        }
        continue;
      }
      float m_used = -INFINITY, l = 0.f;
      for (int t = 0; t < n_steps; ++t) {
        const int e = (g + t) & 1;
        if (ok) ok = warp_wait(s_full + e, (e == 0 ? sc0++ : sc1++) & 1, abort, 40);
        if (ok) tc_fence_after();
        float alpha;
        bool need;
        // keys present in this thread's columns (a flat sequence's or the extra keys' last
        // chunk may be partial): chunk 2t + i of a full step, half i of chunk 2t otherwise
        const bool full = 2 * t + 1 < n_chunks;
        const int nvalid = full ? chunk_valid<kFlat, kExtra>(p, ck, 2 * t + i)
                                : min(max(chunk_valid<kFlat, kExtra>(p, ck, 2 * t) - 64 * i, 0), 64);
        if (full)
          need = softmax_step<128>(ok, tmem + col_s(e) + 128 * i + lane_off, tmem + col_p(e) + 64 * i + lane_off,
                                   smem_u32(s_read + e), p.scale_log2, m_used, l, alpha, xbuf, xe, i, r, bar_id, nvalid);
        else
          need = softmax_step<64>(ok, tmem + col_s(e) + 64 * i + lane_off, tmem + col_p(e) + 32 * i + lane_off,
                                  smem_u32(s_read + e), p.scale_log2, m_used, l, alpha, xbuf, xe, i, r, bar_id, nvalid);
        if (ok && t > 0 && __any_sync(0xffffffffu, need)) {
          // O holds sum P V up to step t-1 with the old reference max: rescale this
          // warpgroup's channels of it
          ok = warp_wait(o_done, (g + t - 1) & 1, abort, 41);
          if (ok) {
            tc_fence_after();
            rescale_o(tO, 2, alpha);
          }
        }
        if (ok) {
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full + e);
        }
      }
      // epilogue: O / l as bf16 (channels [64i, 64i + 64)), LSE = (m + log2 l) ln 2
      if (ok) ok = warp_wait(o_final, uc & 1, abort, 42);
      const float l_all = l + pair_exchange(xbuf, xe, i, r, bar_id, l);
      if (ok) {
        tc_fence_after();
        // row of the output: the token of the tile (window / list form) or of the flat
        // query sequence (rows past Lq of the last query chunk have no output)
        const int64_t rows = kFlat ? p.Lq : p.N;
        const int64_t tok = kFlat ? 128 * static_cast<int64_t>(x.tile) + r : chunk_token(p, x.tile, x.sub, r);
        // (the TMEM loads of store_o are warp-collective: every lane takes part, and only
        // rows that exist are written)
        const bool row_ok = tok < rows;
        store_o(tO, 2, 1.f / l_all,
                reinterpret_cast<uint4*>(p.out + po + (static_cast<int64_t>(x.bh) * rows + (row_ok ? tok : 0)) * 128) +
                    8 * i,
                row_ok);
        if (i == 0 && row_ok)
          p.lse[pl + static_cast<int64_t>(x.bh) * rows + tok] = (m_used + __log2f(l_all)) * 0.69314718055994531f;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);
      }
      g += n_steps;
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

// Merge of n attentions of the same rows over disjoint key sets (parts j = 0..n-1 at
// o + j * part_out, lse + j * part_lse):  L = ln sum_j e^lse_j,  O = sum_j e^(lse_j - L) O_j
// (exact: the softmax over the union, written through the parts' own normalisations).  A
// part with lse = -inf (no keys) has weight 0.  16 threads per 128-channel row, 8 channels
// each; fp32 sums, bf16 result.
__global__ void __launch_bounds__(256) merge_parts_kernel(const __nv_bfloat16* o, const float* lse, int n_parts,
                                                          int64_t part_out, int64_t part_lse, int64_t rows,
                                                          __nv_bfloat16* out, float* lse_out) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 16;
  const int part = threadIdx.x % 16;
  if (row >= rows) return;
  float m = -INFINITY;
  for (int j = 0; j < n_parts; ++j) m = fmaxf(m, lse[j * part_lse + row]);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float L = -INFINITY;
  if (m != -INFINITY) {
    float sum = 0.f;
    for (int j = 0; j < n_parts; ++j) sum += __expf(lse[j * part_lse + row] - m);
    L = m + __logf(sum);
    for (int j = 0; j < n_parts; ++j) {
      const float w = __expf(lse[j * part_lse + row] - L);
      const uint4 x = reinterpret_cast<const uint4*>(o + j * part_out + row * 128)[part];
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += w * __uint_as_float(xs[e] << 16);
        acc[2 * e + 1] += w * __uint_as_float(xs[e] & 0xffff0000u);
      }
    }
  }
  reinterpret_cast<uint4*>(out + row * 128)[part] =
      make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                 pack_bf16x2(acc[6], acc[7]));
  if (part == 0) lse_out[row] = L;
}

}  // namespace dsa
