// C ABI of the 3D-DSA library (declared in include/dsa.h): argument validation, workspace
// layout, TMA tensor maps and kernel launches.  The whole library is this one translation
// unit (the kernels are header-only), so the device status word is unique per device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/dsa.h"
#include "dsa_bwd_bf16.cuh"
#include "dsa_bwd_dq.cuh"
#include "dsa_device_status.cuh"
#include "dsa_fwd_bf16.cuh"
#include "dsa_fwd_f32.cuh"
#include "dsa_fwd_pair.cuh"
#include "dsa_lists.cuh"
#include "dsa_lstsq.cuh"
#include "dsa_plan.cuh"

namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Geom {
  int G[3], w[3];
  int n_tiles, Wt, tile_tokens;
  int64_t N, BH;
};

dsa_status_t check_shape(const dsa_problem_t* p, Geom* g) {
  if (p == nullptr) return DSA_ERR_INVALID_ARG;
  if (p->B <= 0 || p->heads <= 0 || p->d <= 0 || p->T <= 0 || p->H <= 0 || p->W <= 0) return DSA_ERR_INVALID_ARG;
  const int dims[3] = {p->T, p->H, p->W};
  for (int a = 0; a < 3; ++a) {
    if (p->tile[a] <= 0 || p->window[a] <= 0) return DSA_ERR_INVALID_ARG;
    if (dims[a] % p->tile[a] != 0) return DSA_ERR_INVALID_ARG;
    g->G[a] = dims[a] / p->tile[a];
    g->w[a] = p->window[a] < g->G[a] ? p->window[a] : g->G[a];
  }
  if (!(p->scale > 0.f) || !std::isfinite(p->scale)) return DSA_ERR_INVALID_ARG;
  if (p->dtype != DSA_F32 && p->dtype != DSA_BF16) return DSA_ERR_INVALID_ARG;
  const int64_t n_tiles = static_cast<int64_t>(g->G[0]) * g->G[1] * g->G[2];
  const int64_t N = static_cast<int64_t>(p->T) * p->H * p->W;
  const int64_t BH = static_cast<int64_t>(p->B) * p->heads;
  const int64_t tile_tokens = static_cast<int64_t>(p->tile[0]) * p->tile[1] * p->tile[2];
  // the kernels index a (b, head) slice with 32-bit token counts and tile lists with int32
  if (n_tiles * static_cast<int64_t>(g->w[0]) * g->w[1] * g->w[2] > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (N > INT32_MAX / 2 || BH > INT32_MAX / 2 || BH * N > (int64_t(1) << 40)) return DSA_ERR_UNSUPPORTED;
  g->n_tiles = static_cast<int>(n_tiles);
  g->Wt = g->w[0] * g->w[1] * g->w[2];
  g->tile_tokens = static_cast<int>(tile_tokens);
  g->N = N;
  g->BH = BH;
  return DSA_OK;
}

dsa_status_t check_kernel_limits(const dsa_problem_t* p, const Geom& g, bool backward) {
  if (p->dtype == DSA_F32) {
    if (backward) return DSA_ERR_UNSUPPORTED;
    if (p->d != 64 && p->d != 128) return DSA_ERR_UNSUPPORTED;
    if (g.n_tiles > 65535 * 64 || g.BH > 65535) return DSA_ERR_UNSUPPORTED;
    return DSA_OK;
  }
  if (p->d != 128) return DSA_ERR_UNSUPPORTED;
  // a 128-token query chunk and a 64-token key chunk must both be whole (h, w) planes
  const int plane = p->tile[1] * p->tile[2];
  if (plane > 64 || 64 % plane != 0) return DSA_ERR_UNSUPPORTED;
  if (p->tile[0] % (128 / plane) != 0) return DSA_ERR_UNSUPPORTED;
  // the backward reads a query chunk's LSE and D rows as TMA boxes of tw fp32 values, which
  // must be a multiple of 16 bytes
  if (backward && p->tile[2] % 4 != 0) return DSA_ERR_UNSUPPORTED;
  if (g.BH * g.n_tiles * (g.tile_tokens / 128) > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

struct FwdWorkspace {
  int32_t* starts;
  int32_t* kv_tiles;
  size_t bytes;
};

FwdWorkspace fwd_workspace(const Geom& g, void* base) {
  FwdWorkspace w;
  uint8_t* b = static_cast<uint8_t*>(base);
  size_t off = 0;
  w.starts = reinterpret_cast<int32_t*>(b + off);
  off += round_up(sizeof(int32_t) * 3 * g.n_tiles, kAlign);
  w.kv_tiles = reinterpret_cast<int32_t*>(b + off);
  off += round_up(sizeof(int32_t) * static_cast<size_t>(g.n_tiles) * g.Wt, kAlign);
  w.bytes = off;
  return w;
}

struct BwdWorkspace {
  int32_t* starts;
  int32_t* kv_tiles;
  int32_t* row_ptr;
  int32_t* q_tiles;
  float* delta;  // D = rowsum(dO * O), [BH, N]
  size_t bytes;
};

BwdWorkspace bwd_workspace(const Geom& g, void* base) {
  BwdWorkspace w;
  uint8_t* b = static_cast<uint8_t*>(base);
  size_t off = 0;
  w.starts = reinterpret_cast<int32_t*>(b + off);
  off += round_up(sizeof(int32_t) * 3 * g.n_tiles, kAlign);
  w.kv_tiles = reinterpret_cast<int32_t*>(b + off);
  off += round_up(sizeof(int32_t) * static_cast<size_t>(g.n_tiles) * g.Wt, kAlign);
  w.row_ptr = reinterpret_cast<int32_t*>(b + off);
  off += round_up(sizeof(int32_t) * (g.n_tiles + 1), kAlign);
  w.q_tiles = reinterpret_cast<int32_t*>(b + off);
  off += round_up(sizeof(int32_t) * static_cast<size_t>(g.n_tiles) * g.Wt, kAlign);
  w.delta = reinterpret_cast<float*>(b + off);
  off += round_up(sizeof(float) * static_cast<size_t>(g.BH * g.N), kAlign);
  w.bytes = off;
  return w;
}

// Backward over a caller's key-tile lists: the inverse CSR built on the device, then the
// same D scratch as dsa_bwd.
struct ListBwdWorkspace {
  int32_t* counts;   // [n_lists, n_tiles] scratch of the inversion
  int32_t* row_ptr;  // [n_lists, n_tiles + 1] inverse CSR
  int32_t* q_tiles;  // [nnz]
  float* delta;      // [BH, N]
  size_t bytes;
};

ListBwdWorkspace list_bwd_workspace(const Geom& g, int nnz, int n_lists, void* base) {
  ListBwdWorkspace w;
  uint8_t* b = static_cast<uint8_t*>(base);
  size_t off = 0;
  w.counts = reinterpret_cast<int32_t*>(b + off);
  off += round_up(sizeof(int32_t) * static_cast<size_t>(n_lists) * g.n_tiles, kAlign);
  w.row_ptr = reinterpret_cast<int32_t*>(b + off);
  off += round_up(sizeof(int32_t) * static_cast<size_t>(n_lists) * (g.n_tiles + 1), kAlign);
  w.q_tiles = reinterpret_cast<int32_t*>(b + off);
  off += round_up(sizeof(int32_t) * static_cast<size_t>(nnz > 0 ? nnz : 1), kAlign);
  w.delta = reinterpret_cast<float*>(b + off);
  off += round_up(sizeof(float) * static_cast<size_t>(g.BH * g.N), kAlign);
  w.bytes = off;
  return w;
}

dsa::PlanGeom plan_geom(const Geom& g) {
  dsa::PlanGeom pg;
  for (int a = 0; a < 3; ++a) {
    pg.G[a] = g.G[a];
    pg.w[a] = g.w[a];
  }
  pg.n_tiles = g.n_tiles;
  pg.n_window_tiles = g.Wt;
  return pg;
}

// Number of SMs of the current device (persistent kernels launch one CTA per SM).
dsa_status_t sm_count(int* n) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || *n <= 0) return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t launch_status() {
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---- TMA tensor maps (driver entry point fetched through the runtime; no libcuda link)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (thread-safe static initialisation).
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return nullptr;
  }();
  return fn;
}

// A [BH, T, H, W, 128] bf16 tensor seen as 5-D (d, W, H, T, BH); one box is a chunk of
// box_tokens tokens of a tile (tw x th x box_tokens/(tw*th)) times 64 channels, 128-byte
// swizzled.
bool make_token_map(CUtensorMap* map, const void* ptr, const dsa_problem_t* p, const Geom& g, int box_tokens = 128) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const int tcs = box_tokens / (p->tile[1] * p->tile[2]);
  cuuint64_t dims[5] = {128, static_cast<cuuint64_t>(p->W), static_cast<cuuint64_t>(p->H),
                        static_cast<cuuint64_t>(p->T), static_cast<cuuint64_t>(g.BH)};
  cuuint64_t strides[4] = {128 * 2, static_cast<cuuint64_t>(p->W) * 128 * 2,
                           static_cast<cuuint64_t>(p->H) * p->W * 128 * 2,
                           static_cast<cuuint64_t>(p->T) * p->H * p->W * 128 * 2};
  cuuint32_t box[5] = {64, static_cast<cuuint32_t>(p->tile[2]), static_cast<cuuint32_t>(p->tile[1]),
                       static_cast<cuuint32_t>(tcs), 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A [BH, T, H, W] fp32 per-token vector (LSE, D) seen as 4-D (W, H, T, BH); one box is
// the box_tokens tokens of a tile chunk (tw x th x box_tokens/(tw*th)), no swizzle.
bool make_row_map(CUtensorMap* map, const void* ptr, const dsa_problem_t* p, const Geom& g, int box_tokens) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const int tcs = box_tokens / (p->tile[1] * p->tile[2]);
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(p->W), static_cast<cuuint64_t>(p->H), static_cast<cuuint64_t>(p->T),
                        static_cast<cuuint64_t>(g.BH)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(p->W) * 4, static_cast<cuuint64_t>(p->H) * p->W * 4,
                           static_cast<cuuint64_t>(p->T) * p->H * p->W * 4};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(p->tile[2]), static_cast<cuuint32_t>(p->tile[1]),
                       static_cast<cuuint32_t>(tcs), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A flat [BH, L, 128] bf16 token sequence seen as 3-D (128, L, BH); one box is 64 channels
// of box_rows consecutive tokens (rows past L load as zeros).
bool make_flat_map(CUtensorMap* map, const void* ptr, int64_t BH, int64_t L, int box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {128 * 2, static_cast<cuuint64_t>(L) * 128 * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A wait on a barrier that nothing completes: the library's bounded wait runs out, records
// DSA_DEV_TIMEOUT at `site` and the kernel returns (the failure path, exercised on purpose).
__global__ void selftest_wait_kernel(int site) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    dsa::mbar_init(&bar, 1);
    abort_flag = 0;
    dsa::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) dsa::mbar_wait(&bar, 0, &abort_flag, site);
}

// fp32 rows [BH, L] (L * 4 bytes a multiple of 16) seen as 2-D (L, BH); one box is 64
// consecutive rows of one (batch, head) (rows past L load as zeros).
bool make_vec_map(CUtensorMap* map, const void* ptr, int64_t BH, int64_t L) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(L) * 4};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Validation of a caller's CSR on the device (records DSA_DEV_BOUNDS; never faults).
dsa_status_t launch_list_check(const Geom& g, const int32_t* row_ptr, const int32_t* list, int n_lists, int nnz,
                               cudaStream_t s) {
  const int64_t n_ptr = static_cast<int64_t>(n_lists) * (g.n_tiles + 1);
  const int64_t work = n_ptr > nnz ? n_ptr : nnz;
  int64_t blocks = (work + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > 1024) blocks = 1024;
  dsa::list_check_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(row_ptr, list, g.n_tiles, n_lists, nnz);
  return launch_status();
}

dsa_status_t launch_plan(const Geom& g, const int32_t* offsets, int32_t* starts, int32_t* kv_tiles,
                         int32_t* row_ptr, int32_t* q_tiles, cudaStream_t s) {
  const dsa::PlanGeom pg = plan_geom(g);
  dsa::plan_kernel<<<1, 1024, 0, s>>>(pg, offsets, starts, kv_tiles);
  dsa_status_t st = launch_status();
  if (st != DSA_OK || row_ptr == nullptr || q_tiles == nullptr) return st;
  // inverse map: one warp per key tile, at most 8 warps per CTA and 8 CTAs per SM
  int sms = 0;
  if (sm_count(&sms) != DSA_OK) return DSA_ERR_CUDA;
  const int64_t want = (static_cast<int64_t>(g.n_tiles) + 7) / 8;
  const unsigned blocks = static_cast<unsigned>(want < 8 * sms ? want : 8 * sms);
  dsa::plan_inverse_kernel<false><<<blocks, 256, 0, s>>>(pg, starts, row_ptr, nullptr);
  st = launch_status();
  if (st != DSA_OK) return st;
  dsa::plan_scan_kernel<<<1, 1024, 0, s>>>(g.n_tiles, row_ptr);
  st = launch_status();
  if (st != DSA_OK) return st;
  dsa::plan_inverse_kernel<true><<<blocks, 256, 0, s>>>(pg, starts, row_ptr, q_tiles);
  return launch_status();
}

// Clusters of two the CTA-pair forward can keep resident on the current device (one CTA
// per SM), looked up once per device and kernel (atomically cached: host threads may call
// concurrently); 0 if none fits.  Also checks, as for the single-CTA kernel, that the
// kernel got the registers its setmaxnreg split needs.
constexpr int kPairMaxDevices = 128;

dsa_status_t pair_cluster_count(void (*kernel)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
                                               dsa::FwdBf16Params),
                                int sms, int* clusters) {
  static std::atomic<int> cache[2][kPairMaxDevices] = {};
  const int which = kernel == dsa::fwd_pair_kernel<true> ? 1 : 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dsa::fwdp::kSmemBytes) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return DSA_ERR_CUDA;
  if (fa.numRegs < dsa::fwd::kRegsAtLaunch) return DSA_ERR_UNSUPPORTED;
  if (dev >= 0 && dev < kPairMaxDevices) {
    const int c = cache[which][dev].load(std::memory_order_relaxed);
    if (c > 0) {
      *clusters = c;
      return DSA_OK;
    }
  }
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(sms >= 2 ? sms / 2 * 2 : 2), 1, 1);
  cfg.blockDim = dim3(dsa::fwdp::kThreads, 1, 1);
  cfg.dynamicSmemBytes = dsa::fwdp::kSmemBytes;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  if (n > sms / 2) n = sms / 2;
  if (n > 0 && dev >= 0 && dev < kPairMaxDevices) cache[which][dev].store(n, std::memory_order_relaxed);
  *clusters = n;
  return DSA_OK;
}

// kv_tiles: the plan's [n_tiles, Wt] key tiles (row_ptr null) or a caller's key-tile list
// with its CSR offsets row_ptr [n_tiles + 1] and nnz entries (bf16 only).
dsa_status_t launch_fwd(const dsa_problem_t* p, const Geom& g, const void* q, const void* k, const void* v,
                        const int32_t* kv_tiles, void* out, float* lse, cudaStream_t s,
                        const int32_t* row_ptr = nullptr, int nnz = 0, int rp_head_stride = 0,
                        const float* lse_in = nullptr, float* bmap = nullptr, const void* kx = nullptr,
                        const void* vx = nullptr, int Lx = 0) {
  if (p->dtype == DSA_F32) {
    dsa::FwdF32Params fp;
    fp.q = static_cast<const float*>(q);
    fp.k = static_cast<const float*>(k);
    fp.v = static_cast<const float*>(v);
    fp.kv_tiles = kv_tiles;
    fp.out = static_cast<float*>(out);
    fp.lse = lse;
    fp.T = p->T;
    fp.H = p->H;
    fp.W = p->W;
    fp.N = static_cast<int>(g.N);
    fp.tt = p->tile[0];
    fp.th = p->tile[1];
    fp.tw = p->tile[2];
    fp.tile_tokens = g.tile_tokens;
    fp.G1 = g.G[1];
    fp.G2 = g.G[2];
    fp.Wt = g.Wt;
    fp.scale = p->scale;
    const int rows_per_block = dsa::kF32Threads / (p->d / 64);
    dim3 grid(g.n_tiles, static_cast<unsigned>(g.BH), (g.tile_tokens + rows_per_block - 1) / rows_per_block);
    if (p->d == 64)
      dsa::fwd_f32_kernel<64><<<grid, dsa::kF32Threads, 0, s>>>(fp);
    else
      dsa::fwd_f32_kernel<128><<<grid, dsa::kF32Threads, 0, s>>>(fp);
    return launch_status();
  }
  CUtensorMap tq, tk, tv, tkx, tvx;
  if (!make_token_map(&tq, q, p, g, 128) || !make_token_map(&tk, k, p, g, 128) || !make_token_map(&tv, v, p, g, 128))
    return DSA_ERR_CUDA;
  if (Lx > 0) {  // extra (text) keys after every query tile's own
    if (bmap != nullptr || !make_flat_map(&tkx, kx, g.BH, Lx) || !make_flat_map(&tvx, vx, g.BH, Lx))
      return DSA_ERR_CUDA;
  } else {
    tkx = tk;
    tvx = tv;
  }
  dsa::FwdBf16Params bp;
  std::memset(&bp, 0, sizeof(bp));
  bp.Lx = Lx > 0 ? Lx : 0;
  bp.n_split = 1;
  bp.kv_tiles = kv_tiles;
  bp.row_ptr = row_ptr;
  bp.rp_head_stride = rp_head_stride;
  bp.nnz = nnz;
  bp.lse_in = lse_in;
  bp.bmap = bmap;
  bp.out = static_cast<__nv_bfloat16*>(out);
  bp.lse = lse;
  bp.n_tiles = g.n_tiles;
  bp.Wt = g.Wt;
  bp.S = g.tile_tokens / 128;
  bp.G1 = g.G[1];
  bp.G2 = g.G[2];
  bp.tt = p->tile[0];
  bp.th = p->tile[1];
  bp.tw = p->tile[2];
  bp.tcs = 128 / (p->tile[1] * p->tile[2]);
  bp.T = p->T;
  bp.H = p->H;
  bp.W = p->W;
  bp.N = static_cast<int>(g.N);
  bp.scale_log2 = p->scale * 1.4426950408889634f;
  bp.n_units = static_cast<int>(g.BH * bp.S * g.n_tiles);
  const bool map_mode = bmap != nullptr;
  int sms = 0;
  if (sm_count(&sms) != DSA_OK) return DSA_ERR_CUDA;
  if (!map_mode && row_ptr == nullptr && bp.S % 2 == 0) {
    // the window form with an even number of 128-row chunks per tile: one product per pair
    // of SMs over two chunks of a tile (which share its window)
    auto pk = bp.Lx > 0 ? dsa::fwd_pair_kernel<true> : dsa::fwd_pair_kernel<false>;
    int clusters = 0;
    const dsa_status_t st = pair_cluster_count(pk, sms, &clusters);
    if (st != DSA_OK) return st;
    if (clusters > 0) {
      const int pairs = bp.n_units / 2;
      const unsigned grid = static_cast<unsigned>(2 * (clusters < pairs ? clusters : pairs));
      pk<<<grid, dsa::fwdp::kThreads, dsa::fwdp::kSmemBytes, s>>>(tq, tk, tv, tkx, tvx, bp);
      return launch_status();
    }
    // no cluster of two fits on this device: the single-CTA kernel below
  }
  auto kernel = map_mode ? dsa::fwd_bf16_kernel<dsa::fwd::kModeMap>
                         : (bp.Lx > 0 ? dsa::fwd_bf16_kernel<dsa::fwd::kModeFwdX> : dsa::fwd_bf16_kernel<dsa::fwd::kModeFwd>);
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dsa::fwd::kSmemBytes) != cudaSuccess)
    return DSA_ERR_CUDA;
  // the kernel's setmaxnreg split needs exactly the registers it was compiled for at launch
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return DSA_ERR_CUDA;
  if (fa.numRegs < dsa::fwd::kRegsAtLaunch) return DSA_ERR_UNSUPPORTED;
  // the block-map pass takes whole query tiles (all their chunks) per CTA
  const int units = map_mode ? bp.n_units / bp.S : bp.n_units;
  const unsigned grid = static_cast<unsigned>(units < sms ? units : sms);
  kernel<<<grid, dsa::fwd::kThreads, dsa::fwd::kSmemBytes, s>>>(tq, tk, tv, tkx, tvx, bp);
  return launch_status();
}

// Dense attention of Lq flat query rows over Lk flat key rows and Lx flat extra key rows
// ([BH, L, 128] bf16 each), the main keys cut into n_split parts: part j writes
// out + j * part_out ([BH, Lq, 128] bf16) and lse + j * part_lse ([BH, Lq] fp32).
dsa_status_t launch_flat(const void* q, const void* k, const void* v, const void* kx, const void* vx, int64_t BH,
                         int Lq, int Lk, int Lx, int n_split, float scale, void* out, float* lse, int64_t part_out,
                         int64_t part_lse, cudaStream_t s) {
  CUtensorMap tq, tk, tv, tkx, tvx;
  if (!make_flat_map(&tq, q, BH, Lq) || !make_flat_map(&tk, k, BH, Lk) || !make_flat_map(&tv, v, BH, Lk))
    return DSA_ERR_CUDA;
  if (Lx > 0) {
    if (!make_flat_map(&tkx, kx, BH, Lx) || !make_flat_map(&tvx, vx, BH, Lx)) return DSA_ERR_CUDA;
  } else {
    tkx = tk;
    tvx = tv;
  }
  dsa::FwdBf16Params bp;
  std::memset(&bp, 0, sizeof(bp));
  bp.out = static_cast<__nv_bfloat16*>(out);
  bp.lse = lse;
  bp.Lq = Lq;
  bp.Lk = Lk;
  bp.Lx = Lx > 0 ? Lx : 0;
  bp.n_split = n_split;
  bp.part_out = part_out;
  bp.part_lse = part_lse;
  bp.n_tiles = 1;
  bp.S = 1;
  bp.N = Lq;
  bp.n_units = static_cast<int>(BH * ((Lq + 127) / 128) * n_split);
  bp.scale_log2 = scale * 1.4426950408889634f;
  auto kernel = dsa::fwd_bf16_kernel<dsa::fwd::kModeFlat>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dsa::fwd::kSmemBytes) != cudaSuccess)
    return DSA_ERR_CUDA;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return DSA_ERR_CUDA;
  if (fa.numRegs < dsa::fwd::kRegsAtLaunch) return DSA_ERR_UNSUPPORTED;
  int sms = 0;
  if (sm_count(&sms) != DSA_OK) return DSA_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(bp.n_units < sms ? bp.n_units : sms);
  kernel<<<grid, dsa::fwd::kThreads, dsa::fwd::kSmemBytes, s>>>(tq, tk, tv, tkx, tvx, bp);
  return launch_status();
}

dsa_status_t launch_merge_parts(const void* o, const float* lse, int n_parts, int64_t part_out, int64_t part_lse,
                                int64_t rows, void* out, float* lse_out, cudaStream_t s) {
  dsa::merge_parts_kernel<<<static_cast<unsigned>((rows * 16 + 255) / 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(o), lse, n_parts, part_out, part_lse, rows, static_cast<__nv_bfloat16*>(out),
      lse_out);
  return launch_status();
}

// Key tiles of each query tile as the forward takes them: the window plan's kv_tiles
// (row_ptr null) or a caller's CSR (row_ptr, nnz entries, rp_head_stride 0 or nTiles + 1).
struct FwdKeys {
  const int32_t* kv;
  const int32_t* row_ptr;
  int nnz, rp_head_stride;
};

// Parameters of the dQ kernel for the problem's tile geometry (the window / list form).
dsa::BwdDqParams dq_params(const dsa_problem_t* p, const Geom& g, const float* lse, const float* delta, void* dq) {
  dsa::BwdDqParams dp;
  std::memset(&dp, 0, sizeof(dp));
  dp.lse = lse;
  dp.delta = delta;
  dp.dq = static_cast<__nv_bfloat16*>(dq);
  dp.n_tiles = g.n_tiles;
  dp.Wt = g.Wt;
  dp.S = g.tile_tokens / 128;
  dp.KS = g.tile_tokens / 128;
  dp.n_units = static_cast<int>(g.BH * g.n_tiles * dp.S);
  dp.G1 = g.G[1];
  dp.G2 = g.G[2];
  dp.tt = p->tile[0];
  dp.th = p->tile[1];
  dp.tw = p->tile[2];
  dp.tcs = 128 / (p->tile[1] * p->tile[2]);
  dp.kcs = 128 / (p->tile[1] * p->tile[2]);
  dp.T = p->T;
  dp.H = p->H;
  dp.W = p->W;
  dp.N = static_cast<int>(g.N);
  dp.scale = p->scale;
  dp.scale_log2 = p->scale * 1.4426950408889634f;
  dp.n_split = 1;
  return dp;
}

template <bool kFlat, bool kExtra>
dsa_status_t launch_dq(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tkx, const CUtensorMap& tvx,
                       const dsa::BwdDqParams& dp, cudaStream_t s) {
  auto kernel = dsa::bwd_dq_kernel<kFlat, kExtra>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dsa::bdq::kSmemBytes) != cudaSuccess)
    return DSA_ERR_CUDA;
  // the kernel's setmaxnreg split needs exactly the registers it was compiled for at launch
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return DSA_ERR_CUDA;
  if (fa.numRegs < dsa::bdq::kRegsAtLaunch) return DSA_ERR_UNSUPPORTED;
  int sms = 0;
  if (sm_count(&sms) != DSA_OK) return DSA_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(dp.n_units < sms ? dp.n_units : sms);
  kernel<<<grid, dsa::bdq::kThreads, dsa::bdq::kSmemBytes, s>>>(tk, tv, tkx, tvx, dp);
  return launch_status();
}

// The backward of the window and key-tile-list forms: D = rowsum(dO * O), the key-major
// kernel for dK and dV over the inverse lists (row_ptr, q_tiles), and the query-major
// kernel for dQ over the forward's lists; no dQ accumulator, no atomics.
dsa_status_t launch_bwd_det(const dsa_problem_t* p, const Geom& g, const void* q, const void* k, const void* v,
                            const void* out, const float* lse, const void* dout, const int32_t* row_ptr,
                            const int32_t* q_tiles, int inv_head_stride, const FwdKeys& fk, float* delta, void* dq,
                            void* dk, void* dv, cudaStream_t s) {
  const int64_t rows = g.BH * g.N;
  dsa::bwd_preprocess<<<static_cast<unsigned>((rows * 16 + 255) / 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), delta, rows);
  dsa_status_t st = launch_status();
  if (st != DSA_OK) return st;
  CUtensorMap tq, tk, tv, tdo, tlse, tdel;
  if (!make_token_map(&tq, q, p, g, 64) || !make_token_map(&tk, k, p, g, 128) ||
      !make_token_map(&tv, v, p, g, 128) || !make_token_map(&tdo, dout, p, g, 64) ||
      !make_row_map(&tlse, lse, p, g, 64) || !make_row_map(&tdel, delta, p, g, 64))
    return DSA_ERR_CUDA;
  dsa::BwdBf16Params bp;
  std::memset(&bp, 0, sizeof(bp));
  bp.row_ptr = row_ptr;
  bp.rp_head_stride = inv_head_stride;
  bp.q_tiles = q_tiles;
  bp.dk = static_cast<__nv_bfloat16*>(dk);
  bp.dv = static_cast<__nv_bfloat16*>(dv);
  bp.n_tiles = g.n_tiles;
  bp.KU = g.tile_tokens / 128;
  bp.QS = g.tile_tokens / 64;
  bp.n_units = static_cast<int>(g.BH * g.n_tiles * bp.KU);
  bp.G1 = g.G[1];
  bp.G2 = g.G[2];
  bp.tt = p->tile[0];
  bp.th = p->tile[1];
  bp.tw = p->tile[2];
  bp.kcs = 128 / (p->tile[1] * p->tile[2]);
  bp.qcs = 64 / (p->tile[1] * p->tile[2]);
  bp.T = p->T;
  bp.H = p->H;
  bp.W = p->W;
  bp.N = static_cast<int>(g.N);
  bp.scale = p->scale;
  bp.scale_log2 = p->scale * 1.4426950408889634f;
  bp.n_split = 1;
  {
    auto kernel = dsa::bwd_bf16_kernel<false, false>;
    constexpr uint32_t smem = dsa::bwd::kSmemBytes;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return DSA_ERR_CUDA;
    int sms = 0;
    if (sm_count(&sms) != DSA_OK) return DSA_ERR_CUDA;
    const unsigned grid = static_cast<unsigned>(bp.n_units < sms ? bp.n_units : sms);
    kernel<<<grid, dsa::bwd::kThreads, smem, s>>>(tq, tk, tv, tdo, tlse, tdel, tq, tdo, tlse, tdel, bp);
    st = launch_status();
    if (st != DSA_OK) return st;
  }
  // dQ: 128-row query chunks over the forward's key lists, 128 keys per step (the K and V
  // maps of 128-token boxes serve both kernels)
  dsa::BwdDqParams dp = dq_params(p, g, lse, delta, dq);
  dp.q = static_cast<const __nv_bfloat16*>(q);
  dp.dout = static_cast<const __nv_bfloat16*>(dout);
  dp.kv_tiles = fk.kv;
  dp.row_ptr = fk.row_ptr;
  dp.rp_head_stride = fk.rp_head_stride;
  dp.nnz = fk.nnz;
  return launch_dq<false, false>(tk, tv, tk, tv, dp, s);
}

}  // namespace

extern "C" {

int32_t dsa_version(void) { return 100; }

const char* dsa_status_string(dsa_status_t s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported problem";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "device wait timed out";
    case DSA_ERR_WORKSPACE: return "workspace too small";
    case DSA_ERR_DEVICE: return "device bounds check failed";
  }
  return "unknown status";
}

dsa_status_t dsa_plan_shape(const dsa_problem_t* p, int32_t* n_tiles, int32_t* window_tiles) {
  Geom g;
  dsa_status_t st = check_shape(p, &g);
  if (st != DSA_OK) return st;
  if (n_tiles) *n_tiles = g.n_tiles;
  if (window_tiles) *window_tiles = g.Wt;
  return DSA_OK;
}

size_t dsa_workspace_size(const dsa_problem_t* p, int32_t kind) {
  Geom g;
  if (check_shape(p, &g) != DSA_OK) return 0;
  if (kind == DSA_WS_FWD) return fwd_workspace(g, nullptr).bytes;
  if (kind == DSA_WS_BWD) return bwd_workspace(g, nullptr).bytes;
  return 0;
}

dsa_status_t dsa_plan(const dsa_problem_t* p, const int32_t* tile_offsets, int32_t* starts, int32_t* kv_tiles,
                      int32_t* inv_row_ptr, int32_t* inv_q_tiles, void* stream) {
  Geom g;
  dsa_status_t st = check_shape(p, &g);
  if (st != DSA_OK) return st;
  if (!tile_offsets || !starts || !kv_tiles) return DSA_ERR_INVALID_ARG;
  if ((inv_row_ptr == nullptr) != (inv_q_tiles == nullptr)) return DSA_ERR_INVALID_ARG;
  return launch_plan(g, tile_offsets, starts, kv_tiles, inv_row_ptr, inv_q_tiles, static_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_fwd(const dsa_problem_t* p, const void* q, const void* k, const void* v,
                     const int32_t* tile_offsets, void* out, float* lse, void* workspace, size_t ws_bytes,
                     void* stream) {
  Geom g;
  dsa_status_t st = check_shape(p, &g);
  if (st != DSA_OK) return st;
  if (!q || !k || !v || !tile_offsets || !out || !lse) return DSA_ERR_INVALID_ARG;
  st = check_kernel_limits(p, g, false);
  if (st != DSA_OK) return st;
  const size_t elem_align = p->dtype == DSA_BF16 ? 16 : 4;
  if (!aligned(q, elem_align) || !aligned(k, elem_align) || !aligned(v, elem_align) || !aligned(out, elem_align) ||
      !aligned(lse, 4) || !aligned(tile_offsets, 4))
    return DSA_ERR_INVALID_ARG;
  FwdWorkspace ws = fwd_workspace(g, workspace);
  if (workspace == nullptr || ws_bytes < ws.bytes || !aligned(workspace, kAlign)) return DSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_plan(g, tile_offsets, ws.starts, ws.kv_tiles, nullptr, nullptr, s);
  if (st != DSA_OK) return st;
  return launch_fwd(p, g, q, k, v, ws.kv_tiles, out, lse, s);
}

namespace {
// Groups of (batch, head) slices the host-buffer forward pipelines over.
constexpr int64_t kHostGroups = 24;

// Internal streams and events of one host-buffer forward call, released when the call
// returns (the runtime keeps destroyed streams and events alive until their work is done).
struct HostPipeline {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, end = nullptr;
  cudaEvent_t ev_in[kHostGroups] = {}, ev_fwd[kHostGroups] = {};
  int n = 0;
  bool init(int groups) {
    n = groups;
    if (cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&start, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&end, cudaEventDisableTiming) != cudaSuccess)
      return false;
    for (int i = 0; i < n; ++i)
      if (cudaEventCreateWithFlags(&ev_in[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&ev_fwd[i], cudaEventDisableTiming) != cudaSuccess)
        return false;
    return true;
  }
  ~HostPipeline() {
    for (int i = 0; i < n; ++i) {
      if (ev_in[i]) cudaEventDestroy(ev_in[i]);
      if (ev_fwd[i]) cudaEventDestroy(ev_fwd[i]);
    }
    if (start) cudaEventDestroy(start);
    if (end) cudaEventDestroy(end);
    if (in) cudaStreamDestroy(in);
    if (out) cudaStreamDestroy(out);
  }
};
}  // namespace

size_t dsa_fwd_host_bytes(const dsa_problem_t* p) {
  Geom g;
  if (check_shape(p, &g) != DSA_OK) return 0;
  const size_t elem = p->dtype == DSA_BF16 ? 2 : 4;
  const size_t tok = static_cast<size_t>(g.BH * g.N) * p->d * elem;
  return 4 * round_up(tok, kAlign) + round_up(sizeof(float) * g.BH * g.N, kAlign) +
         round_up(sizeof(int32_t) * 3 * g.n_tiles, kAlign) + fwd_workspace(g, nullptr).bytes;
}

dsa_status_t dsa_fwd_host(const dsa_problem_t* p, const void* q_host, const void* k_host, const void* v_host,
                          const int32_t* tile_offsets_host, void* out_host, float* lse_host, void* dev,
                          size_t dev_bytes, void* stream) {
  Geom g;
  dsa_status_t st = check_shape(p, &g);
  if (st != DSA_OK) return st;
  if (!q_host || !k_host || !v_host || !tile_offsets_host || !out_host || !lse_host) return DSA_ERR_INVALID_ARG;
  st = check_kernel_limits(p, g, false);
  if (st != DSA_OK) return st;
  if (dev == nullptr || dev_bytes < dsa_fwd_host_bytes(p) || !aligned(dev, kAlign)) return DSA_ERR_WORKSPACE;
  const size_t elem = p->dtype == DSA_BF16 ? 2 : 4;
  const size_t tok = static_cast<size_t>(g.BH * g.N) * p->d * elem;
  const size_t lse_bytes = sizeof(float) * g.BH * g.N, off_bytes = sizeof(int32_t) * 3 * g.n_tiles;
  uint8_t* b = static_cast<uint8_t*>(dev);
  void* dq = b;
  void* dk = b + round_up(tok, kAlign);
  void* dv = b + 2 * round_up(tok, kAlign);
  void* dout = b + 3 * round_up(tok, kAlign);
  float* dlse = reinterpret_cast<float*>(b + 4 * round_up(tok, kAlign));
  int32_t* doff = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(dlse) + round_up(lse_bytes, kAlign));
  uint8_t* ws = reinterpret_cast<uint8_t*>(doff) + round_up(off_bytes, kAlign);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Pipelined over groups of (batch, head) slices, which are independent problems: the
  // host-to-device copies of group i + 1 run on one internal stream while the forward of
  // group i runs on the caller's stream and the copy back of group i - 1 on another, so
  // the two copy directions and the kernels overlap.  Events order each group's three
  // stages; the caller's stream waits for the last copy back before the call's end.
  const int64_t n_groups = g.BH < kHostGroups ? g.BH : kHostGroups;
  const int64_t per = (g.BH + n_groups - 1) / n_groups;
  const size_t head_tok = static_cast<size_t>(g.N) * p->d * elem, head_lse = sizeof(float) * g.N;
  HostPipeline pl;
  if (!pl.init(static_cast<int>(n_groups))) return DSA_ERR_CUDA;
  if (cudaEventRecord(pl.start, s) != cudaSuccess || cudaStreamWaitEvent(pl.in, pl.start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(pl.out, pl.start, 0) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (cudaMemcpyAsync(doff, tile_offsets_host, off_bytes, cudaMemcpyHostToDevice, pl.in) != cudaSuccess)
    return DSA_ERR_CUDA;
  for (int64_t gi = 0; gi < n_groups; ++gi) {
    const int64_t h0 = gi * per, cnt = (h0 + per <= g.BH ? per : g.BH - h0);
    if (cnt <= 0) break;
    const size_t o_tok = static_cast<size_t>(h0) * head_tok, o_lse = static_cast<size_t>(h0) * head_lse;
    const size_t n_tok = static_cast<size_t>(cnt) * head_tok, n_lse = static_cast<size_t>(cnt) * head_lse;
    const uint8_t* qh = static_cast<const uint8_t*>(q_host) + o_tok;
    const uint8_t* kh = static_cast<const uint8_t*>(k_host) + o_tok;
    const uint8_t* vh = static_cast<const uint8_t*>(v_host) + o_tok;
    uint8_t *qd = static_cast<uint8_t*>(dq) + o_tok, *kd = static_cast<uint8_t*>(dk) + o_tok,
            *vd = static_cast<uint8_t*>(dv) + o_tok, *od = static_cast<uint8_t*>(dout) + o_tok;
    float* ld = dlse + static_cast<size_t>(h0) * g.N;
    if (cudaMemcpyAsync(qd, qh, n_tok, cudaMemcpyHostToDevice, pl.in) != cudaSuccess ||
        cudaMemcpyAsync(kd, kh, n_tok, cudaMemcpyHostToDevice, pl.in) != cudaSuccess ||
        cudaMemcpyAsync(vd, vh, n_tok, cudaMemcpyHostToDevice, pl.in) != cudaSuccess ||
        cudaEventRecord(pl.ev_in[gi], pl.in) != cudaSuccess || cudaStreamWaitEvent(s, pl.ev_in[gi], 0) != cudaSuccess)
      return DSA_ERR_CUDA;
    dsa_problem_t sub = *p;
    sub.B = 1;
    sub.heads = static_cast<int32_t>(cnt);
    st = dsa_fwd(&sub, qd, kd, vd, doff, od, ld, ws, fwd_workspace(g, nullptr).bytes, stream);
    if (st != DSA_OK) return st;
    if (cudaEventRecord(pl.ev_fwd[gi], s) != cudaSuccess || cudaStreamWaitEvent(pl.out, pl.ev_fwd[gi], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t*>(out_host) + o_tok, od, n_tok, cudaMemcpyDeviceToHost, pl.out) !=
            cudaSuccess ||
        cudaMemcpyAsync(reinterpret_cast<uint8_t*>(lse_host) + o_lse, ld, n_lse, cudaMemcpyDeviceToHost, pl.out) !=
            cudaSuccess)
      return DSA_ERR_CUDA;
  }
  if (cudaEventRecord(pl.end, pl.out) != cudaSuccess || cudaStreamWaitEvent(s, pl.end, 0) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t dsa_bwd(const dsa_problem_t* p, const void* q, const void* k, const void* v, const void* out,
                     const float* lse, const void* dout, const int32_t* tile_offsets, void* dq, void* dk, void* dv,
                     void* workspace, size_t ws_bytes, void* stream) {
  Geom g;
  dsa_status_t st = check_shape(p, &g);
  if (st != DSA_OK) return st;
  if (!q || !k || !v || !out || !lse || !dout || !tile_offsets || !dq || !dk || !dv) return DSA_ERR_INVALID_ARG;
  st = check_kernel_limits(p, g, true);
  if (st != DSA_OK) return st;
  const void* ptrs[] = {q, k, v, out, dout, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!aligned(ptr, 16)) return DSA_ERR_INVALID_ARG;
  if (!aligned(lse, 4) || !aligned(tile_offsets, 4)) return DSA_ERR_INVALID_ARG;
  BwdWorkspace ws = bwd_workspace(g, workspace);
  if (workspace == nullptr || ws_bytes < ws.bytes || !aligned(workspace, kAlign)) return DSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_plan(g, tile_offsets, ws.starts, ws.kv_tiles, ws.row_ptr, ws.q_tiles, s);
  if (st != DSA_OK) return st;
  return launch_bwd_det(p, g, q, k, v, out, lse, dout, ws.row_ptr, ws.q_tiles, 0, FwdKeys{ws.kv_tiles, nullptr, 0, 0},
                        ws.delta, dq, dk, dv, s);
}

size_t dsa_list_workspace_size(const dsa_problem_t* p, int32_t nnz, int32_t per_head, int32_t kind) {
  Geom g;
  if (check_shape(p, &g) != DSA_OK || nnz < 0) return 0;
  if (kind == DSA_WS_FWD) return 0;
  if (kind == DSA_WS_BWD) return list_bwd_workspace(g, nnz, per_head ? static_cast<int>(g.BH) : 1, nullptr).bytes;
  return 0;
}

dsa_status_t dsa_plan_heads(const dsa_problem_t* p, const int32_t* tile_offsets, int32_t* kv_row_ptr, int32_t* kv_list,
                            void* stream) {
  Geom g;
  dsa_status_t st = check_shape(p, &g);
  if (st != DSA_OK) return st;
  if (!tile_offsets || !kv_row_ptr || !kv_list) return DSA_ERR_INVALID_ARG;
  if (g.BH > 65535 || g.BH * g.n_tiles * static_cast<int64_t>(g.Wt) > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (!aligned(tile_offsets, 4) || !aligned(kv_row_ptr, 4) || !aligned(kv_list, 4)) return DSA_ERR_INVALID_ARG;
  dsa::plan_heads_kernel<<<static_cast<unsigned>(g.BH), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      plan_geom(g), tile_offsets, kv_row_ptr, kv_list);
  return launch_status();
}

namespace {
// Argument checks shared by the list entry points; n_lists = 1 or B*heads.
dsa_status_t check_lists(const Geom& g, const int32_t* kv_row_ptr, const int32_t* kv_list, int32_t nnz,
                         int32_t per_head, int* n_lists) {
  if (!kv_row_ptr || nnz < 0 || (nnz > 0 && !kv_list) || (per_head != 0 && per_head != 1)) return DSA_ERR_INVALID_ARG;
  if (!aligned(kv_row_ptr, 4) || (kv_list && !aligned(kv_list, 4))) return DSA_ERR_INVALID_ARG;
  *n_lists = per_head ? static_cast<int>(g.BH) : 1;
  if (static_cast<int64_t>(*n_lists) * (g.n_tiles + 1) > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}
}  // namespace

dsa_status_t dsa_fwd_list(const dsa_problem_t* p, const void* q, const void* k, const void* v,
                          const int32_t* kv_row_ptr, const int32_t* kv_list, int32_t nnz, int32_t per_head, void* out,
                          float* lse, void* stream) {
  Geom g;
  dsa_status_t st = check_shape(p, &g);
  if (st != DSA_OK) return st;
  if (!q || !k || !v || !out || !lse) return DSA_ERR_INVALID_ARG;
  int n_lists = 1;
  st = check_lists(g, kv_row_ptr, kv_list, nnz, per_head, &n_lists);
  if (st != DSA_OK) return st;
  if (p->dtype != DSA_BF16) return DSA_ERR_UNSUPPORTED;
  st = check_kernel_limits(p, g, false);
  if (st != DSA_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4))
    return DSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_list_check(g, kv_row_ptr, kv_list, n_lists, nnz, s);
  if (st != DSA_OK) return st;
  return launch_fwd(p, g, q, k, v, kv_list, out, lse, s, kv_row_ptr, nnz, per_head ? g.n_tiles + 1 : 0);
}

dsa_status_t dsa_bwd_list(const dsa_problem_t* p, const void* q, const void* k, const void* v, const void* out,
                          const float* lse, const void* dout, const int32_t* kv_row_ptr, const int32_t* kv_list,
                          int32_t nnz, int32_t per_head, void* dq, void* dk, void* dv, void* workspace,
                          size_t ws_bytes, void* stream) {
  Geom g;
  dsa_status_t st = check_shape(p, &g);
  if (st != DSA_OK) return st;
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv) return DSA_ERR_INVALID_ARG;
  int n_lists = 1;
  st = check_lists(g, kv_row_ptr, kv_list, nnz, per_head, &n_lists);
  if (st != DSA_OK) return st;
  st = check_kernel_limits(p, g, true);
  if (st != DSA_OK) return st;
  const void* ptrs[] = {q, k, v, out, dout, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!aligned(ptr, 16)) return DSA_ERR_INVALID_ARG;
  if (!aligned(lse, 4)) return DSA_ERR_INVALID_ARG;
  ListBwdWorkspace ws = list_bwd_workspace(g, nnz, n_lists, workspace);
  if (workspace == nullptr || ws_bytes < ws.bytes || !aligned(workspace, kAlign)) return DSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_list_check(g, kv_row_ptr, kv_list, n_lists, nnz, s);
  if (st != DSA_OK) return st;
  dsa::invert_lists_kernel<<<static_cast<unsigned>(n_lists), 1024, 0, s>>>(kv_row_ptr, kv_list, g.n_tiles, nnz,
                                                                           ws.counts, ws.row_ptr, ws.q_tiles);
  st = launch_status();
  if (st != DSA_OK) return st;
  const int stride = per_head ? g.n_tiles + 1 : 0;
  return launch_bwd_det(p, g, q, k, v, out, lse, dout, ws.row_ptr, ws.q_tiles, stride,
                        FwdKeys{kv_list, kv_row_ptr, nnz, stride}, ws.delta, dq, dk, dv, s);
}

dsa_status_t dsa_block_map(const dsa_problem_t* p, const void* q, const void* k, const float* lse,
                           const int32_t* kv_row_ptr, const int32_t* kv_list, int32_t nnz, int32_t per_head, float* map,
                           void* stream) {
  Geom g;
  dsa_status_t st = check_shape(p, &g);
  if (st != DSA_OK) return st;
  if (!q || !k || !lse || !map) return DSA_ERR_INVALID_ARG;
  int n_lists = 1;
  st = check_lists(g, kv_row_ptr, kv_list, nnz, per_head, &n_lists);
  if (st != DSA_OK) return st;
  if (p->dtype != DSA_BF16) return DSA_ERR_UNSUPPORTED;
  st = check_kernel_limits(p, g, false);
  if (st != DSA_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(lse, 4) || !aligned(map, 4)) return DSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t map_bytes = sizeof(float) * static_cast<size_t>(g.BH) * g.n_tiles * g.n_tiles;
  if (cudaMemsetAsync(map, 0, map_bytes, s) != cudaSuccess) return DSA_ERR_CUDA;
  st = launch_list_check(g, kv_row_ptr, kv_list, n_lists, nnz, s);
  if (st != DSA_OK) return st;
  // map mode reads no V (its tensor map is given K's) and writes no O or LSE
  return launch_fwd(p, g, q, k, k, kv_list, nullptr, nullptr, s, kv_row_ptr, nnz, per_head ? g.n_tiles + 1 : 0, lse,
                    map);
}

size_t dsa_lstsq_workspace_size(int32_t m, int32_t p, int32_t batch) {
  (void)m;
  (void)p;
  (void)batch;
  return 0;  // the solve keeps its partial sums in shared memory
}

dsa_status_t dsa_lstsq_factor(int32_t m, int32_t p, const float* M, float lambda, double* L, void* stream) {
  if (m <= 0 || p <= 0 || !M || !L || !(lambda >= 0.f) || !std::isfinite(lambda)) return DSA_ERR_INVALID_ARG;
  if (p > dsa::kLstsqMaxP) return DSA_ERR_UNSUPPORTED;
  if (!aligned(M, 4) || !aligned(L, 8)) return DSA_ERR_INVALID_ARG;
  dsa::lstsq_factor_kernel<<<1, 256, 0, static_cast<cudaStream_t>(stream)>>>(M, m, p, lambda, L);
  return launch_status();
}

dsa_status_t dsa_lstsq_solve(int32_t m, int32_t p, int32_t batch, const float* M, const double* L, const float* S,
                             float* X, void* workspace, size_t ws_bytes, void* stream) {
  (void)workspace;
  (void)ws_bytes;
  if (m <= 0 || p <= 0 || batch <= 0 || !M || !L || !S || !X) return DSA_ERR_INVALID_ARG;
  if (p > dsa::kLstsqMaxP || batch > 65535) return DSA_ERR_UNSUPPORTED;
  if (!aligned(M, 4) || !aligned(L, 8) || !aligned(S, 4) || !aligned(X, 4)) return DSA_ERR_INVALID_ARG;
  // one cluster of kLstsqCluster CTAs per right-hand side (the cluster shape is compiled in)
  dim3 grid(dsa::kLstsqCluster, static_cast<unsigned>(batch));
  dsa::lstsq_solve_kernel<<<grid, dsa::kLstsqThreads, 0, static_cast<cudaStream_t>(stream)>>>(M, S, m, p, L, X);
  return launch_status();
}

namespace {
// Parts the text queries' key sequence (every video token) is cut into: enough units for
// about four waves of persistent CTAs, at most one part per 128-key chunk.
int prefix_split(const Geom& g, int32_t L_text) {
  const int64_t units = g.BH * ((static_cast<int64_t>(L_text) + 127) / 128);
  const int64_t n_main = (g.N + 127) / 128;
  int64_t n = (4 * 148 + units - 1) / (units > 0 ? units : 1);
  if (n > n_main) n = n_main;
  if (n > 16) n = 16;
  return static_cast<int>(n < 1 ? 1 : n);
}

struct PrefixWorkspace {
  int32_t* starts;
  int32_t* kv_tiles;
  void* o_parts;   // [n_split][BH, L_text, 128] bf16 (n_split > 1 only)
  float* l_parts;  // [n_split][BH, L_text] fp32
  int n_split;
  size_t bytes;
};

PrefixWorkspace prefix_workspace(const Geom& g, int32_t L_text, void* base) {
  PrefixWorkspace w;
  FwdWorkspace f = fwd_workspace(g, base);
  w.starts = f.starts;
  w.kv_tiles = f.kv_tiles;
  w.n_split = prefix_split(g, L_text);
  size_t off = f.bytes;
  const size_t rows = static_cast<size_t>(g.BH) * (L_text > 0 ? L_text : 0);
  uint8_t* b = static_cast<uint8_t*>(base);
  w.o_parts = b ? b + off : nullptr;
  if (w.n_split > 1) off += round_up(sizeof(__nv_bfloat16) * rows * 128 * w.n_split, kAlign);
  w.l_parts = b ? reinterpret_cast<float*>(b + off) : nullptr;
  if (w.n_split > 1) off += round_up(sizeof(float) * rows * w.n_split, kAlign);
  w.bytes = off;
  return w;
}
}  // namespace

size_t dsa_prefix_workspace_size(const dsa_problem_t* p, int32_t L_text) {
  Geom g;
  if (check_shape(p, &g) != DSA_OK || L_text < 0) return 0;
  return prefix_workspace(g, L_text, nullptr).bytes;
}

dsa_status_t dsa_fwd_prefix(const dsa_problem_t* p, const void* q, const void* k, const void* v,
                            const int32_t* tile_offsets, int32_t L_text, const void* q_text, const void* k_text,
                            const void* v_text, void* out, float* lse, void* out_text, float* lse_text,
                            void* workspace, size_t ws_bytes, void* stream) {
  Geom g;
  dsa_status_t st = check_shape(p, &g);
  if (st != DSA_OK) return st;
  if (!q || !k || !v || !tile_offsets || !out || !lse || L_text < 0) return DSA_ERR_INVALID_ARG;
  if (L_text > 0 && (!q_text || !k_text || !v_text || !out_text || !lse_text)) return DSA_ERR_INVALID_ARG;
  if (p->dtype != DSA_BF16) return DSA_ERR_UNSUPPORTED;
  st = check_kernel_limits(p, g, false);
  if (st != DSA_OK) return st;
  if (g.BH * ((static_cast<int64_t>(L_text) + 127) / 128) * 16 > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, out, q_text, k_text, v_text, out_text};
  for (const void* ptr : ptrs)
    if (ptr && !aligned(ptr, 16)) return DSA_ERR_INVALID_ARG;
  if (!aligned(lse, 4) || (lse_text && !aligned(lse_text, 4)) || !aligned(tile_offsets, 4)) return DSA_ERR_INVALID_ARG;
  if (workspace == nullptr || ws_bytes < prefix_workspace(g, L_text, nullptr).bytes || !aligned(workspace, kAlign))
    return DSA_ERR_WORKSPACE;
  const PrefixWorkspace ws = prefix_workspace(g, L_text, workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // video queries: their windows, then every text key, in one softmax
  st = launch_plan(g, tile_offsets, ws.starts, ws.kv_tiles, nullptr, nullptr, s);
  if (st != DSA_OK) return st;
  st = launch_fwd(p, g, q, k, v, ws.kv_tiles, out, lse, s, nullptr, 0, 0, nullptr, nullptr, k_text, v_text, L_text);
  if (st != DSA_OK || L_text == 0) return st;
  // text queries: every video key (the video tensor in raster order is a flat sequence of N
  // rows), cut into parts for load balance, then every text key (with part 0)
  const int N = static_cast<int>(g.N);
  const int64_t rows = g.BH * L_text;
  if (ws.n_split == 1)
    return launch_flat(q_text, k, v, k_text, v_text, g.BH, L_text, N, L_text, 1, p->scale, out_text, lse_text, 0, 0,
                       s);
  st = launch_flat(q_text, k, v, k_text, v_text, g.BH, L_text, N, L_text, ws.n_split, p->scale, ws.o_parts,
                   ws.l_parts, rows * 128, rows, s);
  if (st != DSA_OK) return st;
  return launch_merge_parts(ws.o_parts, ws.l_parts, ws.n_split, rows * 128, rows, rows, out_text, lse_text, s);
}

namespace {
// Parts the query chunks of the text keys' backward are cut into: enough units for about
// four waves of persistent CTAs, at most one part per 64-query chunk of the video.
int prefix_bwd_split(const Geom& g, int32_t L_text) {
  const int64_t units = g.BH * ((static_cast<int64_t>(L_text) + 127) / 128);
  const int64_t nqm = (g.N + 63) / 64;
  int64_t n = (4 * 148 + units - 1) / (units > 0 ? units : 1);
  if (n > nqm) n = nqm;
  if (n > 16) n = 16;
  return static_cast<int>(n < 1 ? 1 : n);
}

// Parts the text queries' dQ is cut into over the video keys: enough units for about four
// waves of persistent CTAs, at most one part per 64-key chunk of the video.
int prefix_dq_split(const Geom& g, int32_t L_text) {
  const int64_t units = g.BH * ((static_cast<int64_t>(L_text) + 127) / 128);
  const int64_t nk = (g.N + 127) / 128;
  int64_t n = (4 * 148 + units - 1) / (units > 0 ? units : 1);
  if (n > nk) n = nk;
  if (n > 16) n = 16;
  return static_cast<int>(n < 1 ? 1 : n);
}

struct PrefixBwdWorkspace {
  BwdWorkspace video;
  float* lse_pad;    // [BH, Lp] text LSE, zeros past L
  float* delta_pad;  // [BH, Lp] text D
  float* dk_part;    // [n_split][BH, L, 128] fp32: the text keys' dK, dV per part of the queries
  float* dv_part;
  float* dq_part;    // [n_split_q][BH, L, 128] fp32: the text queries' dQ per part of the keys
  int Lp, n_split, n_split_q;
  size_t bytes;
};

PrefixBwdWorkspace prefix_bwd_workspace(const Geom& g, int32_t L, void* base) {
  PrefixBwdWorkspace w;
  w.video = bwd_workspace(g, base);
  uint8_t* b = static_cast<uint8_t*>(base);
  size_t off = w.video.bytes;
  w.Lp = (L + 63) / 64 * 64;
  w.n_split = prefix_bwd_split(g, L);
  w.n_split_q = prefix_dq_split(g, L);
  const size_t rows = static_cast<size_t>(g.BH) * L, rows_p = static_cast<size_t>(g.BH) * w.Lp;
  auto take = [&](size_t bytes) {
    float* ptr = b ? reinterpret_cast<float*>(b + off) : nullptr;
    off += round_up(bytes, kAlign);
    return ptr;
  };
  w.lse_pad = take(sizeof(float) * rows_p);
  w.delta_pad = take(sizeof(float) * rows_p);
  w.dk_part = take(sizeof(float) * rows * 128 * w.n_split);
  w.dv_part = take(sizeof(float) * rows * 128 * w.n_split);
  w.dq_part = take(sizeof(float) * rows * 128 * w.n_split_q);
  w.bytes = off;
  return w;
}
}  // namespace

size_t dsa_bwd_prefix_workspace_size(const dsa_problem_t* p, int32_t L_text) {
  Geom g;
  if (check_shape(p, &g) != DSA_OK || L_text < 0) return 0;
  return prefix_bwd_workspace(g, L_text, nullptr).bytes;
}

dsa_status_t dsa_bwd_prefix(const dsa_problem_t* p, const void* q, const void* k, const void* v, const void* out,
                            const float* lse, const void* dout, const int32_t* tile_offsets, int32_t L_text,
                            const void* q_text, const void* k_text, const void* v_text, const void* out_text,
                            const float* lse_text, const void* dout_text, void* dq, void* dk, void* dv,
                            void* dq_text, void* dk_text, void* dv_text, void* workspace, size_t ws_bytes,
                            void* stream) {
  Geom g;
  dsa_status_t st = check_shape(p, &g);
  if (st != DSA_OK) return st;
  if (!q || !k || !v || !out || !lse || !dout || !tile_offsets || !dq || !dk || !dv || L_text < 0)
    return DSA_ERR_INVALID_ARG;
  if (L_text > 0 && (!q_text || !k_text || !v_text || !out_text || !lse_text || !dout_text || !dq_text || !dk_text ||
                     !dv_text))
    return DSA_ERR_INVALID_ARG;
  if (p->dtype != DSA_BF16) return DSA_ERR_UNSUPPORTED;
  st = check_kernel_limits(p, g, true);
  if (st != DSA_OK) return st;
  if (g.BH * ((static_cast<int64_t>(L_text) + 127) / 128) * 16 > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, out, dout, dq, dk, dv, q_text, k_text, v_text, out_text, dout_text, dq_text, dk_text,
                        dv_text};
  for (const void* ptr : ptrs)
    if (ptr && !aligned(ptr, 16)) return DSA_ERR_INVALID_ARG;
  if (!aligned(lse, 4) || (lse_text && !aligned(lse_text, 4)) || !aligned(tile_offsets, 4)) return DSA_ERR_INVALID_ARG;
  if (workspace == nullptr || ws_bytes < prefix_bwd_workspace(g, L_text, nullptr).bytes || !aligned(workspace, kAlign))
    return DSA_ERR_WORKSPACE;
  const PrefixBwdWorkspace ws = prefix_bwd_workspace(g, L_text, workspace);
  const BwdWorkspace& wv = ws.video;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_plan(g, tile_offsets, wv.starts, wv.kv_tiles, wv.row_ptr, wv.q_tiles, s);
  if (st != DSA_OK) return st;
  if (L_text == 0)
    return launch_bwd_det(p, g, q, k, v, out, lse, dout, wv.row_ptr, wv.q_tiles, 0,
                          FwdKeys{wv.kv_tiles, nullptr, 0, 0}, wv.delta, dq, dk, dv, s);
  // Every gradient is summed in one CTA in a fixed order (no atomics), as in dsa_bwd:
  //   video keys (dK, dV): the key-major kernel over their windows' queries and every text query;
  //   text keys: the same kernel in the flat-key mode over every video and text query, in parts
  //     whose fp32 sums are added in part order;
  //   video queries (dQ): the query-major kernel over their windows' keys and every text key;
  //   text queries: the query-major kernel in the flat mode over every video key, in parts,
  //     and every text key, the parts' fp32 sums added in part order.
  const int64_t rows = g.BH * g.N;
  dsa::bwd_preprocess<<<static_cast<unsigned>((rows * 16 + 255) / 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), wv.delta, rows);
  st = launch_status();
  if (st != DSA_OK) return st;
  const int64_t prow = g.BH * ws.Lp;
  dsa::bwd_preprocess_flat<<<static_cast<unsigned>((prow * 16 + 255) / 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(out_text), static_cast<const __nv_bfloat16*>(dout_text), lse_text,
      ws.delta_pad, ws.lse_pad, L_text, ws.Lp, g.BH);
  st = launch_status();
  if (st != DSA_OK) return st;
  CUtensorMap tq, tk, tv, tdo, tlse, tdel, tqx, tdox, tlsex, tdx;
  if (!make_token_map(&tq, q, p, g, 64) || !make_token_map(&tk, k, p, g, 128) ||
      !make_token_map(&tv, v, p, g, 128) || !make_token_map(&tdo, dout, p, g, 64) ||
      !make_row_map(&tlse, lse, p, g, 64) || !make_row_map(&tdel, wv.delta, p, g, 64) ||
      !make_flat_map(&tqx, q_text, g.BH, L_text, 64) || !make_flat_map(&tdox, dout_text, g.BH, L_text, 64) ||
      !make_vec_map(&tlsex, ws.lse_pad, g.BH, ws.Lp) || !make_vec_map(&tdx, ws.delta_pad, g.BH, ws.Lp))
    return DSA_ERR_CUDA;
  // video keys
  dsa::BwdBf16Params bp;
  std::memset(&bp, 0, sizeof(bp));
  bp.row_ptr = wv.row_ptr;
  bp.q_tiles = wv.q_tiles;
  bp.dk = static_cast<__nv_bfloat16*>(dk);
  bp.dv = static_cast<__nv_bfloat16*>(dv);
  bp.n_tiles = g.n_tiles;
  bp.KU = g.tile_tokens / 128;
  bp.QS = g.tile_tokens / 64;
  bp.n_units = static_cast<int>(g.BH * g.n_tiles * bp.KU);
  bp.G1 = g.G[1];
  bp.G2 = g.G[2];
  bp.tt = p->tile[0];
  bp.th = p->tile[1];
  bp.tw = p->tile[2];
  bp.kcs = 128 / (p->tile[1] * p->tile[2]);
  bp.qcs = 64 / (p->tile[1] * p->tile[2]);
  bp.T = p->T;
  bp.H = p->H;
  bp.W = p->W;
  bp.N = static_cast<int>(g.N);
  bp.scale = p->scale;
  bp.scale_log2 = p->scale * 1.4426950408889634f;
  bp.Lxq = L_text;
  bp.n_split = 1;
  {
    auto kernel = dsa::bwd_bf16_kernel<false, true>;
    constexpr uint32_t smem = dsa::bwd::kSmemBytes;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return DSA_ERR_CUDA;
    int sms = 0;
    if (sm_count(&sms) != DSA_OK) return DSA_ERR_CUDA;
    const unsigned grid = static_cast<unsigned>(bp.n_units < sms ? bp.n_units : sms);
    kernel<<<grid, dsa::bwd::kThreads, smem, s>>>(tq, tk, tv, tdo, tlse, tdel, tqx, tdox, tlsex, tdx, bp);
    st = launch_status();
    if (st != DSA_OK) return st;
  }
  // text keys: every video query chunk (the video as flat rows), in parts, then every text
  // query chunk; fp32 partial dK, dV per part
  {
    CUtensorMap fq, fk, fv, fdo, flse, fdel;
    if (!make_flat_map(&fq, q, g.BH, g.N, 64) || !make_flat_map(&fk, k_text, g.BH, L_text, 128) ||
        !make_flat_map(&fv, v_text, g.BH, L_text, 128) || !make_flat_map(&fdo, dout, g.BH, g.N, 64) ||
        !make_vec_map(&flse, lse, g.BH, g.N) || !make_vec_map(&fdel, wv.delta, g.BH, g.N))
      return DSA_ERR_CUDA;
    dsa::BwdBf16Params fp;
    std::memset(&fp, 0, sizeof(fp));
    fp.N = static_cast<int>(g.N);
    fp.scale = p->scale;
    fp.scale_log2 = p->scale * 1.4426950408889634f;
    fp.Lxq = L_text;
    fp.Lk = L_text;
    fp.Nq = static_cast<int>(g.N);
    fp.n_split = ws.n_split;
    fp.dk_part = ws.dk_part;
    fp.dv_part = ws.dv_part;
    fp.part_stride = g.BH * static_cast<int64_t>(L_text) * 128;
    fp.n_units = static_cast<int>(g.BH * ((L_text + 127) / 128) * ws.n_split);
    fp.tt = fp.th = fp.tw = 1;  // no tile geometry in the flat-key mode
    fp.T = fp.H = fp.W = 1;
    auto kernel = dsa::bwd_bf16_kernel<true, true>;
    constexpr uint32_t smem = dsa::bwd::kSmemBytes;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return DSA_ERR_CUDA;
    int sms = 0;
    if (sm_count(&sms) != DSA_OK) return DSA_ERR_CUDA;
    const unsigned grid = static_cast<unsigned>(fp.n_units < sms ? fp.n_units : sms);
    kernel<<<grid, dsa::bwd::kThreads, smem, s>>>(fq, fk, fv, fdo, flse, fdel, tqx, tdox, tlsex, tdx, fp);
    st = launch_status();
    if (st != DSA_OK) return st;
    const int64_t n4 = g.BH * static_cast<int64_t>(L_text) * 128 / 4;
    dsa::bwd_kv_combine<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, s>>>(
        ws.dk_part, ws.dv_part, ws.n_split, fp.part_stride, p->scale, n4, static_cast<__nv_bfloat16*>(dk_text),
        static_cast<__nv_bfloat16*>(dv_text));
    st = launch_status();
    if (st != DSA_OK) return st;
  }
  // video queries: dQ over their windows' keys and every text key
  {
    CUtensorMap tk2, tv2, tkx, tvx;
    if (!make_token_map(&tk2, k, p, g, 128) || !make_token_map(&tv2, v, p, g, 128) ||
        !make_flat_map(&tkx, k_text, g.BH, L_text, 128) || !make_flat_map(&tvx, v_text, g.BH, L_text, 128))
      return DSA_ERR_CUDA;
    dsa::BwdDqParams dp = dq_params(p, g, lse, wv.delta, dq);
    dp.q = static_cast<const __nv_bfloat16*>(q);
    dp.dout = static_cast<const __nv_bfloat16*>(dout);
    dp.kv_tiles = wv.kv_tiles;
    dp.Lx = L_text;
    st = launch_dq<false, true>(tk2, tv2, tkx, tvx, dp, s);
    if (st != DSA_OK) return st;
  }
  // text queries: dQ over every video key (flat, in parts) and every text key (with part 0)
  {
    CUtensorMap fk, fv, tkx, tvx;
    if (!make_flat_map(&fk, k, g.BH, g.N, 128) || !make_flat_map(&fv, v, g.BH, g.N, 128) ||
        !make_flat_map(&tkx, k_text, g.BH, L_text, 128) || !make_flat_map(&tvx, v_text, g.BH, L_text, 128))
      return DSA_ERR_CUDA;
    dsa::BwdDqParams dp;
    std::memset(&dp, 0, sizeof(dp));
    dp.q = static_cast<const __nv_bfloat16*>(q_text);
    dp.dout = static_cast<const __nv_bfloat16*>(dout_text);
    dp.lse = ws.lse_pad;
    dp.delta = ws.delta_pad;
    dp.ld_rows = ws.Lp;
    dp.Lq = L_text;
    dp.Lk = static_cast<int>(g.N);
    dp.Lx = L_text;
    dp.n_split = ws.n_split_q;
    dp.dq_part = ws.dq_part;
    dp.part_stride = g.BH * static_cast<int64_t>(L_text) * 128;
    dp.n_units = static_cast<int>(g.BH * ((L_text + 127) / 128) * ws.n_split_q);
    dp.scale = p->scale;
    dp.scale_log2 = p->scale * 1.4426950408889634f;
    dp.tt = dp.th = dp.tw = 1;
    dp.T = dp.H = dp.W = 1;
    dp.S = dp.KS = 1;
    st = launch_dq<true, true>(fk, fv, tkx, tvx, dp, s);
    if (st != DSA_OK) return st;
    const int64_t n8 = g.BH * static_cast<int64_t>(L_text) * 128 / 8;
    dsa::dq_parts_combine<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, s>>>(
        ws.dq_part, ws.n_split_q, dp.part_stride, n8, static_cast<__nv_bfloat16*>(dq_text));
    return launch_status();
  }
}

dsa_status_t dsa_selftest_wait(void* stream) {
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(DSA_SELFTEST_SITE);
  return launch_status();
}

dsa_status_t dsa_device_status(void* stream, int32_t* site, int32_t* block) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int h[4] = {0, 0, 0, 0};
  const int zero[4] = {0, 0, 0, 0};
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(h, dsa::g_status, sizeof(h)) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemcpyToSymbol(dsa::g_status, zero, sizeof(zero)) != cudaSuccess) return DSA_ERR_CUDA;
  if (site) *site = h[1];
  if (block) *block = h[2];
  if (h[0] == dsa::DSA_DEV_TIMEOUT) return DSA_ERR_TIMEOUT;
  if (h[0] == dsa::DSA_DEV_BOUNDS) return DSA_ERR_DEVICE;
  return DSA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Forward for callers that cannot allocate device memory.
//
// Some callers have no way to give this library a workspace: a plugin hosted by an
// inference engine that owns every byte of device memory and hands its plugins none, a
// latency-critical loop that must not call cudaMalloc because it can synchronize the
// whole device, or a process whose memory budget is fixed when it starts.  For them the
// planner's scratch (window starts and key-tile lists) lives in the fixed array below,
// which every GPU that loads this library holds until the process exits.
namespace {

constexpr int kNoAllocPlanInts = 65536;  // 256 KB: 3 starts + Wt key tiles per query tile
static __device__ __align__(256) int32_t g_noalloc_plan[kNoAllocPlanInts];

constexpr int kNoAllocMaxDevices = 128;
struct NoAllocAddr {
  void* ctx;       // the context the address was looked up in
  int32_t* addr;   // device address of g_noalloc_plan in that context
};
NoAllocAddr g_noalloc_addr[kNoAllocMaxDevices];
std::mutex g_noalloc_mutex;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The driver's cuCtxGetCurrent, looked up once through the runtime (no libcuda link).
CtxGetCurrentFn ctx_get_current_fn() {
  static const CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(ptr);
    return nullptr;
  }();
  return fn;
}

void* current_context() {
  CtxGetCurrentFn fn = ctx_get_current_fn();
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_noalloc_plan on the current device.  In host code the array's name
// is only a host-side stand-in, so the address is looked up with the device current and
// cached per device, together with the context it belongs to: if the device's context
// has changed since (cudaDeviceReset, then a new primary context, into which the module
// may load elsewhere), the address is looked up again.
dsa_status_t noalloc_plan_address(int32_t** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return DSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoAllocAddr& e = g_noalloc_addr[dev];
  void* ctx = current_context();
  if (e.addr == nullptr || ctx == nullptr || ctx != e.ctx) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_plan) != cudaSuccess || ptr == nullptr) return DSA_ERR_CUDA;
    e.addr = static_cast<int32_t*>(ptr);
    e.ctx = current_context();  // the lookup makes the device's primary context current
  }
  *addr = e.addr;
  return DSA_OK;
}

}  // namespace

extern "C" dsa_status_t dsa_fwd_noalloc(const dsa_problem_t* p, const void* q, const void* k, const void* v,
                                        const int32_t* tile_offsets, void* out, float* lse, void* stream) {
  Geom g;
  dsa_status_t st = check_shape(p, &g);
  if (st != DSA_OK) return st;
  if (!q || !k || !v || !tile_offsets || !out || !lse) return DSA_ERR_INVALID_ARG;
  st = check_kernel_limits(p, g, false);
  if (st != DSA_OK) return st;
  const size_t elem_align = p->dtype == DSA_BF16 ? 16 : 4;
  if (!aligned(q, elem_align) || !aligned(k, elem_align) || !aligned(v, elem_align) || !aligned(out, elem_align) ||
      !aligned(lse, 4) || !aligned(tile_offsets, 4))
    return DSA_ERR_INVALID_ARG;
  // starts first, then the key-tile lists on a 256-byte boundary
  const int64_t starts_ints = (3 * static_cast<int64_t>(g.n_tiles) + 63) / 64 * 64;
  const int64_t need = starts_ints + static_cast<int64_t>(g.n_tiles) * g.Wt;
  if (need > kNoAllocPlanInts) return DSA_ERR_UNSUPPORTED;
  int32_t* plan = nullptr;
  st = noalloc_plan_address(&plan);
  if (st != DSA_OK) return st;
  // The planner writes every entry the forward reads, so nothing left from an earlier
  // call needs clearing.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_plan(g, tile_offsets, plan, plan + starts_ints, nullptr, nullptr, s);
  if (st != DSA_OK) return st;
  return launch_fwd(p, g, q, k, v, plan + starts_ints, out, lse, s);
}
