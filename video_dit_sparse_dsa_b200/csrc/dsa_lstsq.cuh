// Regularised least squares with a cached factorisation, for the pattern intensities of a
// structural decomposition of attention maps (the MOD-DiT page, Method section, Stage 1
// "Sparsity Map Reconstruction": (M^T M + lambda I) X = M^T S_t, with M fixed by the
// sequence geometry, so M^T M + lambda I is factored once and reused across heads and
// steps).  M: [m, p] fp32 row-major (m observations, p <= 32 patterns); S: [batch, m];
// X: [batch, p].  Sums run in fp64.
//
//   lstsq_factor_kernel : G = M^T M + lambda I, then its Cholesky factor L (lower, fp64,
//                         [p, p]); one CTA, one warp per entry of G;
//   lstsq_solve_kernel  : one launch for a batch of right-hand sides: M^T s_b summed by a
//                         cluster of CTAs per b, then L L^T x = M^T s_b solved.
#pragma once

#include <stdint.h>

#include <cooperative_groups.h>

#include "dsa_device_status.cuh"

namespace dsa {

constexpr int kLstsqMaxP = 32;

__global__ void __launch_bounds__(256) lstsq_factor_kernel(const float* M, int m, int p, float lambda, double* L) {
  __shared__ double G[kLstsqMaxP][kLstsqMaxP];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int e = warp; e < p * p; e += nw) {
    const int a = e / p, b = e % p;
    if (b > a) continue;
    double s = 0.0;
    for (int r = lane; r < m; r += 32)
      s += static_cast<double>(M[static_cast<int64_t>(r) * p + a]) * static_cast<double>(M[static_cast<int64_t>(r) * p + b]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) G[a][b] = s + (a == b ? static_cast<double>(lambda) : 0.0);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Cholesky-Banachiewicz: L[i][j] for j <= i, row by row
    bool pd = true;
    for (int i = 0; i < p; ++i) {
      for (int j = 0; j <= i; ++j) {
        double s = G[i][j];
        for (int t = 0; t < j; ++t) s -= L[i * p + t] * L[j * p + t];
        if (i == j) {
          if (!(s > 0.0)) {
            pd = false;
            s = 1.0;
          }
          L[i * p + i] = sqrt(s);
        } else {
          L[i * p + j] = s / L[j * p + j];
        }
      }
      for (int j = i + 1; j < p; ++j) L[i * p + j] = 0.0;
    }
    if (!pd) device_report(DSA_DEV_BOUNDS, 95);  // M^T M + lambda I is not positive definite
  }
}

// X[b] = (L L^T)^-1 M^T s_b for every right-hand side b, in one launch: a cluster of
// kLstsqCluster CTAs per b (grid (kLstsqCluster, batch)).  CTA r of a cluster sums M^T s_b
// over its contiguous slice of the m rows in fp64 (each thread over rows tid, tid + 512, ...,
// four rows' loads in flight at a time, then the warps' sums in warp order); the cluster's rank-0 CTA adds the CTAs' partial sums
// in rank order, read from their shared memory, and one thread solves L y = r, L^T x = y.
// Every sum runs in a fixed order, so X is the same from run to run.
constexpr int kLstsqCluster = 8;
constexpr int kLstsqThreads = 512;
constexpr int kLstsqUnroll = 4;  // rows per thread whose loads are in flight together

__global__ void __cluster_dims__(kLstsqCluster, 1, 1) __launch_bounds__(kLstsqThreads)
    lstsq_solve_kernel(const float* __restrict__ M, const float* __restrict__ S, int m, int p,
                       const double* __restrict__ L, float* __restrict__ X) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ double warp_acc[kLstsqThreads / 32][kLstsqMaxP];
  __shared__ double part[kLstsqMaxP];
  const int b = blockIdx.y;
  const int rank = static_cast<int>(cluster.block_rank());
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = (m + kLstsqCluster - 1) / kLstsqCluster;
  const int r0 = rank * per, r1 = min(r0 + per, m);
  const float* s = S + static_cast<int64_t>(b) * m;
  double acc[kLstsqMaxP];
#pragma unroll
  for (int a = 0; a < kLstsqMaxP; ++a) acc[a] = 0.0;
  for (int r = r0 + threadIdx.x; r < r1; r += kLstsqUnroll * kLstsqThreads) {
    float sv[kLstsqUnroll];
#pragma unroll
    for (int u = 0; u < kLstsqUnroll; ++u) {
      const int rr = r + u * kLstsqThreads;
      sv[u] = rr < r1 ? s[rr] : 0.f;
    }
#pragma unroll
    for (int a = 0; a < kLstsqMaxP; ++a) {
      if (a < p) {
        float mv[kLstsqUnroll];
#pragma unroll
        for (int u = 0; u < kLstsqUnroll; ++u) {
          const int rr = r + u * kLstsqThreads;
          mv[u] = rr < r1 ? M[static_cast<int64_t>(rr) * p + a] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kLstsqUnroll; ++u) acc[a] += static_cast<double>(sv[u]) * static_cast<double>(mv[u]);
      }
    }
  }
#pragma unroll
  for (int a = 0; a < kLstsqMaxP; ++a) {
    if (a < p) {
      double x = acc[a];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (lane == 0) warp_acc[warp][a] = x;
    }
  }
  __syncthreads();
  if (threadIdx.x < p) {
    double x = 0.0;
    for (int w = 0; w < kLstsqThreads / 32; ++w) x += warp_acc[w][threadIdx.x];
    part[threadIdx.x] = x;
  }
  cluster.sync();  // every CTA's partial sums are in its shared memory
  if (rank == 0 && threadIdx.x == 0) {
    double y[kLstsqMaxP];
    for (int a = 0; a < p; ++a) {
      double r = 0.0;
      for (int k = 0; k < kLstsqCluster; ++k) r += cluster.map_shared_rank(part, k)[a];
      y[a] = r;
    }
    for (int i = 0; i < p; ++i) {  // L y = r
      double t = y[i];
      for (int j = 0; j < i; ++j) t -= L[i * p + j] * y[j];
      y[i] = t / L[i * p + i];
    }
    for (int i = p - 1; i >= 0; --i) {  // L^T x = y
      double t = y[i];
      for (int j = i + 1; j < p; ++j) t -= L[j * p + i] * y[j];
      y[i] = t / L[i * p + i];
    }
    for (int a = 0; a < p; ++a) X[static_cast<int64_t>(b) * p + a] = static_cast<float>(y[a]);
  }
  cluster.sync();  // the other CTAs' shared memory stays valid until rank 0 has read it
}

}  // namespace dsa
