// Regularised least squares with a cached factorisation, for the pattern intensities of a
// structural decomposition of attention maps (the MOD-DiT page, Method section, Stage 1
// "Sparsity Map Reconstruction": (M^T M + lambda I) X = M^T S_t, with M fixed by the
// sequence geometry, so M^T M + lambda I is factored once and reused across heads and
// steps).  M: [m, p] fp32 row-major (m observations, p <= 32 patterns); S: [batch, m];
// X: [batch, p].  Sums run in fp64.
//
//   lstsq_factor_kernel : G = M^T M + lambda I, then its Cholesky factor L (lower, fp64,
//                         [p, p]); one CTA, one warp per entry of G;
//   lstsq_rhs_kernel    : partial right-hand sides M^T s_b over a slice of the m rows
//                         (grid: batch x slices), written per slice for a fixed-order sum;
//   lstsq_solve_kernel  : sums the slices in order and solves L L^T x = r (one warp per b).
#pragma once

#include <stdint.h>

#include "dsa_device_status.cuh"

namespace dsa {

constexpr int kLstsqMaxP = 32;
constexpr int kLstsqSliceRows = 8192;  // rows of M per partial right-hand side

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

// part: [batch, slices, p] fp64
__global__ void __launch_bounds__(256) lstsq_rhs_kernel(const float* M, const float* S, int m, int p, double* part) {
  __shared__ double acc[8][kLstsqMaxP];
  const int b = blockIdx.y, slice = blockIdx.x, slices = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = slice * kLstsqSliceRows, r1 = min(r0 + kLstsqSliceRows, m);
  const float* s = S + static_cast<int64_t>(b) * m;
  for (int a = 0; a < p; ++a) {
    double x = 0.0;
    for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x)
      x += static_cast<double>(s[r]) * static_cast<double>(M[static_cast<int64_t>(r) * p + a]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (lane == 0) acc[warp][a] = x;
  }
  __syncthreads();
  if (threadIdx.x < p) {
    double x = 0.0;
    for (int w = 0; w < 8; ++w) x += acc[w][threadIdx.x];
    part[(static_cast<int64_t>(b) * slices + slice) * p + threadIdx.x] = x;
  }
}

__global__ void __launch_bounds__(32) lstsq_solve_kernel(const double* L, const double* part, int slices, int p,
                                                         float* X) {
  const int b = blockIdx.x;
  if (threadIdx.x != 0) return;
  double y[kLstsqMaxP];
  for (int a = 0; a < p; ++a) {
    double r = 0.0;
    for (int sl = 0; sl < slices; ++sl) r += part[(static_cast<int64_t>(b) * slices + sl) * p + a];
    y[a] = r;
  }
  for (int i = 0; i < p; ++i) {  // L y = r
    double s = y[i];
    for (int t = 0; t < i; ++t) s -= L[i * p + t] * y[t];
    y[i] = s / L[i * p + i];
  }
  for (int i = p - 1; i >= 0; --i) {  // L^T x = y
    double s = y[i];
    for (int t = i + 1; t < p; ++t) s -= L[t * p + i] * y[t];
    y[i] = s / L[i * p + i];
  }
  for (int a = 0; a < p; ++a) X[static_cast<int64_t>(b) * p + a] = static_cast<float>(y[a]);
}

}  // namespace dsa
