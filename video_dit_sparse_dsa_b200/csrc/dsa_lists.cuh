// Key-tile lists (block-sparse form of the operator): query tile i attends to the key
// tiles list[row_ptr[i] .. row_ptr[i+1]) instead of its window box.  The generalisation is
// the MOD-DiT page's (Method section, Stage 2, "Online Block Masking": attention over
// selected key blocks); the window form is the special case row_ptr[i] = i * Wt.
//
//   list_check_kernel   : validates a caller's CSR on the device and records a bounds
//                         error in the status word (the kernels that read the lists clamp
//                         every index, so an invalid list gives wrong numbers, never a fault);
//   invert_lists_kernel : the inverse CSR (for every key tile, the query tiles whose list
//                         holds it, ascending, once per occurrence) that the key-major
//                         backward walks.
#pragma once

#include <stdint.h>

#include "dsa_device_status.cuh"

namespace dsa {

// row_ptr: n_lists * (n_tiles + 1) offsets (one list, or one per (batch, head), each
// head's rows following the previous head's), checked as one non-decreasing sequence from
// 0 to nnz; list: nnz tile indices in [0, n_tiles).
__global__ void __launch_bounds__(256) list_check_kernel(const int32_t* row_ptr, const int32_t* list, int n_tiles,
                                                         int n_lists, int nnz) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t n_ptr = static_cast<int64_t>(n_lists) * (n_tiles + 1);
  if (t0 == 0 && (row_ptr[0] != 0 || row_ptr[n_ptr - 1] != nnz)) device_report(DSA_DEV_BOUNDS, 90);
  for (int64_t i = t0; i + 1 < n_ptr; i += stride)
    if (row_ptr[i + 1] < row_ptr[i]) device_report(DSA_DEV_BOUNDS, 91);
  for (int64_t e = t0; e < nnz; e += stride)
    if (list[e] < 0 || list[e] >= n_tiles) device_report(DSA_DEV_BOUNDS, 92);
}

// Entries of row i of a caller's CSR, clamped into [0, nnz].
__device__ __forceinline__ void list_row(const int32_t* row_ptr, int nnz, int i, int& a, int& b) {
  a = min(max(row_ptr[i], 0), nnz);
  b = min(max(row_ptr[i + 1], a), nnz);
}

// One CTA of 1024 threads per list (blockIdx.x = list h, whose rows are
// row_ptr[h * (n_tiles + 1) ...]).  counts: n_tiles ints of scratch per list.  The inverse
// of list h occupies the same positions [row_ptr[h][0], row_ptr[h][n_tiles]) of
// inv_q_tiles as its entries do of the list, with absolute offsets in inv_row_ptr[h].
// Entries outside [0, n_tiles) are skipped and nothing is written outside the list's own
// positions, whatever the offsets hold (list_check_kernel reports invalid lists).
__global__ void __launch_bounds__(1024) invert_lists_kernel(const int32_t* row_ptr, const int32_t* list, int n_tiles,
                                                            int nnz, int32_t* counts, int32_t* inv_row_ptr,
                                                            int32_t* inv_q_tiles) {
  __shared__ int32_t part[1024];
  const int tid = threadIdx.x, nt = blockDim.x;
  const int64_t h = blockIdx.x;
  row_ptr += h * (n_tiles + 1);
  inv_row_ptr += h * (n_tiles + 1);
  counts += h * n_tiles;
  const int lo = min(max(row_ptr[0], 0), nnz), hi = min(max(row_ptr[n_tiles], lo), nnz);
  for (int j = tid; j < n_tiles; j += nt) counts[j] = 0;
  __syncthreads();
  for (int i = tid; i < n_tiles; i += nt) {
    int a, b;
    list_row(row_ptr, nnz, i, a, b);
    for (int e = a; e < b; ++e) {
      const int j = list[e];
      if (j >= 0 && j < n_tiles) atomicAdd(&counts[j], 1);
    }
  }
  __syncthreads();
  // exclusive scan of counts from lo: each thread sums a contiguous segment, thread 0 scans
  // the segment sums, each thread writes its segment's offsets (capped at hi)
  const int seg = (n_tiles + nt - 1) / nt;
  const int j0 = min(tid * seg, n_tiles), j1 = min(j0 + seg, n_tiles);
  int64_t sum = 0;
  for (int j = j0; j < j1; ++j) sum += counts[j];
  part[tid] = static_cast<int32_t>(min(sum, static_cast<int64_t>(nnz)));
  __syncthreads();
  if (tid == 0) {
    int64_t run = lo;
    for (int t = 0; t < nt; ++t) {
      const int64_t c = part[t];
      part[t] = static_cast<int32_t>(min(run, static_cast<int64_t>(hi)));
      run += c;
    }
    inv_row_ptr[n_tiles] = hi;
  }
  __syncthreads();
  int64_t run = part[tid];
  for (int j = j0; j < j1; ++j) {
    inv_row_ptr[j] = static_cast<int32_t>(min(run, static_cast<int64_t>(hi)));
    run += counts[j];
  }
  __syncthreads();
  for (int j = tid; j < n_tiles; j += nt) counts[j] = 0;
  __syncthreads();
  for (int i = tid; i < n_tiles; i += nt) {
    int a, b;
    list_row(row_ptr, nnz, i, a, b);
    for (int e = a; e < b; ++e) {
      const int j = list[e];
      if (j < 0 || j >= n_tiles) continue;
      const int pos = inv_row_ptr[j] + atomicAdd(&counts[j], 1);
      if (pos < inv_row_ptr[j + 1]) inv_q_tiles[pos] = i;  // always, for a valid list
    }
  }
  __syncthreads();
  // ascending query tiles per row (the fill order above depends on timing)
  for (int j = tid; j < n_tiles; j += nt) {
    const int a = inv_row_ptr[j], b = inv_row_ptr[j + 1];
    for (int x = a + 1; x < b; ++x) {
      const int32_t v = inv_q_tiles[x];
      int y = x - 1;
      while (y >= a && inv_q_tiles[y] > v) {
        inv_q_tiles[y + 1] = inv_q_tiles[y];
        --y;
      }
      inv_q_tiles[y + 1] = v;
    }
  }
}

}  // namespace dsa
