// Device-side status word of the library.  Kernels never trap: a failed device check (a
// bounded wait that ran out, an index outside its buffer) records the first error here
// and the kernel returns.  The host reads and clears it with dsa_device_status().
#pragma once

namespace dsa {

enum DeviceCode { DSA_DEV_OK = 0, DSA_DEV_TIMEOUT = 1, DSA_DEV_BOUNDS = 2 };

// [0] code of the first error, [1] the site that raised it, [2] its blockIdx.x.
// The library is built as one translation unit, so there is one word per device.
static __device__ int g_status[4];

__device__ __forceinline__ void device_report(int code, int site) {
  if (atomicCAS(&g_status[0], 0, code) == 0) {
    g_status[1] = site;
    g_status[2] = static_cast<int>(blockIdx.x);
  }
}

}  // namespace dsa
