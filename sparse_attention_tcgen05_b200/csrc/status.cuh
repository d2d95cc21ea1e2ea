// Device status word shared by all kernels of the library (one translation unit).
#pragma once

#include <cstdint>

#include "../../include/dsa.h"

namespace dsa {

// Default upper bound on any single wait inside a kernel (mbarrier phases).  Kernels here finish
// in milliseconds; a wait this long means a lost arrival, so the kernel records it and exits.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// The bound in force on this device (dsa_set_wait_limit_ns changes it, e.g. so that a test can
// make a wait expire quickly).  Read only on the slow path of a wait.
__device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;

__device__ __forceinline__ uint64_t wait_limit_ns() { return g_wait_limit_ns; }

// Low byte: dsa_status code; bits 8..15: the wait site that expired (for diagnostics).
__device__ int g_device_status;

__device__ __forceinline__ void record_timeout(int site) {
  atomicCAS(&g_device_status, 0, static_cast<int>(DSA_ERR_TIMEOUT) | (site << 8));
}

// A caller-supplied index outside [0, Lk) was treated as an empty slot.
__device__ __forceinline__ void record_bad_index() {
  atomicCAS(&g_device_status, 0, static_cast<int>(DSA_ERR_INVALID_ARG) | (0xFF << 8));
}

}  // namespace dsa
