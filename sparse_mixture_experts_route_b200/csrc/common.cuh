// Shared definitions of the MoE CUDA library: the per-device error word and
// small helpers. Everything is compiled into one translation unit (moe_api.cu).
#pragma once

#include <cstdint>

namespace moe {

// First error recorded by any kernel on this device (0 = none). Kernels only
// ever move it from 0 to a code (atomicCAS); moe_get_device_error reads and
// clears it from the host.
__device__ unsigned int g_device_error = 0u;

__device__ __forceinline__ void record_device_error(unsigned int code) { atomicCAS(&g_device_error, 0u, code); }

// The MOE_CHECKS build (libmoe_checks.so) checks every data-dependent index
// before it is used -- rows read or written through a permutation, expert
// offsets handed to the GEMMs -- and on a bad one records
// MOE_DEVERR_INDEX_CHECK (8) and skips the access instead of faulting. In the
// normal build the checks are constant true and compile away.
#ifdef MOE_CHECKS
constexpr bool kIndexChecks = true;
#else
constexpr bool kIndexChecks = false;
#endif

__device__ __forceinline__ bool index_ok(bool ok) {
  if (!kIndexChecks) return true;
  if (!ok) record_device_error(8u /* MOE_DEVERR_INDEX_CHECK */);
  return ok;
}

// Bounded waits give up after this long. A healthy pipeline stage waits
// microseconds; the limit only ends waits that can no longer complete.
constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // 4 s

__host__ __device__ constexpr int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace moe
