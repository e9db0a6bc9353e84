// Row movement for expert parallelism ("Kimi K3: Open Frontier Intelligence",
// section "Systems Optimization, Load Balancing, and Post-Training
// Alignment": the routed experts are split over ranks, and each rank's
// dispatched token rows travel to the rank that owns their expert and back).
//
// The exchange itself is the caller's collective (an all-to-all over NCCL);
// on each side of it the rows have to be put in the order the next step
// reads: the receiver's rows from every source rank into one expert-major
// block for the grouped GEMM, and the results back into the order they
// arrived in. Both are row gathers, out[i] = src[rows[i]], done here.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace moe {

// out[i] = src[rows[i]] for 0 <= rows[i] < n_src; a row index of -1 writes a
// zero row (padding of a fixed-capacity buffer); any other index outside
// [0, n_src) writes a zero row and records MOE_DEVERR_BAD_ROUTE. Warp per
// output row, 16-byte vectors (vec_per_row = d * 2 / 16), four loads in
// flight per lane.
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4* __restrict__ src, int64_t n_src, const int32_t* __restrict__ rows,
                       int64_t n_out, int vec_per_row, uint4* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (i >= n_out) return;
  const int lane = threadIdx.x & 31;
  const int32_t r = __ldg(rows + i);
  uint4* dst = out + i * vec_per_row;
  if (r < 0 || r >= n_src) {
    if (r != -1 && lane == 0) record_device_error(5u /* MOE_DEVERR_BAD_ROUTE */);
    for (int v = lane; v < vec_per_row; v += 32) dst[v] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const uint4* s = src + static_cast<int64_t>(r) * vec_per_row;
  int v = lane;
  for (; v + 96 < vec_per_row; v += 128) {
    const uint4 a = __ldg(s + v), b = __ldg(s + v + 32), c = __ldg(s + v + 64), d = __ldg(s + v + 96);
    dst[v] = a;
    dst[v + 32] = b;
    dst[v + 64] = c;
    dst[v + 96] = d;
  }
  for (; v < vec_per_row; v += 32) dst[v] = __ldg(s + v);
}

}  // namespace moe
