// Stable LatentMoE ("Kimi K3: Open Frontier Intelligence", section
// "Operational Execution Flow"): two full-width shared experts act on x; the
// routed path projects x to a latent z = x W_dn of width l, its k routed
// experts act on z, their probability-weighted sum u passes an explicit
// RMSNorm, and W_up brings it back to width d:
//   out = sum_s S_s(x) + RMSNorm(u) W_up.
// The experts' GLU is SiTU-GLU (the grouped GEMM's kAct = 1 epilogue). The
// GEMMs are the grouped GEMM kernels (the projections as one-expert GEMMs);
// this file holds the small kernels around them.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"

namespace moe {

// offsets[e] = e * rows for e = 0..n: n experts that each take `rows`
// consecutive rows (the projections: n = 1; the shared experts: n = S).
__global__ void uniform_offsets_kernel(int rows, int n, int32_t* __restrict__ offsets) {
  const int e = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x);
  if (e <= n) offsets[e] = e * rows;
}

// x_rep[s * T + t, :] = x[t, :] for s = 0..S-1: the shared experts' rows, one
// copy of x per shared expert. Thread per 16-byte vector.
__global__ void __launch_bounds__(256)
    repeat_rows_kernel(const uint4* __restrict__ x, int64_t n_vec, int S, uint4* __restrict__ x_rep) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n_vec) return;
  const uint4 v = __ldg(x + i);
  for (int s = 0; s < S; ++s) x_rep[static_cast<int64_t>(s) * n_vec + i] = v;
}

__device__ __forceinline__ float bf16_lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Routed sum and RMSNorm of one token per CTA (256 threads):
//   u = sum_j w[t, j] * y_perm[inv_perm[t, j], :]   (fp32 fma in slot order),
//   n = gamma * u / sqrt(mean(u^2) + eps)            (fp32; gamma may be null),
// stored bf16 [T, l]. Thread i holds vectors i, i + 256, ... (at most kMaxVec
// of 8 values) in registers; the sum of squares is a fixed tree (thread
// partials in vector order, then warp shuffles, then the 8 warp sums in
// order), so results are deterministic.
constexpr int kRmsMaxVec = 4;  // l <= 256 * 4 * 8 = 8192
template <int K>
__global__ void __launch_bounds__(256)
    combine_rmsnorm_kernel(const uint4* __restrict__ y_perm, const int32_t* __restrict__ inv_perm,
                           const float* __restrict__ topk_w, const float* __restrict__ gamma, float eps, int64_t T,
                           int vec_per_row, uint4* __restrict__ n_out) {
  const int64_t t = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ float s_warp[8];
  __shared__ float s_inv;
  int32_t rows[K];
  float ws[K];
#pragma unroll
  for (int j = 0; j < K; ++j) {
    rows[j] = __ldg(inv_perm + t * K + j);
    ws[j] = __ldg(topk_w + t * K + j);
    if (!index_ok(rows[j] >= 0 && rows[j] < T * K)) ws[j] = 0.0f, rows[j] = 0;
  }
  float acc[kRmsMaxVec][8];
  float ss = 0.0f;
#pragma unroll
  for (int q = 0; q < kRmsMaxVec; ++q) {
    const int v = tid + q * 256;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[q][i] = 0.0f;
    if (v < vec_per_row) {
#pragma unroll
      for (int j = 0; j < K; ++j) {
        const uint4 y = __ldg(y_perm + static_cast<int64_t>(rows[j]) * vec_per_row + v);
        const uint32_t yw[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          acc[q][2 * h] = __fmaf_rn(ws[j], bf16_lo_f(yw[h]), acc[q][2 * h]);
          acc[q][2 * h + 1] = __fmaf_rn(ws[j], bf16_hi_f(yw[h]), acc[q][2 * h + 1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = __fmaf_rn(acc[q][i], acc[q][i], ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
  if (lane == 0) s_warp[warp] = ss;
  __syncthreads();
  if (tid == 0) {
    float tot = s_warp[0];
    for (int w = 1; w < 8; ++w) tot = __fadd_rn(tot, s_warp[w]);
    const float l = static_cast<float>(vec_per_row * 8);
    const float den = sqrtf(__fadd_rn(tot / l, eps));
    s_inv = den > 0.0f ? 1.0f / den : 0.0f;  // a zero row with eps = 0 stays zero
  }
  __syncthreads();
  const float inv = s_inv;
#pragma unroll
  for (int q = 0; q < kRmsMaxVec; ++q) {
    const int v = tid + q * 256;
    if (v >= vec_per_row) continue;
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int c = v * 8 + 2 * h;
      const float g0 = gamma ? __ldg(gamma + c) : 1.0f, g1 = gamma ? __ldg(gamma + c + 1) : 1.0f;
      const __nv_bfloat162 p =
          __floats2bfloat162_rn(g0 * (acc[q][2 * h] * inv), g1 * (acc[q][2 * h + 1] * inv));
      o[h] = *reinterpret_cast<const uint32_t*>(&p);
    }
    n_out[t * vec_per_row + v] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// out = a + sum_s b[s] (bf16 rows; fp32 adds in that order, one rounding).
// a [n_vec], b [S][n_vec] 16-byte vectors; thread per vector.
__global__ void __launch_bounds__(256)
    sum_rows_kernel(const uint4* __restrict__ a, const uint4* __restrict__ b, int S, int64_t n_vec,
                    uint4* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n_vec) return;
  float acc[8];
  const uint4 av = __ldg(a + i);
  const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    acc[2 * h] = bf16_lo_f(aw[h]);
    acc[2 * h + 1] = bf16_hi_f(aw[h]);
  }
  for (int s = 0; s < S; ++s) {
    const uint4 bv = __ldg(b + static_cast<int64_t>(s) * n_vec + i);
    const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      acc[2 * h] = __fadd_rn(acc[2 * h], bf16_lo_f(bw[h]));
      acc[2 * h + 1] = __fadd_rn(acc[2 * h + 1], bf16_hi_f(bw[h]));
    }
  }
  uint32_t o[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * h], acc[2 * h + 1]);
    o[h] = *reinterpret_cast<const uint32_t*>(&p);
  }
  out[i] = make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace moe
