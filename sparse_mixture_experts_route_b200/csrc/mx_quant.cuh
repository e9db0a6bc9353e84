// MX block quantisation: the serving format of the MoE layer on "Kimi K3:
// Open Frontier Intelligence" (section "Systems Optimization, Load Balancing,
// and Post-Training Alignment": MXFP4 expert weights, MXFP8 activations).
//
// The page names the formats only; they are taken as the published OCP MX
// formats. Blocks of 32 consecutive values along the reduction axis share one
// power-of-two scale 2^s, stored as the E8M0 code s + 127, with
//   s = floor(log2(max |v|)) - emax,  clamped to [-127, 127],
// emax the exponent of the element type's largest magnitude (2 for E2M1,
// whose largest value is 6 = 1.5 * 2^2; 8 for E4M3, 448 = 1.75 * 2^8); an
// all-zero block takes s = -127. Each element is v * 2^-s converted to the
// element type with round-to-nearest-even, saturating at the largest finite
// magnitude, sign kept (also on zero: the magnitude is converted and the sign
// bit set from the input, so -0 and negatives that round to 0 keep it). One
// code per byte: E2M1 in the low nibble (bit 3 the sign), E4M3 a full byte.
#pragma once

#include <cstdint>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

namespace moe {

constexpr int kMxBlock = 32;

// floor(log2 a) of a nonzero finite float, from its bit pattern.
__device__ __forceinline__ int floor_log2_f32(float a) {
  const uint32_t u = __float_as_uint(a) & 0x7fffffffu;
  const int eb = static_cast<int>(u >> 23);
  return eb > 0 ? eb - 127 : (31 - __clz(static_cast<int>(u))) - 149;  // subnormal: the top set bit
}

// The block scale exponent for a block maximum amax (>= 0) and element emax.
__device__ __forceinline__ int mx_scale_exponent(float amax, int emax) {
  if (amax == 0.0f) return -127;
  return min(127, max(-127, floor_log2_f32(amax) - emax));
}

// 2^-s as a float, exactly (s in [-127, 127]; 2^-127 is subnormal).
__device__ __forceinline__ float mx_inverse_scale(int s) {
  return s < 127 ? __uint_as_float(static_cast<uint32_t>(127 - s) << 23) : __uint_as_float(0x00400000u);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// MXFP8 (E4M3) of x [rows, cols] bf16 (cols % 32 == 0, 16-byte aligned), blocks
// of 32 along each row: codes [rows, cols] (16-byte aligned), scales
// [rows, cols / 32]. One thread per block.
__global__ void __launch_bounds__(256)
    mxfp8_quantize_kernel(const uint4* __restrict__ x, int64_t nblocks, uint8_t* __restrict__ codes,
                          uint8_t* __restrict__ scales) {
  const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
  uint4 q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) q[i] = __ldg(x + b * 4 + i);  // 32 bf16 = 64 bytes
  float v[32];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w4[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[i * 8 + 2 * h] = bf16_lo(w4[h]);
      v[i * 8 + 2 * h + 1] = bf16_hi(w4[h]);
    }
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int s = mx_scale_exponent(amax, 8);
  const float inv = mx_inverse_scale(s);
  scales[b] = static_cast<uint8_t>(s + 127);
  uint32_t packed[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t word = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = v[4 * i + j];
      const uint32_t c = (__nv_cvt_float_to_fp8(__fmul_rn(fabsf(a), inv), __NV_SATFINITE, __NV_E4M3) & 0x7Fu) |
                         (signbit(a) ? 0x80u : 0u);
      word |= c << (8 * j);
    }
    packed[i] = word;
  }
  uint4* dst = reinterpret_cast<uint4*>(codes + b * kMxBlock);
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
}

// MXFP4 (E2M1) of w [K, N] bf16 (N contiguous, K % 32 == 0), blocks of 32
// along K for each column: codes [K, N] (one per byte), scales [K / 32, N].
// One thread per (block, column); neighbouring threads take neighbouring
// columns, so every load and store is coalesced.
__global__ void __launch_bounds__(256)
    mxfp4_quantize_kernel(const uint16_t* __restrict__ w, int64_t K, int64_t N, uint8_t* __restrict__ codes,
                          uint8_t* __restrict__ scales) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= (K / kMxBlock) * N) return;
  const int64_t b = g / N, n = g - b * N;
  float v[32];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v[i] = __uint_as_float(static_cast<uint32_t>(__ldg(w + (b * kMxBlock + i) * N + n)) << 16);
    amax = fmaxf(amax, fabsf(v[i]));
  }
  const int s = mx_scale_exponent(amax, 2);
  const float inv = mx_inverse_scale(s);
  scales[g] = static_cast<uint8_t>(s + 127);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t c = (__nv_cvt_float_to_fp4(__fmul_rn(fabsf(v[i]), inv), __NV_E2M1, cudaRoundNearest) & 0x7u) |
                       (signbit(v[i]) ? 0x8u : 0u);
    codes[(b * kMxBlock + i) * N + n] = static_cast<uint8_t>(c);
  }
}

// mxfp4_quantize_kernel with four neighbouring columns per thread, for
// N % 4 == 0 with w 8-byte and codes/scales 4-byte aligned: each row of a
// block is one 8-byte load and one 4-byte store, so a warp moves 256 bytes of
// w and 128 bytes of codes per row instead of 64 and 32. The block stays in
// registers as packed bf16 pairs; the maxima are taken on the magnitudes' bit
// patterns (for non-negative floats the integer order is the numeric order),
// two columns per 32-bit SIMD max.
__global__ void __launch_bounds__(256)
    mxfp4_quantize_x4_kernel(const uint2* __restrict__ w, int64_t K, int64_t N4, uint32_t* __restrict__ codes,
                             uint32_t* __restrict__ scales) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= (K / kMxBlock) * N4) return;
  const int64_t b = g / N4, n4 = g - b * N4;
  const uint2* src = w + b * kMxBlock * N4 + n4;
  uint2 q[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) q[i] = __ldg(src + i * N4);
  uint32_t m01 = 0u, m23 = 0u;  // |bf16| bit patterns of columns (0, 1) and (2, 3)
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    m01 = __vmaxu2(m01, q[i].x & 0x7FFF7FFFu);
    m23 = __vmaxu2(m23, q[i].y & 0x7FFF7FFFu);
  }
  const float amax[4] = {bf16_lo(m01), bf16_hi(m01), bf16_lo(m23), bf16_hi(m23)};
  float inv[4];
  uint32_t sc = 0u;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int s = mx_scale_exponent(amax[c], 2);
    inv[c] = mx_inverse_scale(s);
    sc |= static_cast<uint32_t>(s + 127) << (8 * c);
  }
  scales[g] = sc;
  uint32_t* dst = codes + b * kMxBlock * N4 + n4;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t h[2] = {q[i].x, q[i].y};
    uint32_t word = 0u;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t bits = c & 1 ? h[c >> 1] >> 16 : h[c >> 1] & 0xFFFFu;
      const float a = __uint_as_float((bits & 0x7FFFu) << 16);
      const uint32_t code = (__nv_cvt_float_to_fp4(__fmul_rn(a, inv[c]), __NV_E2M1, cudaRoundNearest) & 0x7u) |
                            ((bits >> 12) & 0x8u);
      word |= code << (8 * c);
    }
    dst[i * N4] = word;
  }
}

}  // namespace moe
