// Operand preparation for the MX expert feed-forward (MXFP4 expert weights,
// MXFP8 activations: the serving format of "Kimi K3: Open Frontier
// Intelligence", section "Systems Optimization, Load Balancing, and
// Post-Training Alignment"). The element and scale rules are those of
// mx_quant.cuh; this file only lays the results out the way the block-scaled
// tensor-core GEMM (mx_gemm.cuh) reads them.
//
// Layouts (all byte arrays):
//   packed weights  Wq[E][N][K / 2]: for output feature n of expert e, the
//       E2M1 codes of w[e][0..K)[n] along K, two per byte, element 2i in the
//       low nibble of byte i (K-major: the reduction axis is contiguous, as the
//       tensor core requires for 4-bit operands).
//   scale atoms: the E8M0 scales of a 128-row x 128-K tile form one 512-byte
//       atom; row m (0..127) and 32-element block kb (0..3) of the tile sit at
//       byte 16 * (m % 32) + 4 * (m / 32) + kb, which is the order in which one
//       tcgen05.cp of 32 rows x 128 bits, broadcast to the four TMEM lane
//       quadrants, leaves row m's four scales in lane m, column m / 32.
//       Weights: SFw[E][N / 128][K / 128][512]. Token operands (x and h): one
//       run of atoms per GEMM token tile, SFt[tile][K / 128][512], row m of a
//       tile being its m-th token row.
#pragma once

#include <cstdint>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "mx_quant.cuh"

namespace moe {

constexpr int kMxAtomBytes = 512;
constexpr int kMxTileRows = 112;  // token rows per GEMM tile (the MMA's N)

__host__ __device__ constexpr int64_t mx_atom_offset(int m, int kb) { return 16 * (m % 32) + 4 * (m / 32) + kb; }

// E2M1 code (sign in bit 3) of v * 2^-s, inv = 2^-s.
__device__ __forceinline__ uint32_t mx_e2m1_code(float v, float inv) {
  return (__nv_cvt_float_to_fp4(__fmul_rn(fabsf(v), inv), __NV_E2M1, cudaRoundNearest) & 0x7u) |
         (signbit(v) ? 0x8u : 0u);
}

// E4M3 code (sign in bit 7) of v * 2^-s, inv = 2^-s.
__device__ __forceinline__ uint32_t mx_e4m3_code(float v, float inv) {
  return (__nv_cvt_float_to_fp8(__fmul_rn(fabsf(v), inv), __NV_SATFINITE, __NV_E4M3) & 0x7Fu) |
         (signbit(v) ? 0x80u : 0u);
}

// W [E][K][N] bf16 (N contiguous; K % 128 == 0, N % 128 == 0) -> packed
// K-major E2M1 codes and weight scale atoms. One thread per (expert, 32-row
// block of K, column n); neighbouring threads take neighbouring columns, so
// the bf16 reads are coalesced. Each thread writes its 16 code bytes with one
// 16-byte store and its scale byte into the atom.
__global__ void __launch_bounds__(256)
    mx_pack_weights_kernel(const uint16_t* __restrict__ w, int E, int K, int N, uint8_t* __restrict__ wq,
                           uint8_t* __restrict__ sf) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int KB = K / kMxBlock;
  if (g >= static_cast<int64_t>(E) * KB * N) return;
  const int n = static_cast<int>(g % N);
  const int64_t eb = g / N;
  const int b = static_cast<int>(eb % KB);
  const int e = static_cast<int>(eb / KB);
  const uint16_t* src = w + (static_cast<int64_t>(e) * K + static_cast<int64_t>(b) * kMxBlock) * N + n;
  float v[32];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v[i] = __uint_as_float(static_cast<uint32_t>(__ldg(src + static_cast<int64_t>(i) * N)) << 16);
    amax = fmaxf(amax, fabsf(v[i]));
  }
  const int s = mx_scale_exponent(amax, 2);
  const float inv = mx_inverse_scale(s);
  uint32_t word[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t acc = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc |= mx_e2m1_code(v[8 * j + i], inv) << (4 * i);
    word[j] = acc;
  }
  uint8_t* dst = wq + (static_cast<int64_t>(e) * N + n) * (K / 2) + static_cast<int64_t>(b) * 16;
  *reinterpret_cast<uint4*>(dst) = make_uint4(word[0], word[1], word[2], word[3]);
  const int64_t atom = (static_cast<int64_t>(e) * (N / 128) + n / 128) * (K / 128) + b / 4;
  sf[atom * kMxAtomBytes + mx_atom_offset(n % 128, b % 4)] = static_cast<uint8_t>(s + 127);
}

// x [T][d] bf16 -> MXFP8 rows in dispatch order plus per-tile scale atoms, in
// one pass: CTA (t, s) for token t takes the blocks s * blockDim.x + i,
// (s + gridDim.y) * blockDim.x + i, ... (one thread per 32-element block; a
// step of few tokens spreads each token over several CTAs); each block's codes
// and scale go to all k of the token's dispatched rows. Pair (t, j) has expert
// e = idx[t * k + j] and row r = inv_perm[t * k + j]; its tile is
// prefix[e] + (r - offsets[e]) / kMxTileRows and its row in the tile
// (r - offsets[e]) % kMxTileRows. d % 128 == 0.
__global__ void __launch_bounds__(256)
    mx_quantize_dispatch_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ idx,
                                const int32_t* __restrict__ inv_perm, const int32_t* __restrict__ offsets,
                                const int32_t* __restrict__ prefix, int d, int k, int E, uint8_t* __restrict__ xq,
                                uint8_t* __restrict__ sft) {
  const int t = blockIdx.x;
  const int nblk = d / kMxBlock;
  __shared__ int32_t s_row[16], s_tile[16], s_m[16];
  if (threadIdx.x < k) {
    const int64_t pr = static_cast<int64_t>(t) * k + threadIdx.x;
    const int e = __ldg(idx + pr);
    const int r = __ldg(inv_perm + pr);
    const bool ok = e >= 0 && e < E && index_ok(r >= 0 && r < static_cast<int64_t>(gridDim.x) * k);
    const int local = ok ? r - __ldg(offsets + e) : 0;
    s_row[threadIdx.x] = ok ? r : -1;
    s_tile[threadIdx.x] = ok ? __ldg(prefix + e) + local / kMxTileRows : 0;
    s_m[threadIdx.x] = local % kMxTileRows;
    if (!ok) record_device_error(5u /* MOE_DEVERR_BAD_ROUTE */);
  }
  __syncthreads();
  for (int b = static_cast<int>(blockIdx.y * blockDim.x + threadIdx.x); b < nblk;
       b += static_cast<int>(gridDim.y * blockDim.x)) {
    uint4 q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = __ldg(x + (static_cast<int64_t>(t) * nblk + b) * 4 + i);
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
    uint32_t packed[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t word = 0u;
#pragma unroll
      for (int j = 0; j < 4; ++j) word |= mx_e4m3_code(v[4 * i + j], inv) << (8 * j);
      packed[i] = word;
    }
    for (int j = 0; j < k; ++j) {
      const int r = s_row[j];
      if (r < 0) continue;
      uint4* dst = reinterpret_cast<uint4*>(xq + static_cast<int64_t>(r) * d + static_cast<int64_t>(b) * kMxBlock);
      dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
      const int64_t atom = static_cast<int64_t>(s_tile[j]) * (d / 128) + b / 4;
      sft[atom * kMxAtomBytes + mx_atom_offset(s_m[j], b % 4)] = static_cast<uint8_t>(s + 127);
    }
  }
}

}  // namespace moe
