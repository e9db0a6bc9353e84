// Dispatch (permute) and combine (unpermute).
//
// Dispatch follows "Kimi K3: Open Frontier Intelligence", section
// "Operational Execution Flow": each token is sent to its active routed
// experts. Layout built here: a stable counting sort of the T*k (token, slot)
// pairs by expert, so expert e owns rows offsets[e] .. offsets[e+1]-1 in
// ascending token order. Three passes, no atomics that decide an order:
//   hist    per block of kPairsPerBlock consecutive pairs: a per-expert count;
//   scan    per expert: total, exclusive scan over experts (offsets), and each
//           block's first row for each expert;
//   scatter per block, one warp walking its pairs in order 32 at a time; the
//           rank among equal experts inside a group of 32 comes from
//           __match_any_sync, so the result is the sequential counting sort.
// The combine (same page and section: the routed output is the
// probability-weighted sum of the selected experts' outputs) accumulates the k
// rows of a token in fp32 in ascending slot order.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"

namespace moe {

constexpr int kPairsPerBlock = 512;

__global__ void __launch_bounds__(256)
    permute_hist_kernel(const int32_t* __restrict__ topk_idx, int64_t n_pairs, int E, int32_t* __restrict__ block_hist) {
  extern __shared__ int32_t cnt[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int64_t q0 = static_cast<int64_t>(blockIdx.x) * kPairsPerBlock;
  const int64_t q1 = min(n_pairs, q0 + kPairsPerBlock);
  for (int64_t q = q0 + threadIdx.x; q < q1; q += blockDim.x) {
    const int e = topk_idx[q];
    if (e >= 0 && e < E)
      atomicAdd(&cnt[e], 1);
    else
      record_device_error(5u /* MOE_DEVERR_BAD_ROUTE */);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) block_hist[static_cast<int64_t>(blockIdx.x) * E + e] = cnt[e];
}

// One block of 1024 threads; thread e owns expert e (E <= 1024).
// In: block_hist[nblk][E] counts. Out: offsets[0..E]; block_hist rewritten in
// place with each block's first row per expert.
__global__ void __launch_bounds__(1024)
    permute_scan_kernel(int32_t* __restrict__ block_hist, int nblk, int E, int32_t* __restrict__ offsets) {
  __shared__ int32_t warp_sums[32];
  const int e = threadIdx.x;
  constexpr int kBatch = 16;  // block counts in flight per thread
  int32_t total = 0;
  if (e < E)
    for (int b0 = 0; b0 < nblk; b0 += kBatch) {
      int32_t c[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        c[u] = (b0 + u < nblk) ? block_hist[static_cast<int64_t>(b0 + u) * E + e] : 0;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) total += c[u];
    }
  // exclusive scan of `total` over the block
  const int lane = e & 31, w = e >> 5;
  int32_t incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[w] = incl;
  __syncthreads();
  if (w == 0) {
    int32_t ws = warp_sums[lane];
    int32_t wincl = ws;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, wincl, o);
      if (lane >= o) wincl += y;
    }
    warp_sums[lane] = wincl - ws;  // exclusive prefix of warp totals
  }
  __syncthreads();
  const int32_t excl = warp_sums[w] + incl - total;
  if (e < E) {
    offsets[e] = excl;
    if (e == E - 1) offsets[E] = excl + total;
    int32_t run = excl;
    for (int b0 = 0; b0 < nblk; b0 += kBatch) {
      int32_t c[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        c[u] = (b0 + u < nblk) ? block_hist[static_cast<int64_t>(b0 + u) * E + e] : 0;
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (b0 + u < nblk) {
          block_hist[static_cast<int64_t>(b0 + u) * E + e] = run;
          run += c[u];
        }
    }
  }
}

// One warp per block of kPairsPerBlock pairs.
__global__ void __launch_bounds__(32)
    permute_scatter_kernel(const int32_t* __restrict__ topk_idx, int64_t n_pairs, int E, int k,
                           const int32_t* __restrict__ block_base, int32_t* __restrict__ perm_token,
                           int32_t* __restrict__ inv_perm) {
  extern __shared__ int32_t base[];
  const int lane = threadIdx.x;
  for (int e = lane; e < E; e += 32) base[e] = block_base[static_cast<int64_t>(blockIdx.x) * E + e];
  __syncwarp();
  const int64_t q0 = static_cast<int64_t>(blockIdx.x) * kPairsPerBlock;
  const int64_t q1 = min(n_pairs, q0 + kPairsPerBlock);
  for (int64_t g = q0; g < q1; g += 32) {
    const int64_t q = g + lane;
    const bool valid = q < q1;
    int e = valid ? topk_idx[q] : -1;
    if (valid && (e < 0 || e >= E)) e = -2;  // reported by the hist pass; never written
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int32_t row = 0;
    if (e >= 0) row = base[e] + rank;
    __syncwarp();
    if (e >= 0 && rank == 0) base[e] += __popc(peers);
    __syncwarp();
    if (e >= 0) {
      perm_token[row] = static_cast<int32_t>(q / k);
      inv_perm[q] = row;
    }
  }
}

// x_perm[row, :] = x[perm_token[row], :], 16-byte vectors, one warp per row;
// each lane keeps 4 loads in flight. x has n_src rows (checked in the
// MOE_CHECKS build).
__global__ void __launch_bounds__(256)
    permute_copy_rows_kernel(const uint4* __restrict__ x, int64_t n_src, const int32_t* __restrict__ perm_token,
                             int64_t n_rows, int vec_per_row, uint4* __restrict__ x_perm) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const int lane = threadIdx.x & 31;
  const int32_t tok = __ldg(perm_token + row);
  if (!index_ok(tok >= 0 && tok < n_src)) return;
  const uint4* src = x + static_cast<int64_t>(tok) * vec_per_row;
  uint4* dst = x_perm + row * vec_per_row;
  int v = lane;
  for (; v + 96 < vec_per_row; v += 128) {
    const uint4 a = __ldg(src + v), b = __ldg(src + v + 32), c = __ldg(src + v + 64), d = __ldg(src + v + 96);
    __stcs(dst + v, a);
    __stcs(dst + v + 32, b);
    __stcs(dst + v + 64, c);
    __stcs(dst + v + 96, d);
  }
  for (; v < vec_per_row; v += 32) __stcs(dst + v, __ldg(src + v));
}

// x_perm[inv_perm[t, j], :] = x[t, :] for every slot j of token t: one CTA of
// 128 threads per token reads the row once (8 vectors of 16 bytes per thread
// per pass) and writes its k copies, so x crosses HBM once however many
// experts a token picks. Same result as the row-by-row gather.
__global__ void __launch_bounds__(128)
    permute_copy_tokens_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ inv_perm, int k,
                               int vec_per_row, uint4* __restrict__ x_perm) {
  constexpr int kVec = 8;
  const int64_t t = blockIdx.x;
  const int tid = threadIdx.x;
  int32_t dst_row[16];
  const int64_t n_rows = static_cast<int64_t>(gridDim.x) * k;  // x_perm has T k rows
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    dst_row[j] = (j < k) ? __ldg(inv_perm + t * k + j) : 0;
    if (j < k && !index_ok(dst_row[j] >= 0 && dst_row[j] < n_rows)) dst_row[j] = -1;
  }
  const uint4* src = x + t * vec_per_row;
  for (int v0 = 0; v0 < vec_per_row; v0 += 128 * kVec) {
    uint4 r[kVec];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const int v = v0 + u * 128 + tid;
      if (v < vec_per_row) r[u] = __ldg(src + v);
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j >= k) break;
      if (kIndexChecks && dst_row[j] < 0) continue;
      uint4* dst = x_perm + static_cast<int64_t>(dst_row[j]) * vec_per_row;
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int v = v0 + u * 128 + tid;
        if (v < vec_per_row) __stcs(dst + v, r[u]);
      }
    }
  }
}

// out[t, :] = sum_j w[t, j] * y_perm[inv_perm[t, j], :]; fp32 fma in ascending
// j, one rounding to bf16. One thread per 16-byte vector (8 values) of one
// token, with K (the number of slots) fixed at compile time so all K row loads
// are in flight together.
template <int K>
__global__ void __launch_bounds__(256)
    unpermute_kernel(const uint4* __restrict__ y_perm, const int32_t* __restrict__ inv_perm,
                     const float* __restrict__ topk_w, int64_t T, int vec_per_row, uint4* __restrict__ out) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t t = g / vec_per_row;
  const int v = static_cast<int>(g - t * vec_per_row);
  if (t >= T) return;
  uint4 y[K];
  float ws[K];
#pragma unroll
  for (int j = 0; j < K; ++j) {
    const int32_t row = __ldg(inv_perm + t * K + j);
    ws[j] = __ldg(topk_w + t * K + j);
    // y_perm has T K rows; the MOE_CHECKS build skips (adds zero for) a bad one
    y[j] = index_ok(row >= 0 && row < T * K) ? __ldg(y_perm + static_cast<int64_t>(row) * vec_per_row + v)
                                              : make_uint4(0u, 0u, 0u, 0u);
  }
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
  for (int j = 0; j < K; ++j) {
    const uint32_t yw[4] = {y[j].x, y[j].y, y[j].z, y[j].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[2 * q] = __fmaf_rn(ws[j], __uint_as_float(yw[q] << 16), acc[2 * q]);
      acc[2 * q + 1] = __fmaf_rn(ws[j], __uint_as_float(yw[q] & 0xFFFF0000u), acc[2 * q + 1]);
    }
  }
  uint32_t o[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
    o[q] = *reinterpret_cast<const uint32_t*>(&p);
  }
  out[t * vec_per_row + v] = make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace moe

namespace moe {

constexpr int kSmallDispatchPairs = 2048;  // fused single-block dispatch up to this many (token, slot) pairs

// Dispatch for few pairs in one block of 1024 threads (E <= 1024): per-expert
// counts, exclusive scan (offsets), the stable counting-sort scatter (one warp
// walks the pairs in order, 32 at a time, ranks from __match_any_sync), and the
// token-block prefixes of both grouped GEMMs (blocks of rows0 and of rows1
// rows), so a decode step needs one launch here instead of four. It also
// clears zero_n words at zero_buf (the K-split tickets of the gate/up GEMM
// that follows; zero_n may be 0).
__global__ void __launch_bounds__(1024)
    dispatch_small_kernel(const int32_t* __restrict__ topk_idx, int n_pairs, int E, int k, int rows0, int rows1,
                          int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token, int32_t* __restrict__ inv_perm,
                          int32_t* __restrict__ prefix0, int32_t* __restrict__ prefix1, unsigned int* __restrict__ zero_buf,
                          int zero_n) {
  __shared__ int32_t cnt[1024];
  __shared__ int32_t base[1024];
  __shared__ int32_t wsum[3][32];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  cnt[tid] = 0;
  for (int i = tid; i < zero_n; i += 1024) zero_buf[i] = 0u;
  __syncthreads();
  for (int q = tid; q < n_pairs; q += 1024) {
    const int e = topk_idx[q];
    if (e >= 0 && e < E)
      atomicAdd(&cnt[e], 1);
    else
      record_device_error(5u /* MOE_DEVERR_BAD_ROUTE */);
  }
  __syncthreads();
  // exclusive scans over experts: rows, rows0-row blocks and rows1-row blocks
  const int32_t c = (tid < E) ? cnt[tid] : 0;
  int32_t v[3] = {c, (c + rows0 - 1) / rows0, (c + rows1 - 1) / rows1};
  int32_t incl[3];
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    incl[m] = v[m];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl[m], o);
      if (lane >= o) incl[m] += y;
    }
    if (lane == 31) wsum[m][w] = incl[m];
  }
  __syncthreads();
  if (w < 3) {
    const int32_t ws = wsum[w][lane];
    int32_t wi = ws;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    wsum[w][lane] = wi - ws;
  }
  __syncthreads();
  if (tid < E) {
    int32_t* outs[3] = {offsets, prefix0, prefix1};
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      const int32_t excl = wsum[m][w] + incl[m] - v[m];
      outs[m][tid] = excl;
      if (tid == E - 1) outs[m][E] = excl + v[m];
      if (m == 0) base[tid] = excl;
    }
  }
  __syncthreads();
  if (w == 0) {
    for (int g = 0; g < n_pairs; g += 32) {
      const int q = g + lane;
      int e = (q < n_pairs) ? topk_idx[q] : -1;
      if (q < n_pairs && (e < 0 || e >= E)) e = -2;
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      int32_t row = 0;
      if (e >= 0) row = base[e] + rank;
      __syncwarp();
      if (e >= 0 && rank == 0) base[e] += __popc(peers);
      __syncwarp();
      if (e >= 0) {
        perm_token[row] = q / k;
        inv_perm[q] = row;
      }
    }
  }
}

}  // namespace moe
