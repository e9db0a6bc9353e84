// Quantile Balancing (QB) bias update, "Kimi K3: Open Frontier Intelligence",
// section "Systems Optimization, Load Balancing, and Post-Training
// Alignment": the router's per-expert biases come from the (1 - k/n)-quantile,
// over tokens, of the margins s[t,e] - alpha_t, alpha_t being token t's cutoff
// under top-(k+1) routing; the quantiles are recovered from per-expert binned
// histograms that data-parallel ranks add up with one integer all-reduce.
// The page's update formula is garbled; the reading taken (the dual step of
// the balanced-assignment LP the page names) is: alpha_t = (k+1)-th largest
// s[t,e] + b[e]; beta_e = the ceil(m k / n)-th largest margin of expert e;
// new bias b[e] = -beta_e, with beta_e taken at the lower edge of its bin.
//
// Arithmetic (fp32, every operation rounded as written, so that the counts
// are reproducible bit for bit):
//   v = s + b;  alpha = (k+1)-th largest v;  mu = s - alpha;  t = mu - lo;
//   bin = !(t >= 0) ? 0 : (t * inv_w >= B ? B - 1 : trunc(t * inv_w)),
//   so a NaN margin counts in bin 0 and +inf in bin B - 1,
//   inv_w = fp32(B) / fp32(hi - lo) (computed on the host).
// Three kernels: cutoffs (warp per token), histogram (CTA per 8 experts x a
// token slice, counts in shared memory, then added into H with 64-bit
// atomics), bias (warp per expert, a scan of the bins from the top).
#pragma once

#include <cstdint>

#include "common.cuh"
#include "router.cuh"  // float_order_key

namespace moe {

constexpr int kQbExpertsPerCta = 8;
constexpr int kQbMaxBins = 1536;  // 8 x 1536 x 4 bytes = 48 KB of shared counts

__device__ __forceinline__ float float_from_order_key(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// alpha[t] = (k+1)-th largest of s[t,e] + b[e] (b may be null), E <= 32 * MAXV.
// Warp per token; each of k rounds removes one copy of the current maximum
// (order keys: every finite value's key is above 0, which marks "removed").
template <int MAXV>
__global__ void __launch_bounds__(256)
    qb_cutoffs_kernel(const float* __restrict__ s, const float* __restrict__ b, int T, int E, int k,
                      float* __restrict__ alpha) {
  const int t = static_cast<int>(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5));
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  uint32_t key[MAXV];
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int e = i * 32 + lane;
    key[i] = e < E ? float_order_key(__fadd_rn(__ldg(s + static_cast<int64_t>(t) * E + e),
                                               b != nullptr ? __ldg(b + e) : 0.0f))
                   : 0u;
  }
  for (int r = 0; r <= k; ++r) {
    uint32_t lm = 0u;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) lm = max(lm, key[i]);
    const uint32_t m = __reduce_max_sync(0xffffffffu, lm);
    if (r == k) {
      if (lane == 0) alpha[t] = float_from_order_key(m);
      break;
    }
    int mine = 0x7fffffff;  // lowest index of this lane holding the maximum
#pragma unroll
    for (int i = MAXV - 1; i >= 0; --i)
      if (key[i] == m) mine = i * 32 + lane;
    const int win = __reduce_min_sync(0xffffffffu, mine);
#pragma unroll
    for (int i = 0; i < MAXV; ++i)
      if (i * 32 + lane == win) key[i] = 0u;
  }
}

// H[e][bin] += count of tokens t in this CTA's slice with the margin of
// expert e in that bin. Grid: (ceil(E / 8), token slices); 256 threads, thread
// (slot j = tid % 8, row tid / 8) takes expert e0 + j of tokens t0 + row,
// t0 + row + 32, ..., so the 8 logits of one token are read together.
// Dynamic shared memory: 8 * B * 4 bytes.
__global__ void __launch_bounds__(256)
    qb_histogram_kernel(const float* __restrict__ s, const float* __restrict__ alpha, int T, int E, float lo,
                        float inv_w, int B, int tokens_per_cta, unsigned long long* __restrict__ H) {
  extern __shared__ uint32_t qb_counts[];  // [8][B]
  const int e0 = blockIdx.x * kQbExpertsPerCta;
  const int t0 = blockIdx.y * tokens_per_cta;
  const int t1 = min(T, t0 + tokens_per_cta);
  for (int i = threadIdx.x; i < kQbExpertsPerCta * B; i += blockDim.x) qb_counts[i] = 0u;
  __syncthreads();
  const int j = threadIdx.x % kQbExpertsPerCta;
  const int e = e0 + j;
  if (e < E) {
    const float fB = static_cast<float>(B);
    for (int t = t0 + static_cast<int>(threadIdx.x) / kQbExpertsPerCta; t < t1; t += 32) {
      const float mu = __fsub_rn(__ldg(s + static_cast<int64_t>(t) * E + e), __ldg(alpha + t));
      const float tt = __fsub_rn(mu, lo);
      const float f = __fmul_rn(tt, inv_w);
      // a NaN margin (a NaN logit, or infinities that cancel) fails tt >= 0
      // and counts in bin 0, like a margin below lo
      const int bin = !(tt >= 0.0f) ? 0 : (f >= fB ? B - 1 : static_cast<int>(f));
      atomicAdd(&qb_counts[j * B + bin], 1u);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kQbExpertsPerCta * B; i += blockDim.x) {
    const int jj = i / B;
    if (e0 + jj < E && qb_counts[i] != 0u)
      atomicAdd(H + static_cast<int64_t>(e0 + jj) * B + (i - jj * B),
                static_cast<unsigned long long>(qb_counts[i]));
  }
}

// Per expert (warp per expert): the highest bin whose count from the top
// reaches r = ceil(m_total k / n), or bin 0; bias = -(lo + bin * w) in fp32.
__global__ void __launch_bounds__(256)
    qb_bias_kernel(const unsigned long long* __restrict__ H, int E, int B, float lo, float w, long long r,
                   int32_t* __restrict__ bins, float* __restrict__ bias) {
  const int e = static_cast<int>(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5));
  const int lane = threadIdx.x & 31;
  if (e >= E) return;
  const unsigned long long* h = H + static_cast<int64_t>(e) * B;
  unsigned long long run = 0ull;
  int found = -1;
  for (int top = B - 1; top >= 0 && found < 0; top -= 32) {
    const int bin = top - lane;  // lane 0 takes the highest bin of this group
    unsigned long long v = bin >= 0 ? h[bin] : 0ull;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    const unsigned int hit = __ballot_sync(0xffffffffu, bin >= 0 && run + v >= static_cast<unsigned long long>(r));
    if (hit != 0u) found = top - (__ffs(hit) - 1);
    run += __shfl_sync(0xffffffffu, v, 31);
  }
  if (found < 0) found = 0;
  if (lane == 0) {
    bins[e] = found;
    bias[e] = -__fadd_rn(lo, __fmul_rn(static_cast<float>(found), w));
  }
}

}  // namespace moe
