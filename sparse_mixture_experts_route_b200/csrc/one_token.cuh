// The whole layer for one token in one cooperative launch: router, dispatch,
// both expert GEMMs and the combine ("Kimi K3: Open Frontier Intelligence",
// section "Operational Execution Flow": 896 experts, 16 active per token; the
// gate, its softmax and the unnormalised top-k as in the gating code on "Kimi
// K3: The Open Model That Just Cornered the AI Frontier", section
// "Mixture-of-Experts with Dynamic Load Balancing").
//
// A one-token step streams the router matrix and then k experts' weights; as
// separate launches each step pays its own start-up and drain. Here one CTA
// per SM runs, in order:
//   1. the logits of eight experts (router_one_token_logits: all d rows of
//      W_router for those experts, streamed through the stage ring; CTAs past
//      E / 8 only wait), into a global [E] array;
//   2. a grid barrier (a count of arrived CTAs, bounded wait);
//   3. the top-k of all E logits in every CTA (the same code on the same
//      values, so every CTA selects the same experts), and the dispatch tables
//      in shared memory: every selected expert has one row, in ascending
//      expert order;
//   4. the CTA's share of the chunk-queue feed-forward (fused_cta_run: gate/up
//      chunks, then down chunks, taken from one queue), the token operand of
//      the gate/up GEMM read straight from x; the epilogue warps first take the
//      softmax statistics and the k weights, which only the combine needs;
//   5. a second grid barrier, then the combine out = sum_j w_j y_row(j) (fp32
//      fma in slot order, one rounding), its 16-byte vectors spread over all
//      CTAs.
// The arithmetic and its order are those of the separate launches (router,
// feed-forward, combine), so the output is bit-identical to theirs. The TMEM
// allocation, barrier set-up and descriptor prefetches of step 4 happen
// before step 1. Both barrier counts must be zero at launch.
#pragma once

#include <cstdint>

#include "common.cuh"
#include "expert_gemm.cuh"
#include "ptx.cuh"
#include "router.cuh"
#include "router_stream.cuh"

namespace moe {

constexpr int kOneTokenMaxK = 16;
static_assert(router_one_smem_bytes() <= GemmCfg<1>::kStages * GemmCfg<1>::kStageBytes,
              "the router's shared memory fits in the feed-forward's stage ring");
static_assert(kR1Slots <= kFusedAuxBars, "router barriers");
// the one-token kernel's dynamic shared memory: the feed-forward's layout,
// then the E <= 1024 logits (kept until the epilogue warps have taken the
// weights), plus the slack for aligning the base to 1024 bytes
constexpr int kOtLogitsOffset = (GemmCfg<1>::kStages * GemmCfg<1>::kStageBytes + kFusedBarrierBytes +
                                 kFusedQueue * 4 + 3 * (1024 + 1) * 4 + 15) / 16 * 16;
constexpr int kOneTokenSmemBytes = kOtLogitsOffset + 1024 * 4 + 1024;
static_assert(kOneTokenSmemBytes <= 232448 - 4096, "shared memory per CTA (dynamic + static)");

struct OneTokenArgs {
  const uint16_t* x;          // [d] bf16
  const float* bias;          // [E] or null
  int d, E, k;
  float* logits;              // [E] (written in step 1)
  unsigned int* sync;         // [2] CTAs past step 1 / past step 4; zero at launch
  int32_t* topk_idx;          // [k] written by CTA 0 (the step's routing, kept in the workspace)
  float* topk_w;              // [k]
  int32_t* inv_perm;          // [k]
  unsigned int* zero_buf;     // the feed-forward's tickets and counters, cleared before the first barrier
  int zero_n;
  unsigned int* h_ready;      // [E]
  unsigned int* claim;        // the chunk counter
  uint16_t* out;              // [d] bf16
};

// Spins until *count reaches target, for at most kWaitLimitNs; false if the
// limit ran out.
__device__ __forceinline__ bool wait_count_bounded(const unsigned int* count, unsigned int target) {
  if (ld_acquire_gpu(count) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  while (ld_acquire_gpu(count) < target)
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

// Warps 2..9 (the epilogue warps) as one group of 256 threads.
struct EpilogueWarpsSync {
  __device__ __forceinline__ void operator()() const { asm volatile("bar.sync 6, 256;" ::: "memory"); }
};

__global__ void __launch_bounds__(kGemmThreads, 1)
    moe_one_token_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA0,
                         const __grid_constant__ CUtensorMap tmBs0, const __grid_constant__ CUtensorMap tmA1,
                         const __grid_constant__ CUtensorMap tmBs1, const GemmParams p0, const GemmParams p1,
                         const OneTokenArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int32_t s_idx[kOneTokenMaxK];
  __shared__ float s_w[kOneTokenMaxK];
  __shared__ int32_t s_row[kOneTokenMaxK];
  __shared__ int s_fail;
  const FusedCta fc = fused_cta_layout(smem_raw, a.E);
  float* s_l = reinterpret_cast<float*>(fc.smem + kOtLogitsOffset);  // after the tables
  const int tid = threadIdx.x, warp = tid >> 5;
  const unsigned int G = gridDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + tid; i < a.zero_n;
       i += static_cast<int64_t>(G) * blockDim.x)
    a.zero_buf[i] = 0u;
  fused_cta_setup(fc, &tmA0, &tmBs0, &tmA1, &tmBs1);
  if (tid == 0) {
    s_fail = 0;
    tma_prefetch_desc(&tmW);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();

  // 1. the logits of experts 8 g .. 8 g + 7 (threads 0..255; W ring in the stage ring)
  if (static_cast<int>(blockIdx.x) < ceil_div(a.E, kR1Experts) && tid < 256) {
    if (!router_one_token_logits(&tmW, a.x, a.bias, a.d, a.E, static_cast<int>(blockIdx.x) * kR1Experts, fc.smem,
                                 fc.aux_bar, a.logits))
      s_fail = 1;
  }
  // 2. every CTA's logits (and cleared counters) are out
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    atomicAdd(a.sync, 1u);
    if (!wait_count_bounded(a.sync, G)) {
      record_device_error(7u /* MOE_DEVERR_WAIT_TIMEOUT_DEPENDENCY */);
      s_fail = 1;
    }
  }
  __syncthreads();

  // 3. top-k (threads 0..255; the weights come later), then the dispatch tables
  if (tid < 256) {
    for (int e = tid; e < a.E; e += 256) s_l[e] = __ldcg(a.logits + e);
    FirstWarps8Sync()();
    if (!cta_topk_histogram_256(s_l, a.E, a.k, 0.0f, 1.0f, s_idx, nullptr, FirstWarps8Sync()))
      cta_topk_rounds_256(s_l, a.E, a.k, 0.0f, 1.0f, s_idx, nullptr, FirstWarps8Sync());
  }
  __syncthreads();
  for (int e = tid; e <= a.E; e += blockDim.x) {
    int32_t below = 0;
    for (int j = 0; j < a.k; ++j) below += (s_idx[j] < e) ? 1 : 0;
    fc.s_off[e] = below;
    fc.s_pre0[e] = below;
    fc.s_pre1[e] = below;
  }
  if (tid < a.k) {
    int32_t row = 0;
    for (int j = 0; j < a.k; ++j) row += (s_idx[j] < s_idx[tid]) ? 1 : 0;
    s_row[tid] = row;
    if (blockIdx.x == 0) {
      a.topk_idx[tid] = s_idx[tid];
      a.inv_perm[tid] = row;
    }
  }
  fence_proxy_async_shared();  // the ring held the router's chunk sums; TMA fills it next
  __syncthreads();

  // 4. both expert GEMMs; the epilogue warps first take the softmax
  // statistics and the weights of the k selected experts
  if (warp >= 2) {
    float M, S;
    cta_softmax_stats_256(s_l, a.E, &M, &S, EpilogueWarpsSync(), tid - 64);
    if (tid - 64 < a.k) {
      const float wj = softmax_weight(s_l[s_idx[tid - 64]], M, S);
      s_w[tid - 64] = wj;
      if (blockIdx.x == 0) a.topk_w[tid - 64] = wj;
    }
  }
  if (!s_fail) fused_cta_run(fc, &tmA0, &tmBs0, &tmA1, &tmBs1, p0, p1, a.h_ready, a.claim);
  fused_cta_teardown(fc);

  // 5. the combine, once every CTA's rows of y are stored
  if (tid == 0) {
    __threadfence();
    atomicAdd(a.sync + 1, 1u);
    if (!wait_count_bounded(a.sync + 1, G)) {
      record_device_error(7u /* MOE_DEVERR_WAIT_TIMEOUT_DEPENDENCY */);
      s_fail = 1;
    }
  }
  __syncthreads();
  if (s_fail) return;
  const int vpr = a.d / 8;
  const uint4* y = reinterpret_cast<const uint4*>(p1.out);
  for (int v = static_cast<int>(blockIdx.x) + static_cast<int>(G) * tid; v < vpr;
       v += static_cast<int>(G * blockDim.x)) {
    uint4 yv[kOneTokenMaxK];
#pragma unroll
    for (int j = 0; j < kOneTokenMaxK; ++j)
      if (j < a.k) yv[j] = __ldcg(y + static_cast<int64_t>(s_row[j]) * vpr + v);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < kOneTokenMaxK; ++j) {
      if (j < a.k) {
        const float wj = s_w[j];
        const uint32_t yw[4] = {yv[j].x, yv[j].y, yv[j].z, yv[j].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[2 * q] = __fmaf_rn(wj, __uint_as_float(yw[q] << 16), acc[2 * q]);
          acc[2 * q + 1] = __fmaf_rn(wj, __uint_as_float(yw[q] & 0xFFFF0000u), acc[2 * q + 1]);
        }
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat162 pr = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
      o[q] = *reinterpret_cast<const uint32_t*>(&pr);
    }
    reinterpret_cast<uint4*>(a.out)[v] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace moe
