// Few-token router: logits, softmax over all experts and top-k for T <= 16
// tokens (one launch for T = 1), the decode regime where the step reads the
// whole fp32 gate matrix W_router[d, E] for a handful of rows and is bound by
// that read.
//
// Same gate and numerics as router.cuh (one linear map d -> E, softmax over
// the expert axis, top-k of the probabilities without renormalisation, as in
// the gating code on "Kimi K3: The Open Model That Just Cornered the AI
// Frontier", section "Mixture-of-Experts with Dynamic Load Balancing"), and
// the same fixed fp32 order, so the logits are bit-identical to the other
// router kernels:
//   p_c = fma chain over the 128 input indices of chunk c, from +0, ascending;
//   l   = ((p_0 + p_1) + ...) + p_{C-1}, then + b_e.
//
// Layout of the work: CTA (g, c) owns experts [128 g, 128 g + 128) and input
// chunk c. It pulls its W tile (<= 128 rows of <= 512 bytes) into shared
// memory with one bulk copy per row, all issued up front on one mbarrier, so
// the whole matrix is in flight at once across the grid; widens its chunk of
// x for every token; and writes p_c for every (token, expert) it owns.
// With one token the same launch finishes the job: the last CTA of expert
// group g to finish (an atomic ticket, after a fence) adds the group's C
// partials in ascending c (+ bias) into the final logits; the last group to
// finish then takes softmax and top-k with all 256 threads. Which CTA does a
// reduction depends on timing, but every sum is taken in the fixed order, so
// the results are deterministic. The tickets must be zero at launch; the last
// CTAs put them back to zero. With more tokens the kernel writes the partials
// only and router_reduce_topk_kernel follows.
#pragma once

#include <cstdint>

#include "common.cuh"
#include "ptx.cuh"
#include "router.cuh"

namespace moe {

constexpr int kRsExperts = 128;  // experts per CTA
constexpr int kRsRows = 128;     // input indices per CTA (one chunk)
constexpr int kRsThreads = 256;
constexpr int kRsMaxTokens = 16;

__host__ __device__ constexpr int router_stream_smem_bytes(int tmax) {
  return kRsRows * kRsExperts * 4 + kRsRows * tmax * 4;
}

// The dispatch tables of a one-token step, written by the router's last CTA
// when offsets != nullptr (the same values the dispatch kernels would write:
// with one token every selected expert has exactly one row, in ascending
// expert order): expert offsets and both GEMM token-block prefixes
// (offsets[e] = prefix[e] = number of selected experts below e), perm_token
// (all token 0), inv_perm (the row of each slot); zero_n words of zero_buf are
// cleared (the feed-forward's tickets and counters), by all CTAs at the start.
struct RouteDispatch {
  int32_t* offsets;
  int32_t* perm_token;
  int32_t* inv_perm;
  int32_t* prefix0;
  int32_t* prefix1;
  unsigned int* zero_buf;
  int zero_n;
};

// The end of a one-token route, by one CTA of 256 threads once all E logits
// are in global memory: softmax and top-k, and, when disp.offsets != nullptr,
// the dispatch tables of the step.
__device__ __forceinline__ void one_token_finish(const float* logits, int E, int k, int32_t* topk_idx,
                                                 float* topk_w, const RouteDispatch& disp) {
  __shared__ float s_l[1024];
  __shared__ int32_t s_sel[16];
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += 256) s_l[e] = __ldcg(logits + e);
  __syncthreads();
  cta_softmax_topk_256(s_l, E, k, topk_idx, topk_w);
  if (disp.offsets == nullptr) return;
  __syncthreads();  // the selection (written by warp 0) is visible to the CTA
  if (tid < k) s_sel[tid] = __ldcg(topk_idx + tid);
  __syncthreads();
  for (int e = tid; e <= E; e += 256) {
    int32_t below = 0;
    for (int j = 0; j < k; ++j) below += (s_sel[j] < e) ? 1 : 0;
    disp.offsets[e] = below;
    disp.prefix0[e] = below;
    disp.prefix1[e] = below;
  }
  if (tid < k) {
    int32_t row = 0;
    for (int j = 0; j < k; ++j) row += (s_sel[j] < s_sel[tid]) ? 1 : 0;
    disp.perm_token[tid] = 0;
    disp.inv_perm[tid] = row;
  }
}

template <int TMAX>
__global__ void __launch_bounds__(kRsThreads)
    router_stream_kernel(const uint16_t* __restrict__ x, const float* __restrict__ W, const float* __restrict__ bias,
                         int T, int d, int E, int k, float* __restrict__ part, float* __restrict__ logits,
                         unsigned int* __restrict__ tickets, int32_t* __restrict__ topk_idx,
                         float* __restrict__ topk_w, const RouteDispatch disp) {
  static_assert(TMAX == 1 || TMAX == 4 || TMAX == 16, "token tile");
  extern __shared__ __align__(128) uint8_t rs_smem[];
  float* ws = reinterpret_cast<float*>(rs_smem);  // [kRsRows][kRsExperts]
  float* xs = ws + kRsRows * kRsExperts;          // [kRsRows][TMAX]
  __shared__ __align__(8) uint64_t bar;
  __shared__ unsigned int s_ticket;

  const int g = blockIdx.x, c = blockIdx.y;
  const int G = gridDim.x, C = gridDim.y;
  const int e0 = g * kRsExperts;
  const int ne = min(kRsExperts, E - e0);  // a multiple of 4 (E % 4 == 0)
  const int r0 = c * kRsRows;
  const int nr = min(kRsRows, d - r0);     // 128, or 64 for the last chunk when d % 128 == 64
  const int tid = threadIdx.x;

  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  if (TMAX == 1 && disp.zero_buf != nullptr) {
    // the feed-forward's counters, cleared by all CTAs at once (only the next
    // launch reads them)
    const int64_t nth = static_cast<int64_t>(G) * C * kRsThreads;
    for (int64_t i = (static_cast<int64_t>(c) * G + g) * kRsThreads + tid; i < disp.zero_n; i += nth)
      disp.zero_buf[i] = 0u;
  }
  __syncthreads();
  if (tid == 0) mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(nr * ne * 4));
  __syncthreads();
  {
    const uint64_t pol = l2_policy_evict_first();  // read once per call
    for (int r = tid; r < nr; r += kRsThreads)
      bulk_load(ws + r * kRsExperts, W + static_cast<int64_t>(r0 + r) * E + e0, static_cast<uint32_t>(ne * 4), &bar,
                pol);
  }
  // the chunk of x for every token, widened exactly: xs[i][t]
  for (int v = tid; v < TMAX * (kRsRows / 8); v += kRsThreads) {
    const int t = v / (kRsRows / 8), q = v % (kRsRows / 8);
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (t < T && q * 8 < nr) u = *reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * d + r0 + q * 8);
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      xs[(q * 8 + 2 * h) * TMAX + t] = __uint_as_float(w4[h] << 16);
      xs[(q * 8 + 2 * h + 1) * TMAX + t] = __uint_as_float(w4[h] & 0xFFFF0000u);
    }
  }
  __syncthreads();
  if (!mbar_wait_bounded(&bar, 0u, kWaitLimitNs, nullptr)) {
    record_device_error(6u /* MOE_DEVERR_WAIT_TIMEOUT_ROUTER */);
    return;
  }

  // p_c for experts e0 + 2p, e0 + 2p + 1 and tokens q*TS .. q*TS + TS - 1
  constexpr int NS = TMAX >= 4 ? 4 : 1;
  constexpr int TS = TMAX / NS;
  const int p = tid & 63, q = tid >> 6;
  if (q < NS && 2 * p < ne) {
    float acc[TS][2];
#pragma unroll
    for (int j = 0; j < TS; ++j) acc[j][0] = acc[j][1] = 0.0f;
#pragma unroll 8
    for (int i = 0; i < nr; ++i) {
      const float2 w2 = *reinterpret_cast<const float2*>(ws + i * kRsExperts + 2 * p);
      float xv[TS];
      if constexpr (TS >= 4) {
#pragma unroll
        for (int j = 0; j < TS; j += 4) {
          const float4 x4 = *reinterpret_cast<const float4*>(xs + i * TMAX + q * TS + j);
          xv[j] = x4.x, xv[j + 1] = x4.y, xv[j + 2] = x4.z, xv[j + 3] = x4.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < TS; ++j) xv[j] = xs[i * TMAX + q * TS + j];
      }
#pragma unroll
      for (int j = 0; j < TS; ++j) {
        acc[j][0] = __fmaf_rn(xv[j], w2.x, acc[j][0]);
        acc[j][1] = __fmaf_rn(xv[j], w2.y, acc[j][1]);
      }
    }
#pragma unroll
    for (int j = 0; j < TS; ++j) {
      const int t = q * TS + j;
      if (t < T)
        *reinterpret_cast<float2*>(part + (static_cast<int64_t>(c) * T + t) * E + e0 + 2 * p) =
            make_float2(acc[j][0], acc[j][1]);
    }
  }

  // Several tokens: the ordered sums, softmax and top-k run as a second launch
  // (router_reduce_topk_kernel, one CTA per token), which spreads the T x E x C
  // partial reads and the T top-k selections over the whole GPU.
  if constexpr (TMAX > 1) return;

  // One token: the last CTA of this expert group adds the group's partials in
  // chunk order
  __threadfence();
  __syncthreads();
  if (tid == 0) s_ticket = atomicAdd(&tickets[g], 1u);
  __syncthreads();
  if (s_ticket != static_cast<unsigned int>(C - 1)) return;
  __threadfence();
  if (tid < ne) {
    // one expert per thread; 28 chunk partials in flight, then the ordered adds
    const int e = e0 + tid;
    const float* src = part + e;  // token 0; plane c at src + c * E
    float l = __ldcg(src);
    for (int c0 = 1; c0 < C; c0 += 28) {
      float pv[28];
#pragma unroll
      for (int u = 0; u < 28; ++u) pv[u] = (c0 + u < C) ? __ldcg(src + static_cast<int64_t>(c0 + u) * E) : 0.0f;
#pragma unroll
      for (int u = 0; u < 28; ++u)
        if (c0 + u < C) l = __fadd_rn(l, pv[u]);
    }
    if (bias != nullptr) l = __fadd_rn(l, __ldg(bias + e));
    logits[e] = l;
  }

  // the last group to finish takes softmax and top-k with the whole CTA
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    tickets[g] = 0u;
    s_ticket = atomicAdd(&tickets[G], 1u);
  }
  __syncthreads();
  if (s_ticket != static_cast<unsigned int>(G - 1)) return;
  __threadfence();
  if (tid == 0) tickets[G] = 0u;
  one_token_finish(logits, E, k, topk_idx, topk_w, disp);
}


// One-token router without cross-CTA partial sums, for d <= kR1MaxD: CTA g
// owns experts [8 g, 8 g + 8) and streams all d rows of W_router for them
// (TMA boxes of 8 experts x 256 rows, fp32, 32 KB stages of 1024 rows in a
// ring of four). The 256 threads form four groups of 64; group q takes the
// stages q, q + 4, ... (ring slot q), and thread (c, e) of a group runs the
// fma chain of chunk c (128 rows) of that stage for expert e, in the stated
// order. When a group has read its slot it loads the slot's next stage
// itself. Each CTA then adds its experts' C chunk sums in chunk order (+ bias)
// and writes the final logits; the last CTA to finish (a ticket) takes the
// softmax, the top-k and the dispatch tables. Same arithmetic and order as
// the other router kernels, so the logits are bit-identical; two dependent
// rounds of global partial sums fewer than router_stream_kernel<1>.
constexpr int kR1Experts = 8;
constexpr int kR1StageRows = 1024;
constexpr int kR1BoxRows = 256;
constexpr int kR1Slots = 4;
constexpr int kR1MaxD = 8192;
// x is widened into shared memory with 8 floats of padding after every
// 128-value chunk, so the four chunks a warp reads at once sit in different
// banks.
__host__ __device__ constexpr int router_one_x_floats() { return kR1MaxD + (kR1MaxD / 128) * 8; }
__host__ __device__ constexpr int router_one_smem_bytes() {
  return kR1Slots * kR1StageRows * kR1Experts * 4 + router_one_x_floats() * 4 + (kR1MaxD / 128) * kR1Experts * 4;
}

// The logits of experts [e0, e0 + 8) of one token, by threads 0..255 of the
// calling CTA (every one of them calls it; tid = threadIdx.x). `sm` holds
// router_one_smem_bytes() of shared memory (W ring, widened x, chunk sums) and
// full[kR1Slots] are mbarriers initialised to count 1 and fenced by the caller.
// Named barriers 1..5 are used. A warp's 32 threads are four chunks x eight
// experts, and chunk c of a group starts its chain c steps after chunk 0, so at
// each step the four chunks read rows in four different bank groups (every
// chain still runs over its rows in ascending order). Returns false when a
// wait for W gave up (MOE_DEVERR_WAIT_TIMEOUT_ROUTER recorded).
__device__ __forceinline__ bool router_one_token_logits(const CUtensorMap* tmW, const uint16_t* __restrict__ x,
                                                        const float* __restrict__ bias, int d, int E, int e0,
                                                        uint8_t* sm, uint64_t* full, float* __restrict__ logits) {
  float* ws = reinterpret_cast<float*>(sm);                      // [slot][1024 rows][8 experts]
  float* xs = ws + kR1Slots * kR1StageRows * kR1Experts;         // x widened, chunk c at 136 c
  float* part = xs + router_one_x_floats();                      // chunk sums [C][8]
  const int tid = threadIdx.x;
  const int nst = (d + kR1StageRows - 1) / kR1StageRows;
  const int C = (d + 127) / 128;
  // stage j into slot j % 4: its boxes of 256 rows that start inside d
  auto issue = [&](int j) {
    const int slot = j % kR1Slots;
    const int r0 = j * kR1StageRows;
    const int nbox = min(kR1StageRows / kR1BoxRows, (d - r0 + kR1BoxRows - 1) / kR1BoxRows);
    mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nbox * kR1BoxRows * kR1Experts * 4));
    for (int b = 0; b < nbox; ++b)
      tma_load_2d(ws + (slot * kR1StageRows + b * kR1BoxRows) * kR1Experts, tmW, &full[slot], e0,
                  r0 + b * kR1BoxRows, l2_policy_evict_first());
  };
  if (tid == 0)
    for (int j = 0; j < kR1Slots && j < nst; ++j) issue(j);
  for (int v = tid; v < d / 8; v += 256) {
    const uint4 u = *reinterpret_cast<const uint4*>(x + v * 8);
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
    float* dst = xs + v * 8 + (v >> 4) * 8;  // 16 vectors of 8 per 128-value chunk
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      dst[2 * h] = __uint_as_float(w4[h] << 16);
      dst[2 * h + 1] = __uint_as_float(w4[h] & 0xFFFF0000u);
    }
  }
  FirstWarps8Sync()();
  const int grp = tid >> 6, t = tid & 63, cl = t >> 3, e = t & 7;
  const int skew = cl & 3;  // the chunk's place among the warp's four
  bool ok = true;
  for (int j = grp; j < nst; j += kR1Slots) {
    if (ok && !mbar_wait_bounded(&full[grp], static_cast<uint32_t>((j / kR1Slots) & 1), kWaitLimitNs, nullptr)) {
      record_device_error(6u /* MOE_DEVERR_WAIT_TIMEOUT_ROUTER */);
      ok = false;
    }
    const int row0 = j * kR1StageRows + cl * 128;
    if (ok && row0 < d) {
      const int nr = min(128, d - row0);
      const float* wp = ws + (grp * kR1StageRows + cl * 128) * kR1Experts + e;
      const float* xp = xs + row0 + (row0 >> 7) * 8;
      // step s reads row s - skew: steps skew..2, then 3..nr-1 for every
      // chunk of the warp at once, then nr..nr+skew-1
      const float* xq = xp - skew;
      const float* wq = wp - skew * kR1Experts;
      float acc = 0.0f;
      for (int s = skew; s < 3; ++s) acc = __fmaf_rn(xq[s], wq[s * kR1Experts], acc);
#pragma unroll 8
      for (int s = 3; s < nr; ++s) acc = __fmaf_rn(xq[s], wq[s * kR1Experts], acc);
      for (int s = nr; s < nr + skew; ++s) acc = __fmaf_rn(xq[s], wq[s * kR1Experts], acc);
      part[(j * (kR1StageRows / 128) + cl) * kR1Experts + e] = acc;
    }
    // the group has read its slot: load the slot's next stage
    asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(64) : "memory");
    if (t == 0 && j + kR1Slots < nst) {
      fence_proxy_async_shared();
      issue(j + kR1Slots);
    }
  }
  FirstWarps8Sync()();
  if (tid < kR1Experts && e0 + tid < E) {
    float l = part[tid];
    for (int c = 1; c < C; ++c) l = __fadd_rn(l, part[c * kR1Experts + tid]);
    if (bias != nullptr) l = __fadd_rn(l, __ldg(bias + e0 + tid));
    logits[e0 + tid] = l;
  }
  return ok;
}

__global__ void __launch_bounds__(256)
    router_one_token_kernel(const __grid_constant__ CUtensorMap tmW, const uint16_t* __restrict__ x,
                            const float* __restrict__ bias, int d, int E, int k, float* __restrict__ logits,
                            unsigned int* __restrict__ tickets, int32_t* __restrict__ topk_idx,
                            float* __restrict__ topk_w, const RouteDispatch disp) {
  extern __shared__ __align__(128) uint8_t r1_smem[];
  __shared__ __align__(8) uint64_t full[kR1Slots];
  __shared__ unsigned int s_ticket;
  const int g = blockIdx.x, G = gridDim.x, tid = threadIdx.x;
  if (disp.zero_buf != nullptr) {
    // the feed-forward's counters, cleared by all CTAs at once (only the next
    // launch reads them)
    for (int64_t i = static_cast<int64_t>(g) * 256 + tid; i < disp.zero_n; i += static_cast<int64_t>(G) * 256)
      disp.zero_buf[i] = 0u;
  }
  if (tid == 0) {
    for (int s = 0; s < kR1Slots; ++s) mbar_init(&full[s], 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
  }
  __syncthreads();
  router_one_token_logits(&tmW, x, bias, d, E, g * kR1Experts, r1_smem, full, logits);
  __threadfence();
  __syncthreads();
  if (tid == 0) s_ticket = atomicAdd(&tickets[0], 1u);
  __syncthreads();
  if (s_ticket != static_cast<unsigned int>(G - 1)) return;
  __threadfence();
  if (tid == 0) tickets[0] = 0u;
  one_token_finish(logits, E, k, topk_idx, topk_w, disp);
}

}  // namespace moe
