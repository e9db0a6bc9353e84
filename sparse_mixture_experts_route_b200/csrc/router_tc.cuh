// Router for many tokens: tensor-core screening plus an exact re-check.
//
// Computes the same routing as router.cuh (the gate of "Kimi K3: The Open Model
// That Just Cornered the AI Frontier", section "Mixture-of-Experts with Dynamic
// Load Balancing": softmax over all experts, top-k, unnormalised values) and the
// same bits, in less time when T * E is large:
//
//  1. prep: W_router [d, E] fp32 -> a chunk-interleaved exact copy Wc
//     [E][128][32][2] fp32 (offset j of chunks l and l + 32 side by side) and
//     Wt_hi / Wt_lo [E, d] bf16 with Wt_hi = bf16(W), Wt_lo = bf16(W - Wt_hi),
//     so |W - Wt_hi - Wt_lo| <= 2^-17 |W|; an upper bound of each column norm
//     ||W_e||_2 and of each token norm ||x_t||_2.
//  2. screen: A[t, e] = x_t . Wt_hi[e] + x_t . Wt_lo[e] (+ b_e) on tcgen05
//     (bf16 x bf16 products are exact in fp32; fp32 accumulation in TMEM), with
//     the K range split over CTAs and the partials added in a fixed order.
//  3. re-check, per token: tau = k-th largest A; every expert with
//     A_e >= tau - 2 eps_t is a candidate, where eps_t bounds |A - L| for the
//     exact-order fp32 logit L (below); each candidate's L is recomputed in the
//     stated order (fma chains over 128-index chunks, chunks added in order,
//     bias last) and the top-k is taken over the candidates by L (ties -> lower
//     index). Any expert outside the window has L < tau - eps_t, while the k
//     experts with the largest A all have L >= tau - eps_t, so it cannot be
//     selected: the result equals the exact-order routing.
//     Weights: exp(L_j - m) / s with m = max_e A_e and s the sum of exp(L_e - m)
//     over the candidates plus exp(A_e - m) over the other experts.
//
// eps_t = 2^-11 ||x_t||_2 max_e ||W_e||_2 + 2^-20 (|A| + |b|)_max bound: the
// Cauchy-Schwarz bound on sum_i |x_i W_ie| times a relative accumulation error
// of 2^-11, about four times the worst case of fp32 accumulation with
// truncation over d/16 MMA steps of 16 products (d = 7168) plus the rounding
// of the exact-order sum itself. If more than kMaxCand experts fall in the
// window (never seen on the workloads), every expert of that token is
// recomputed, which is exact but slow.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "router.cuh"

namespace moe {

constexpr int kRtBK = 64;          // K per stage
constexpr int kRtThreads = 192;    // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kMaxCand = 32;       // candidate window capacity per token
constexpr float kRtEpsRel = 1.0f / 2048.0f;

// ---------------------------------------------------------------- 1. prep

// W [d, E] -> Wt_hi / Wt_lo [E, d] (bf16, K-major for the screen), and fp64
// partial sums of squares of each column over this block's 256 input indices:
// part[blockIdx.y][e]. Block (32, 8): a 32-expert x 256-index slab, transposed
// through shared memory.
__global__ void __launch_bounds__(256)
    router_prep_kernel(const float* __restrict__ W, int d, int E, uint16_t* __restrict__ Wt_hi,
                       uint16_t* __restrict__ Wt_lo, double* __restrict__ part) {
  __shared__ float tile[256][33];  // the whole 256 (i) x 32 (e) slab, padded
  __shared__ double ssq[8][32];
  const int e0 = blockIdx.x * 32, i0 = blockIdx.y * 256;
  const int tx = threadIdx.x, ty = threadIdx.y;
  // load the slab, coalesced along e, every load of the thread in flight at once;
  // thread (tx, ty) sums the squares of rows ty, ty + 8, ... of column e0 + tx
  double acc = 0.0;
#pragma unroll
  for (int r = ty; r < 256; r += 8) {
    const int i = i0 + r, e = e0 + tx;
    const float v = (i < d && e < E) ? __ldg(W + static_cast<int64_t>(i) * E + e) : 0.0f;
    tile[r][tx] = v;
    acc += static_cast<double>(v) * static_cast<double>(v);
  }
  __syncthreads();
  // store transposed: rows e, coalesced along i
#pragma unroll
  for (int r = ty; r < 32; r += 8) {
    const int e = e0 + r;
    if (e >= E) continue;
#pragma unroll
    for (int sub = 0; sub < 8; ++sub) {
      const int i = i0 + sub * 32 + tx;
      if (i < d) {
        const float v = tile[sub * 32 + tx][r];
        const int64_t at = static_cast<int64_t>(e) * d + i;
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
        Wt_hi[at] = *reinterpret_cast<const uint16_t*>(&hi);
        Wt_lo[at] = *reinterpret_cast<const uint16_t*>(&lo);
      }
    }
  }
  ssq[ty][tx] = acc;  // column e0 + tx, rows ty, ty + 8, ... of this slab
  __syncthreads();
  if (ty == 0 && e0 + tx < E) {
    double s = 0.0;
    for (int r = 0; r < 8; ++r) s += ssq[r][tx];
    part[static_cast<int64_t>(blockIdx.y) * E + e0 + tx] = s;
  }
}

// W [d, E] -> Wc [E][128][32][2] fp32: Wc[e][j][l][h] = W[128 c + j][e] for
// chunk c = 32 h + l (0 past d). For one expert and one offset j inside a
// chunk, lane l of a warp reads chunks l and l + 32 with one 8-byte load.
// Block (32, 8) handles 32 experts x 4 offsets j x all chunks (C <= 64).
__global__ void __launch_bounds__(256)
    router_interleave_kernel(const float* __restrict__ W, int d, int E, int C, float* __restrict__ Wc) {
  __shared__ float tile[4][64][33];  // [j][c][e]
  const int e0 = blockIdx.x * 32, j0 = blockIdx.y * 4;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int rc = ty; rc < 4 * 64; rc += 8) {
    const int j = rc / 64, c = rc - j * 64;
    const int i = c * 128 + j0 + j, e = e0 + tx;
    tile[j][c][tx] = (c < C && i < d && e < E) ? __ldg(W + static_cast<int64_t>(i) * E + e) : 0.0f;
  }
  __syncthreads();
  for (int r = ty; r < 32 * 4; r += 8) {
    const int el = r / 4, j = r % 4, e = e0 + el;
    if (e >= E) continue;
    float2* dst = reinterpret_cast<float2*>(Wc + (static_cast<int64_t>(e) * 128 + j0 + j) * 64);
    dst[tx] = make_float2(tile[j][tx][el], tile[j][tx + 32][el]);
  }
}

// wnorm[e] >= ||W_e||_2 (fp64 sum of the partials, rounded up to fp32), and
// wnorm[E] = max_e wnorm[e]. One block of up to 1024 threads.
__global__ void __launch_bounds__(1024)
    router_wnorm_kernel(const double* __restrict__ part, int nparts, int E, float* __restrict__ wnorm) {
  __shared__ float red[32];
  float mx = 0.0f;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    double s = 0.0;
    for (int p = 0; p < nparts; ++p) s += part[static_cast<int64_t>(p) * E + e];
    const float n = __double2float_ru(sqrt(s) * (1.0 + 1e-12));
    wnorm[e] = n;
    mx = fmaxf(mx, n);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = (threadIdx.x < (blockDim.x + 31) / 32) ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (threadIdx.x == 0) wnorm[E] = v;
  }
}

// xnorm[t] >= ||x_t||_2: warp per token, fp32 sum of squares scaled up by
// (1 + 2^-10), which exceeds the relative error of the fp32 sum for d <= 32768.
// Also resets the re-check's overflow counter.
__global__ void __launch_bounds__(256)
    router_xnorm_kernel(const uint4* __restrict__ x, int T, int vec_per_row, float* __restrict__ xnorm,
                        int32_t* __restrict__ overflow) {
  if (blockIdx.x == 0 && threadIdx.x == 0) overflow[0] = 0;  // the re-check appends to it
  const int t = static_cast<int>(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5));  // no overflow for T < 2^31
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  float s = 0.0f;
  for (int v = lane; v < vec_per_row; v += 32) {
    const uint4 q = __ldg(x + static_cast<int64_t>(t) * vec_per_row + v);
    const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = __uint_as_float(w4[j] << 16), b = __uint_as_float(w4[j] & 0xFFFF0000u);
      s = fmaf(a, a, s);
      s = fmaf(b, b, s);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) xnorm[t] = __fsqrt_ru(s * (1.0f + 1.0f / 1024.0f));
}

// -------------------------------------------------------------- 2. screen

// Apart[s][t][e] = sum over the s-th K range of x_t . (Wt_hi[e] + Wt_lo[e]),
// fp32, for one tile of 128 experts (UMMA M, A operand) x 256 tokens (N, B
// operand) per CTA; the K ranges are summed in order by the re-check. Both
// operands K-major with 128-byte swizzle; two MMAs (hi, lo) per K step into one
// accumulator of 256 TMEM columns.
constexpr int kScrE = 128;           // experts per tile
constexpr int kScrT = 256;           // tokens per tile
constexpr int kScrStages = 3;
constexpr int kScrStageBytes = 2 * kScrE * kRtBK * 2 + kScrT * kRtBK * 2;  // 64 KB
constexpr int kScrSmemBytes = kScrStages * kScrStageBytes + 256 + 1024;

__global__ void __launch_bounds__(kRtThreads, 1)
    router_screen_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmHi,
                         const __grid_constant__ CUtensorMap tmLo, int T, int d, int E, int kb_per_split,
                         float* __restrict__ Apart) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + kScrStages * kScrStageBytes);
  uint64_t* empty_bar = full_bar + kScrStages;
  uint64_t* acc_bar = empty_bar + kScrStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kScrT, e0 = blockIdx.y * kScrE, split = blockIdx.z;
  const int KB = d / kRtBK;
  const int kb0 = split * kb_per_split, kb1 = min(KB, kb0 + kb_per_split);
  constexpr uint32_t kCols = 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kScrStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(acc_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmHi);
      tma_prefetch_desc(&tmLo);
      const uint64_t pol = l2_policy_evict_normal();
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, kWaitLimitNs, abort_flag)) {
          record_device_error(1u /* MOE_DEVERR_WAIT_TIMEOUT_PRODUCER */);
          *abort_flag = 1;
          ok = false;
          break;
        }
        uint8_t* st = smem + s * kScrStageBytes;
        mbar_arrive_expect_tx(&full_bar[s], static_cast<uint32_t>(kScrStageBytes));
        const int k0 = kb * kRtBK;
        tma_load_2d(st, &tmHi, &full_bar[s], k0, e0, pol);
        tma_load_2d(st + kScrE * kRtBK * 2, &tmLo, &full_bar[s], k0, e0, pol);
        tma_load_2d(st + 2 * kScrE * kRtBK * 2, &tmX, &full_bar[s], k0, t0, pol);
        tma_load_2d(st + 2 * kScrE * kRtBK * 2 + 128 * kRtBK * 2, &tmX, &full_bar[s], k0, t0 + 128, pol);
        ++issued;
        if (++s == kScrStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) {
        for (int i = 0; i < kScrStages && i < issued; ++i) {
          s = (s == 0) ? kScrStages - 1 : s - 1;
          if (s == kScrStages - 1) ph ^= 1u;
          mbar_wait_bounded(&full_bar[s], ph, kWaitLimitNs, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(128u, 256u, 0u, 0u);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_bounded(&full_bar[s], ph, kWaitLimitNs, abort_flag)) {
          record_device_error(2u /* MOE_DEVERR_WAIT_TIMEOUT_MMA */);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t hi_addr = smem_u32(smem + s * kScrStageBytes);
        const uint32_t lo_addr = hi_addr + kScrE * kRtBK * 2;
        const uint32_t x_addr = lo_addr + kScrE * kRtBK * 2;
#pragma unroll
        for (int kk = 0; kk < kRtBK / 16; ++kk) {
          const uint64_t xdesc = umma_smem_desc_sw128(x_addr + kk * 32, 16, 1024);
          const uint64_t hdesc = umma_smem_desc_sw128(hi_addr + kk * 32, 16, 1024);
          const uint64_t ldesc = umma_smem_desc_sw128(lo_addr + kk * 32, 16, 1024);
          tc_mma_bf16(tmem_base, hdesc, xdesc, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          tc_mma_bf16(tmem_base, ldesc, xdesc, idesc, 1u);
        }
        tc_commit(&empty_bar[s]);
        if (++s == kScrStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      tc_commit(acc_bar);  // completes when every MMA above has
      if (!ok) mbar_wait_bounded(acc_bar, 0u, kWaitLimitNs, nullptr);
    }
  } else {
    const int q = warp & 3;
    const int e = e0 + q * 32 + lane;  // this thread's TMEM lane = expert
    if (mbar_wait_bounded(acc_bar, 0u, kWaitLimitNs, abort_flag)) {
      tc_fence_after_sync();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      float* plane = Apart + static_cast<int64_t>(split) * T * E;
      const int nt = min(kScrT, T - t0);
      for (int c0 = 0; c0 < nt; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c0), v);
        tmem_ld_wait();
        if (e < E) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c0 + i < nt) plane[static_cast<int64_t>(t0 + c0 + i) * E + e] = __uint_as_float(v[i]);
        }
      }
    } else {
      record_device_error(3u /* MOE_DEVERR_WAIT_TIMEOUT_EPILOGUE */);
      *abort_flag = 1;
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kCols);
  }
}

// ------------------------------------------------------------ 3. re-check

constexpr int kRcWarps = 4;               // warps per CTA; one CTA per token
constexpr int kRcXsBytes = 128 * 32 * 4;  // x staged as [j][l] bf16 pairs (16 KB)

// Stage x_t as xs[j][l] = (x[128 l + j], x[128 (l + 32) + j]) bf16 pairs (0 past
// d) with 16-byte loads; `tid` / `nthreads` split the work.
__device__ __forceinline__ void stage_x_pairs(const uint16_t* __restrict__ xt, int d, int tid, int nthreads,
                                              uint32_t* xs) {
  uint16_t* xh = reinterpret_cast<uint16_t*>(xs);
  const uint4* xv = reinterpret_cast<const uint4*>(xt);
  for (int v = tid; v < 128 * 64 / 8; v += nthreads) {  // 8 values of one chunk per vector
    const int i0 = v * 8, c = i0 >> 7, j0 = i0 & 127;
    uint4 q = make_uint4(0u, 0u, 0u, 0u);
    if (i0 < d) q = __ldg(xv + v);
    const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      xh[((j0 + 2 * u) * 32 + (c & 31)) * 2 + (c >> 5)] = static_cast<uint16_t>(w4[u] & 0xFFFFu);
      xh[((j0 + 2 * u + 1) * 32 + (c & 31)) * 2 + (c >> 5)] = static_cast<uint16_t>(w4[u] >> 16);
    }
  }
}

// Chunk partials of the exact-order logit of one expert: lane l runs the fma
// chains of chunks l and l + 32 (each from +0, offsets j ascending), reading
// its two chunks of Wc with one 8-byte load and of xs with one 4-byte load per
// offset. The Wc loads come from L2, so 32 offsets of them are issued before
// their fmas (four L2 round trips per expert); the xs loads are shared-memory
// reads issued in the fma loop. FULL: d % 128 == 0.
template <bool FULL>
__device__ __forceinline__ void exact_chunk_pairs(const uint32_t* __restrict__ xs, const float2* __restrict__ wce,
                                                  int d, int lane, float& p0, float& p1) {
  constexpr int kB = 32;
  const int n0 = FULL ? 128 : max(0, min(128, d - lane * 128));
  const int n1 = FULL ? 128 : max(0, min(128, d - (lane + 32) * 128));
  p0 = 0.0f;
  p1 = 0.0f;
  for (int j = 0; j < 128; j += kB) {
    float2 w[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) w[u] = __ldg(wce + (j + u) * 32 + lane);
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const uint32_t xv = xs[(j + u) * 32 + lane];
      const float xa = __uint_as_float(xv << 16), xb = __uint_as_float(xv & 0xFFFF0000u);
      if (FULL || j + u < n0) p0 = __fmaf_rn(xa, w[u].x, p0);
      if (FULL || j + u < n1) p1 = __fmaf_rn(xb, w[u].y, p1);
    }
  }
}

// Ordered sum of C chunk partials (ascending c), read from shared memory in
// batches of 8.
__device__ __forceinline__ float ordered_chunk_sum(const float* part, int C) {
  float l = part[0];
  for (int c0 = 1; c0 < C; c0 += 8) {
    float pc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) pc[u] = part[min(c0 + u, 63)];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (c0 + u < C) l = __fadd_rn(l, pc[u]);
  }
  return l;
}

// One CTA (4 warps) per token. A[t, :] holds the screened logits with the
// bias already added (router_reduce_partials_kernel).
//  1. warp 0: softmax statistics; candidates by descending A (ties -> lower
//     index) up to the window A >= tau - 2 eps; warps 1-3 meanwhile stage x.
//     A token whose window holds more than kMaxCand experts is appended to
//     `overflow` and finished by router_fallback_kernel.
//  2. all warps: exact-order logits of the candidates (candidate j by warp j % 4).
//  3. warp 0: top-k over the candidates by (L desc, index asc); the softmax
//     denominator uses L for the candidates and A for the other experts.
template <int MAXV, bool FULL>
__global__ void __launch_bounds__(kRcWarps * 32, 6)
    router_recheck_kernel(const float* __restrict__ A, const uint16_t* __restrict__ x, const float* __restrict__ Wc,
                          const float* __restrict__ bias, const float* __restrict__ xnorm,
                          const float* __restrict__ wnorm, int T, int d, int E, int k, int32_t* __restrict__ topk_idx,
                          float* __restrict__ topk_w, int32_t* __restrict__ overflow) {
  __shared__ uint32_t xs[kRcXsBytes / 4];
  __shared__ float s_part[kRcWarps][64];
  __shared__ int s_e[kMaxCand];
  __shared__ float s_a[kMaxCand], s_l[kMaxCand];
  __shared__ int s_nc;
  __shared__ float s_m, s_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  const int C = (d + 127) / 128;

  if (warp == 0) {
    float v[MAXV];
    float m = -INFINITY, amax = 0.0f, bmax = 0.0f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int e = i * 32 + lane;
      v[i] = (e < E) ? __ldcs(A + static_cast<int64_t>(t) * E + e) : -INFINITY;
    }
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      if (i * 32 + lane < E) {
        m = fmaxf(m, v[i]);
        amax = fmaxf(amax, fabsf(v[i]));
      }
    }
    if (bias != nullptr)
      for (int e = lane; e < E; e += 32) bmax = fmaxf(bmax, fabsf(__ldg(bias + e)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
    }
    float ssum = 0.0f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i)
      if (i * 32 + lane < E) ssum += expf(v[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
    const float eps =
        kRtEpsRel * __ldg(xnorm + t) * __ldg(wnorm + E) + (amax + bmax + 1.0f) * (1.0f / 1048576.0f);

    uint32_t taken = 0u;
    int nc = 0;
    float tau = 0.0f;
    const int limit = (E <= kMaxCand) ? E : kMaxCand;
    bool overflowed = false;
    while (true) {
      // warp arg-max by (A desc, index asc): a lane's values are in ascending
      // expert order, so a strict '>' keeps its lowest index among equal
      // values; across lanes the largest order key wins, then the lowest index
      float lv = -INFINITY;
      int li = -1;
#pragma unroll
      for (int i = 0; i < MAXV; ++i) {
        const int e = i * 32 + lane;
        const bool cand = e < E && !((taken >> i) & 1u);
        if (cand && (li < 0 || v[i] > lv)) {
          lv = v[i];
          li = e;
        }
      }
      const uint32_t key = li < 0 ? 0u : float_order_key(lv + 0.0f);
      const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
      if (kmax == 0u) break;                        // every expert taken
      const uint32_t win =
          __reduce_min_sync(0xffffffffu, (li >= 0 && key == kmax) ? static_cast<uint32_t>(li) : 0xffffffffu);
      const int bi = static_cast<int>(win);
      const float bv = __shfl_sync(0xffffffffu, lv, bi & 31);
      if (nc == k - 1) tau = bv;
      if (nc >= k && bv < tau - 2.0f * eps) break;  // outside the window
      if (nc == limit) {                            // window too wide: exact fallback
        overflowed = true;
        break;
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      if (lane == 0) {
        s_e[nc] = bi;
        s_a[nc] = bv;
      }
      ++nc;
    }
    if (lane == 0) {
      if (overflowed) {
        const int slot = atomicAdd(overflow, 1);
        overflow[1 + slot] = t;
        nc = 0;
      }
      s_nc = nc;
      s_m = m;
      s_s = ssum;
    }
  } else {
    stage_x_pairs(x + static_cast<int64_t>(t) * d, d, threadIdx.x - 32, (kRcWarps - 1) * 32, xs);
  }
  __syncthreads();
  const int nc = s_nc;
  if (nc == 0) return;  // overflowed: finished by the fallback kernel

  // 2. exact-order logits; candidates in ascending expert order across warps
  //    would share L1 lines, but the list is short, so it is taken as extracted
  for (int j = warp; j < nc; j += kRcWarps) {
    const int e = s_e[j];
    float p0, p1;
    exact_chunk_pairs<FULL>(xs, reinterpret_cast<const float2*>(Wc + static_cast<int64_t>(e) * 128 * 64), d, lane, p0,
                            p1);
    s_part[warp][lane] = p0;
    s_part[warp][lane + 32] = p1;
    __syncwarp();
    if (lane == 0) {
      float l = ordered_chunk_sum(s_part[warp], C);
      if (bias != nullptr) l = __fadd_rn(l, __ldg(bias + e));
      s_l[j] = l;
    }
    __syncwarp();
  }
  __syncthreads();

  // 3. top-k by (L desc, index asc); denominator with exact L for candidates
  if (warp == 0) {
    const float m = s_m;
    const bool mine = lane < nc;
    const int my_e = mine ? s_e[lane] : 0x7fffffff;
    const float my_l = mine ? s_l[lane] : -INFINITY;
    float corr = mine ? (expf(my_l - m) - expf(s_a[lane] - m)) : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) corr += __shfl_xor_sync(0xffffffffu, corr, o);
    const float s = s_s + corr;
    // each candidate's slot is its rank among the candidates by (L desc,
    // index asc); the k best are written
    int rank = 0;
    for (int q = 0; q < nc; ++q) {
      const float lq = s_l[q];
      const int eq = s_e[q];
      rank += (lq > my_l || (lq == my_l && eq < my_e)) ? 1 : 0;
    }
    if (mine && rank < k) {
      topk_idx[static_cast<int64_t>(t) * k + rank] = my_e;
      topk_w[static_cast<int64_t>(t) * k + rank] = expf(my_l - m) / s;
    }
  }
}

// Tokens whose candidate window overflowed: every expert's exact-order logit,
// then the top-k over all of them (exact softmax). One CTA (4 warps) per
// listed token; the grid is an upper bound and blocks past the count return.
__global__ void __launch_bounds__(128)
    router_fallback_kernel(const int32_t* __restrict__ overflow, const uint16_t* __restrict__ x,
                           const float* __restrict__ Wc, const float* __restrict__ bias, int d, int E, int k,
                           int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  __shared__ uint32_t xs[128 * 32];
  __shared__ float s_l[1024];
  __shared__ float s_part[4][64];
  if (static_cast<int>(blockIdx.x) >= overflow[0]) return;
  const int t = overflow[1 + blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = (d + 127) / 128;
  stage_x_pairs(x + static_cast<int64_t>(t) * d, d, threadIdx.x, 128, xs);
  __syncthreads();
  for (int e = warp; e < E; e += 4) {
    float p0, p1;
    exact_chunk_pairs<false>(xs, reinterpret_cast<const float2*>(Wc + static_cast<int64_t>(e) * 128 * 64), d, lane, p0,
                             p1);
    s_part[warp][lane] = p0;
    s_part[warp][lane + 32] = p1;
    __syncwarp();
    if (lane == 0) {
      float l = s_part[warp][0];
      for (int c = 1; c < C; ++c) l = __fadd_rn(l, s_part[warp][c]);
      if (bias != nullptr) l = __fadd_rn(l, __ldg(bias + e));
      s_l[e] = l;
    }
    __syncwarp();
  }
  __syncthreads();
  if (warp != 0) return;
  float m = -INFINITY;
  for (int e = lane; e < E; e += 32) m = fmaxf(m, s_l[e]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float s = 0.0f;
  for (int e = lane; e < E; e += 32) s += expf(s_l[e] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      const float l = s_l[e];
      if (l != -INFINITY && (bi == 0x7fffffff || l > bv)) {  // ascending e per lane: first max wins ties
        bv = l;
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      topk_idx[static_cast<int64_t>(t) * k + j] = bi;
      topk_w[static_cast<int64_t>(t) * k + j] = expf(bv - m) / s;
      s_l[bi] = -INFINITY;  // taken
    }
    __syncwarp();
  }
}

}  // namespace moe
