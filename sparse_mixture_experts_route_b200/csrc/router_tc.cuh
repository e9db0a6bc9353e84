// Router for many tokens: tensor-core screening plus an exact re-check.
//
// Computes the same routing as router.cuh (the gate of "Kimi K3: The Open Model
// That Just Cornered the AI Frontier", section "Mixture-of-Experts with Dynamic
// Load Balancing": softmax over all experts, top-k, unnormalised values) and the
// same bits, in less time when T * E is large:
//
//  1. prep: W_router [d, E] fp32 -> a chunk-interleaved exact copy Wc [E][128][C]
//     fp32 (Wc[e][j][c] = W[128 c + j][e]) and Wt_hi / Wt_lo [E, d] bf16 with Wt_hi = bf16(W), Wt_lo = bf16(W - Wt_hi),
//     so |W - Wt_hi - Wt_lo| <= 2^-17 |W|; an upper bound of each column norm
//     ||W_e||_2 and of each token norm ||x_t||_2.
//  2. screen: A[t, e] = x_t . Wt_hi[e] + x_t . Wt_lo[e] (+ b_e) on tcgen05
//     (bf16 x bf16 products are exact in fp32; fp32 accumulation in TMEM).
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

namespace moe {

constexpr int kRtM = 128;          // tokens per tile (UMMA M)
constexpr int kRtBK = 64;          // K per stage
constexpr int kRtStages = 4;
constexpr int kRtThreads = 192;    // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kMaxCand = 32;       // candidate window capacity per token
constexpr float kRtEpsRel = 1.0f / 2048.0f;

__host__ __device__ constexpr int rt_stage_bytes(int ne) { return kRtM * kRtBK * 2 + 2 * ne * kRtBK * 2; }
__host__ __device__ constexpr int rt_smem_bytes(int ne) { return kRtStages * rt_stage_bytes(ne) + 256 + 1024; }

// ---------------------------------------------------------------- 1. prep

// W [d, E] -> Wt_hi / Wt_lo [E, d] (bf16, K-major for the screen), and fp64
// partial sums of squares of each column over this block's 256 input indices:
// part[blockIdx.y][e]. Block (32, 8): a 32-expert x 256-index slab, transposed
// through shared memory.
__global__ void __launch_bounds__(256)
    router_prep_kernel(const float* __restrict__ W, int d, int E, uint16_t* __restrict__ Wt_hi,
                       uint16_t* __restrict__ Wt_lo, double* __restrict__ part) {
  __shared__ float tile[32][33];
  __shared__ double ssq[8][32];
  const int e0 = blockIdx.x * 32, i0 = blockIdx.y * 256;
  const int tx = threadIdx.x, ty = threadIdx.y;
  double acc = 0.0;
  for (int sub = 0; sub < 8; ++sub) {
    const int ib = i0 + sub * 32;
    // load 32 (i) x 32 (e), coalesced along e
    for (int r = ty; r < 32; r += 8) {
      const int i = ib + r, e = e0 + tx;
      const float v = (i < d && e < E) ? __ldg(W + static_cast<int64_t>(i) * E + e) : 0.0f;
      tile[r][tx] = v;
      acc += static_cast<double>(v) * static_cast<double>(v);
    }
    __syncthreads();
    // store transposed: rows e, coalesced along i
    for (int r = ty; r < 32; r += 8) {
      const int e = e0 + r, i = ib + tx;
      if (e < E && i < d) {
        const float v = tile[tx][r];
        const int64_t at = static_cast<int64_t>(e) * d + i;
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
        Wt_hi[at] = *reinterpret_cast<const uint16_t*>(&hi);
        Wt_lo[at] = *reinterpret_cast<const uint16_t*>(&lo);
      }
    }
    __syncthreads();
  }
  ssq[ty][tx] = acc;  // column e0 + tx, rows ty, ty + 8, ... of this slab
  __syncthreads();
  if (ty == 0 && e0 + tx < E) {
    double s = 0.0;
    for (int r = 0; r < 8; ++r) s += ssq[r][tx];
    part[static_cast<int64_t>(blockIdx.y) * E + e0 + tx] = s;
  }
}

// W [d, E] -> Wc [E][128][C] fp32 with Wc[e][j][c] = W[c * 128 + j][e] (0 past
// d): for one expert and one offset j inside a chunk, the C chunks are adjacent,
// so a warp whose lanes each run one chunk's fma chain reads 32 consecutive
// floats per step. Block (32, 8) handles 32 experts x 4 offsets j x all chunks.
__global__ void __launch_bounds__(256)
    router_interleave_kernel(const float* __restrict__ W, int d, int E, int C, float* __restrict__ Wc) {
  __shared__ float tile[4][64][33];  // [j][c][e]; C <= 64 (d <= 8192)
  const int e0 = blockIdx.x * 32, j0 = blockIdx.y * 4;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int rc = ty; rc < 4 * C; rc += 8) {
    const int j = rc / C, c = rc - j * C;
    const int i = c * 128 + j0 + j, e = e0 + tx;
    tile[j][c][tx] = (i < d && e < E) ? __ldg(W + static_cast<int64_t>(i) * E + e) : 0.0f;
  }
  __syncthreads();
  for (int r = ty; r < 32 * 4; r += 8) {
    const int el = r / 4, j = r % 4, e = e0 + el;
    if (e >= E) continue;
    float* dst = Wc + (static_cast<int64_t>(e) * 128 + j0 + j) * C;
    for (int c = tx; c < C; c += 32) dst[c] = tile[j][c][el];
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
__global__ void __launch_bounds__(256)
    router_xnorm_kernel(const uint4* __restrict__ x, int T, int vec_per_row, float* __restrict__ xnorm) {
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
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

// A[t, e] = x_t . (Wt_hi[e] + Wt_lo[e]) (+ b_e), fp32, for one tile of 128
// tokens x NE experts per CTA. Both operands K-major with 128-byte swizzle.
__global__ void __launch_bounds__(kRtThreads, 1)
    router_screen_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmHi,
                         const __grid_constant__ CUtensorMap tmLo, const float* __restrict__ bias, int T, int d,
                         int E, int ne, float* __restrict__ A) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stage_bytes = rt_stage_bytes(ne);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + kRtStages * stage_bytes);
  uint64_t* empty_bar = full_bar + kRtStages;
  uint64_t* acc_bar = empty_bar + kRtStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.y * kRtM, e0 = blockIdx.x * ne;
  const int KB = d / kRtBK;
  const uint32_t tmem_cols = static_cast<uint32_t>(ne < 32 ? 32 : ne);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRtStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(acc_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
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
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, kWaitLimitNs, abort_flag)) {
          record_device_error(1u /* MOE_DEVERR_WAIT_TIMEOUT_PRODUCER */);
          *abort_flag = 1;
          ok = false;
          break;
        }
        uint8_t* st = smem + s * stage_bytes;
        mbar_arrive_expect_tx(&full_bar[s], static_cast<uint32_t>(stage_bytes));
        tma_load_2d(st, &tmX, &full_bar[s], kb * kRtBK, t0, pol);
        tma_load_2d(st + kRtM * kRtBK * 2, &tmHi, &full_bar[s], kb * kRtBK, e0, pol);
        tma_load_2d(st + kRtM * kRtBK * 2 + ne * kRtBK * 2, &tmLo, &full_bar[s], kb * kRtBK, e0, pol);
        ++issued;
        if (++s == kRtStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) {
        for (int i = 0; i < kRtStages && i < issued; ++i) {
          s = (s == 0) ? kRtStages - 1 : s - 1;
          if (s == kRtStages - 1) ph ^= 1u;
          mbar_wait_bounded(&full_bar[s], ph, kWaitLimitNs, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(128u, static_cast<uint32_t>(ne), 0u, 0u);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_bounded(&full_bar[s], ph, kWaitLimitNs, abort_flag)) {
          record_device_error(2u /* MOE_DEVERR_WAIT_TIMEOUT_MMA */);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_addr = smem_u32(smem + s * stage_bytes);
        const uint32_t hi_addr = a_addr + kRtM * kRtBK * 2;
        const uint32_t lo_addr = hi_addr + ne * kRtBK * 2;
#pragma unroll
        for (int kk = 0; kk < kRtBK / 16; ++kk) {
          const uint64_t adesc = umma_smem_desc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t hdesc = umma_smem_desc_sw128(hi_addr + kk * 32, 16, 1024);
          const uint64_t ldesc = umma_smem_desc_sw128(lo_addr + kk * 32, 16, 1024);
          tc_mma_bf16(tmem_base, adesc, hdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          tc_mma_bf16(tmem_base, adesc, ldesc, idesc, 1u);
        }
        tc_commit(&empty_bar[s]);
        if (++s == kRtStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      tc_commit(acc_bar);  // also drains: completes when every MMA above has
      if (!ok) mbar_wait_bounded(acc_bar, 0u, kWaitLimitNs, nullptr);
    }
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int t = t0 + r;
    if (mbar_wait_bounded(acc_bar, 0u, kWaitLimitNs, abort_flag)) {
      tc_fence_after_sync();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      for (int c0 = 0; c0 < ne; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c0), v);
        tmem_ld_wait();
        if (t < T) {
          float* row = A + static_cast<int64_t>(t) * E;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int e = e0 + c0 + i;
            if (e < E) {
              float a = __uint_as_float(v[i]);
              if (bias != nullptr) a = __fadd_rn(a, __ldg(bias + e));
              row[e] = a;
            }
          }
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
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// ------------------------------------------------------------ 3. re-check

// One CTA (128 threads) per token.
//   warp 0: softmax statistics over A and the candidate window;
//   warps 0-3: exact-order logits of the candidates; lane l runs the fma chains
//              of chunks l and l + 32 (reading the chunk-interleaved copy Wc
//              and x staged as xs[j][c], both conflict-free and coalesced);
//   warp 0: top-k over the candidates by (L desc, index asc); the softmax
//           denominator uses L for the candidates and A for every other expert.
template <int MAXV>
__global__ void __launch_bounds__(128)
    router_recheck_kernel(const float* __restrict__ A, const uint16_t* __restrict__ x, const float* __restrict__ Wc,
                          const float* __restrict__ bias, const float* __restrict__ xnorm,
                          const float* __restrict__ wnorm, int T, int d, int E, int k, int32_t* __restrict__ topk_idx,
                          float* __restrict__ topk_w) {
  constexpr int kChunk = 128;
  extern __shared__ float xs[];  // [kChunk][C]: xs[j * C + c] = x[c * 128 + j] (0 past d)
  __shared__ int s_cand[1024];
  __shared__ float s_L[1024];
  __shared__ float s_A[1024];
  __shared__ float s_part[4][64];
  __shared__ int s_nc;
  __shared__ float s_m, s_s;

  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = (d + kChunk - 1) / kChunk;

  for (int i = threadIdx.x; i < kChunk * C; i += blockDim.x) {
    const int c = i / kChunk, j = i - c * kChunk;  // coalesced reads of x along i
    const float v = (i < d) ? __uint_as_float(static_cast<uint32_t>(x[static_cast<int64_t>(t) * d + i]) << 16) : 0.0f;
    xs[j * C + c] = v;
  }

  if (warp == 0) {
    float v[MAXV];
    float m = -INFINITY, amax = 0.0f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int e = i * 32 + lane;
      v[i] = (e < E) ? A[static_cast<int64_t>(t) * E + e] : -INFINITY;
      if (e < E) {
        m = fmaxf(m, v[i]);
        amax = fmaxf(amax, fabsf(v[i]));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    }
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i)
      if (i * 32 + lane < E) s += expf(v[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    float bmax = 0.0f;
    if (bias != nullptr) {
      for (int e = lane; e < E; e += 32) bmax = fmaxf(bmax, fabsf(__ldg(bias + e)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
    }
    const float eps = kRtEpsRel * __ldg(xnorm + t) * __ldg(wnorm + E) + (amax + bmax + 1.0f) * (1.0f / 1048576.0f);

    // extract by descending A (ties -> lower index) until past the window
    uint32_t taken = 0u;
    int nc = 0;
    float tau = 0.0f;
    bool overflow = false;
    const int limit = (E <= kMaxCand) ? E : kMaxCand;
    while (true) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < MAXV; ++i) {
        const int e = i * 32 + lane;
        if (e < E && !((taken >> i) & 1u) && (bi == 0x7fffffff || v[i] > bv)) {
          bv = v[i];
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
      if (bi == 0x7fffffff) break;                  // every expert taken
      if (nc == k - 1) tau = bv;
      if (nc >= k && bv < tau - 2.0f * eps) break;  // outside the window
      if (nc == limit) {
        overflow = true;
        break;
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      if (lane == 0) {
        s_cand[nc] = bi;
        s_A[nc] = bv;
      }
      ++nc;
    }
    if (overflow) {  // recompute every expert of this token (exact, slow, rare)
#pragma unroll
      for (int i = 0; i < MAXV; ++i) {
        const int e = i * 32 + lane;
        if (e < E) {
          s_cand[e] = e;
          s_A[e] = v[i];
        }
      }
      nc = E;
    }
    if (lane == 0) {
      s_nc = nc;
      s_m = m;
      s_s = s;
    }
  }
  __syncthreads();

  const int nc = s_nc;
  for (int j = warp; j < nc; j += 4) {
    const int e = s_cand[j];
    const float* wc = Wc + static_cast<int64_t>(e) * kChunk * C;
    const int c0 = lane, c1 = lane + 32;
    const int n0 = min(kChunk, d - c0 * kChunk), n1 = min(kChunk, d - c1 * kChunk);
    float p0 = 0.0f, p1 = 0.0f;
    if (c1 < C) {
#pragma unroll 8
      for (int i = 0; i < kChunk; ++i) {
        const float w0 = __ldg(wc + i * C + c0), w1 = __ldg(wc + i * C + c1);
        if (i < n0) p0 = __fmaf_rn(xs[i * C + c0], w0, p0);
        if (i < n1) p1 = __fmaf_rn(xs[i * C + c1], w1, p1);
      }
    } else if (c0 < C) {
#pragma unroll 8
      for (int i = 0; i < kChunk; ++i) {
        const float w0 = __ldg(wc + i * C + c0);
        if (i < n0) p0 = __fmaf_rn(xs[i * C + c0], w0, p0);
      }
    }
    if (c0 < C) s_part[warp][c0] = p0;
    if (c1 < C) s_part[warp][c1] = p1;
    __syncwarp();
    if (lane == 0) {
      float l = s_part[warp][0];
      for (int c = 1; c < C; ++c) l = __fadd_rn(l, s_part[warp][c]);
      if (bias != nullptr) l = __fadd_rn(l, __ldg(bias + e));
      s_L[j] = l;
    }
    __syncwarp();
  }
  __syncthreads();

  if (warp == 0) {
    const float m = s_m;
    // denominator: exact-order logits for the candidates, screened ones elsewhere
    float corr = 0.0f;
    for (int c = lane; c < nc; c += 32) corr += expf(s_L[c] - m) - expf(s_A[c] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) corr += __shfl_xor_sync(0xffffffffu, corr, o);
    const float s = s_s + corr;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff, bslot = -1;
      for (int c = lane; c < nc; c += 32) {
        const int e = s_cand[c];
        if (e < 0) continue;
        const float L = s_L[c];
        if (bi == 0x7fffffff || L > bv || (L == bv && e < bi)) {
          bv = L;
          bi = e;
          bslot = c;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        const int os = __shfl_xor_sync(0xffffffffu, bslot, o);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
          bv = ov;
          bi = oi;
          bslot = os;
        }
      }
      if (lane == 0) {
        topk_idx[static_cast<int64_t>(t) * k + j] = bi;
        topk_w[static_cast<int64_t>(t) * k + j] = expf(bv - m) / s;
        s_cand[bslot] = -1;  // taken
      }
      __syncwarp();
    }
  }
}

}  // namespace moe
