// Router: logits, softmax over all experts, top-k.
//
// Follows the gating code on "Kimi K3: The Open Model That Just Cornered the
// AI Frontier" (section "Mixture-of-Experts with Dynamic Load Balancing"): one
// gate projection from d_model to n_experts, softmax over the expert axis,
// top-k of the probabilities, values returned without renormalisation.
//
// Numerics (the pages fix none): fp32 with x widened exactly from bf16.
// Summation order, fixed so routing is reproducible bit for bit:
//   p_c = fma chain over the 128 consecutive input indices of chunk c (from +0),
//   l   = ((p_0 + p_1) + p_2) + ... + p_{C-1},   then l = l + b_e.
// Selection compares these fp32 logits (softmax is monotone, so the chosen set
// equals top-k of the probabilities); equal logits go to the lower index.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"

namespace moe {

constexpr int kRouterChunk = 128;  // input indices per ordered partial sum
constexpr int kRouterBK = 32;      // input indices staged in shared memory per step

// Order-preserving map of a non-NaN float to an unsigned key.
__device__ __forceinline__ uint32_t float_order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Logits of a [BM tokens x BN experts] tile.
//   SPLIT = false: the CTA walks every chunk in order and writes final logits
//                  (+ bias) to out[t * E + e].
//   SPLIT = true : the CTA handles chunk blockIdx.z only and writes its partial
//                  p_c to out[(c * T + t) * E + e]; router_reduce_partials_kernel
//                  adds the partials in ascending c. Both modes give identical bits.
// Requires d % 32 == 0. Threads: (BM / TM) * (BN / TN).
template <int BM, int BN, int TM, int TN, bool SPLIT>
__global__ void __launch_bounds__((BM / TM) * (BN / TN), 2)
    router_logits_kernel(const uint16_t* __restrict__ x, const float* __restrict__ W,
                         const float* __restrict__ bias, int T, int d, int E, float* __restrict__ out) {
  constexpr int NT = (BM / TM) * (BN / TN);
  constexpr int TX = BN / TN;
  static_assert(TM % 2 == 0 && TN == 4, "micro-tile layout");
  static_assert(NT >= 64 && NT <= 256, "block size");
  __shared__ __align__(16) float xs[2][kRouterBK][BM];
  __shared__ __align__(16) float ws[2][kRouterBK][BN];

  const int tid = threadIdx.x;
  const int tx = tid % TX, ty = tid / TX;
  const int e0 = blockIdx.x * BN, t0 = blockIdx.y * BM;
  const int nchunks = (d + kRouterChunk - 1) / kRouterChunk;
  const int c_begin = SPLIT ? blockIdx.z : 0;
  const int c_end = SPLIT ? blockIdx.z + 1 : nchunks;
  const int k_begin = c_begin * kRouterChunk;
  const int k_end = min(d, c_end * kRouterChunk);
  const int nsteps = (k_end - k_begin) / kRouterBK;

  // staging registers for the next step
  constexpr int XV = (BM * kRouterBK / 8 + NT - 1) / NT;  // uint4 (8 bf16) loads of x per thread
  constexpr int WV = (BN * kRouterBK + NT - 1) / NT;      // scalar loads of W per thread
  uint4 xr[XV];
  float wr[WV];

  auto load_step = [&](int k0) {
#pragma unroll
    for (int v = 0; v < XV; ++v) {
      const int m = tid + v * NT;  // m in [0, BM*BK/8)
      const int r = m / (kRouterBK / 8), cg = m % (kRouterBK / 8);
      const int t = t0 + r;
      if (m < BM * kRouterBK / 8 && t < T)
        xr[v] = *reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * d + k0 + cg * 8);
      else
        xr[v] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int v = 0; v < WV; ++v) {
      const int m = tid + v * NT;
      const int kk = m / BN, col = m % BN;
      const int e = e0 + col;
      wr[v] = (m < BN * kRouterBK && e < E) ? __ldg(W + static_cast<int64_t>(k0 + kk) * E + e) : 0.0f;
    }
  };
  auto store_step = [&](int buf) {
#pragma unroll
    for (int v = 0; v < XV; ++v) {
      const int m = tid + v * NT;
      if (m < BM * kRouterBK / 8) {
        const int r = m / (kRouterBK / 8), cg = m % (kRouterBK / 8);
        const uint32_t w4[4] = {xr[v].x, xr[v].y, xr[v].z, xr[v].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          xs[buf][cg * 8 + 2 * q][r] = __uint_as_float(w4[q] << 16);
          xs[buf][cg * 8 + 2 * q + 1][r] = __uint_as_float(w4[q] & 0xFFFF0000u);
        }
      }
    }
#pragma unroll
    for (int v = 0; v < WV; ++v) {
      const int m = tid + v * NT;
      if (m < BN * kRouterBK) ws[buf][m / BN][m % BN] = wr[v];
    }
  };

  float acc[TM][TN], lsum[TM][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.0f, lsum[i][j] = 0.0f;

  if (nsteps > 0) {
    load_step(k_begin);
    store_step(0);
  }
  __syncthreads();
  for (int s = 0; s < nsteps; ++s) {
    const int buf = s & 1;
    const int k0 = k_begin + s * kRouterBK;
    if (s + 1 < nsteps) load_step(k0 + kRouterBK);
#pragma unroll
    for (int kk = 0; kk < kRouterBK; ++kk) {
      float a[TM], b[TN];
#pragma unroll
      for (int i = 0; i < TM; i += 2) {
        const float2 v = *reinterpret_cast<const float2*>(&xs[buf][kk][ty * TM + i]);
        a[i] = v.x;
        a[i + 1] = v.y;
      }
      const float4 bv = *reinterpret_cast<const float4*>(&ws[buf][kk][tx * TN]);
      b[0] = bv.x, b[1] = bv.y, b[2] = bv.z, b[3] = bv.w;
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
    }
    // end of a 128-index chunk (or of the input): fold the chunk partial in order
    const int k_next = k0 + kRouterBK;
    if (!SPLIT && (k_next % kRouterChunk == 0 || k_next == k_end)) {
      const bool first = (k_next <= kRouterChunk);
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) {
          lsum[i][j] = first ? acc[i][j] : __fadd_rn(lsum[i][j], acc[i][j]);
          acc[i][j] = 0.0f;
        }
    }
    if (s + 1 < nsteps) store_step(buf ^ 1);
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int t = t0 + ty * TM + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      const int e = e0 + tx * TN + j;
      if (e >= E) continue;
      if (SPLIT) {
        out[(static_cast<int64_t>(blockIdx.z) * T + t) * E + e] = acc[i][j];
      } else {
        float l = lsum[i][j];
        if (bias != nullptr) l = __fadd_rn(l, __ldg(bias + e));
        out[static_cast<int64_t>(t) * E + e] = l;
      }
    }
  }
}

// Split mode, second half: thread per (t, e) adds the C per-chunk partials in
// ascending chunk order, then the bias, writing the final logit over plane 0.
// Each thread reads only its own column of partials, so the in-place write is safe.
__global__ void __launch_bounds__(256)
    router_reduce_partials_kernel(float* __restrict__ lg, int nsplit, const float* __restrict__ bias, int T, int E) {
  const int64_t n = static_cast<int64_t>(T) * E;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float l = lg[i];
  int c = 1;
  for (; c + 8 <= nsplit; c += 8) {
    float p[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) p[u] = lg[static_cast<int64_t>(c + u) * n + i];
#pragma unroll
    for (int u = 0; u < 8; ++u) l = __fadd_rn(l, p[u]);
  }
  for (; c < nsplit; ++c) l = __fadd_rn(l, lg[static_cast<int64_t>(c) * n + i]);
  if (bias != nullptr) l = __fadd_rn(l, __ldg(bias + static_cast<int>(i % E)));
  lg[i] = l;
}

// One warp per token: softmax over all E final logits in fp32, then k rounds
// of warp arg-max (ties -> lower index). MAXV >= ceil(E / 32).
template <int MAXV>
__global__ void __launch_bounds__(256)
    router_topk_kernel(const float* __restrict__ lg, int T, int E, int k, int32_t* __restrict__ topk_idx,
                       float* __restrict__ topk_w) {
  const int warp = static_cast<int>(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5));  // no overflow for T < 2^31
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  const int t = warp;
  float v[MAXV];
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int e = i * 32 + lane;
    v[i] = (e < E) ? __ldcs(lg + static_cast<int64_t>(t) * E + e) : -INFINITY;
  }
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) m = fmaxf(m, v[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i)
    if (i * 32 + lane < E) s += expf(v[i] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);

  uint32_t taken = 0u;
  for (int j = 0; j < k; ++j) {
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
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == 0) {
      topk_idx[static_cast<int64_t>(t) * k + j] = bi;
      topk_w[static_cast<int64_t>(t) * k + j] = expf(bv - m) / s;
    }
  }
}

}  // namespace moe

namespace moe {

// The barrier of the threads that run the CTA-wide helpers below: the whole
// CTA, or, in a CTA of more than 256 threads, threads 0..255 alone (named
// barrier 5).
struct CtaSync {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};
struct FirstWarps8Sync {
  __device__ __forceinline__ void operator()() const { asm volatile("bar.sync 5, 256;" ::: "memory"); }
};

// The probability of a logit l given the softmax statistics of its token:
// exp(l - M) / S. The CTA-wide top-k helpers below and the one-launch
// one-token kernel (which takes the weights after the selection) share this
// expression, so both give the same bits.
__device__ __forceinline__ float softmax_weight(float l, float M, float S) { return expf(l - M) / S; }

// Softmax statistics of one token's E <= 1024 logits held in shared memory,
// by a CTA of 256 threads: M = max_e l_e and S = sum_e exp(l_e - M), the sum
// taken per warp in a fixed shuffle order and then over the warps in order.
template <class Sync = CtaSync>
__device__ __forceinline__ void cta_softmax_stats_256(const float* s_l, int E, float* M, float* S, Sync sync = Sync(),
                                                      int tid = threadIdx.x) {
  __shared__ float s_wm[8], s_ws[8];
  const int lane = tid & 31, w = tid >> 5;
  float m = -INFINITY;
  for (int e = tid; e < E; e += 256) m = fmaxf(m, s_l[e]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) s_wm[w] = m;
  sync();
  float gm = s_wm[0];
#pragma unroll
  for (int q = 1; q < 8; ++q) gm = fmaxf(gm, s_wm[q]);
  float s = 0.0f;
  for (int e = tid; e < E; e += 256) s += expf(s_l[e] - gm);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) s_ws[w] = s;
  sync();
  float gs = s_ws[0];
#pragma unroll
  for (int q = 1; q < 8; ++q) gs += s_ws[q];
  *M = gm;
  *S = gs;
}

// For one warp: the bin of a 256-bin histogram (hist, bins ascending) that
// holds the kk-th largest element, and how many elements lie in higher bins.
__device__ __forceinline__ void warp_find_bin_from_top(const unsigned* hist, unsigned kk, unsigned* bin,
                                                       unsigned* above) {
  const int lane = threadIdx.x & 31;
  unsigned h[8];
  unsigned tot = 0u;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    h[q] = hist[lane * 8 + q];
    tot += h[q];
  }
  unsigned suf = tot;  // inclusive suffix sum over lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += y;
  }
  unsigned cum = suf - tot;  // elements in the bins of higher lanes
#pragma unroll
  for (int q = 7; q >= 0; --q) {
    if (cum < kk && cum + h[q] >= kk) {
      *bin = static_cast<unsigned>(lane * 8 + q);
      *above = cum;
    }
    cum += h[q];
  }
}

// Top-k by (logit desc, index asc) of one token's E <= 1024 logits held in
// shared memory, by a CTA of 256 threads, without sequential arg-max rounds:
// two 8-bit histogram passes over the top 16 bits of the order keys locate
// the bin that holds the k-th largest logit; every logit in or above that bin
// is a candidate, and a candidate's output slot is its exact rank among the
// candidates by the key (order key of the logit, -0 taken as +0; then the
// complemented index), a total order. Returns false, writing nothing, when
// more than 64 logits are candidates (heavy ties); the caller then takes
// cta_topk_rounds_256. out_w may be null (indices only).
template <class Sync = CtaSync>
__device__ __forceinline__ bool cta_topk_histogram_256(const float* s_l, int E, int k, float M, float S,
                                                       int32_t* out_idx, float* out_w, Sync sync = Sync()) {
  __shared__ unsigned s_hist[256];
  __shared__ unsigned s_sel[4];
  __shared__ unsigned s_ncand;
  __shared__ uint64_t s_ckey[64];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  uint32_t key[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = tid + 256 * i;
    key[i] = (e < E) ? float_order_key(s_l[e] + 0.0f) : 0u;
  }
  // pass 1: the top byte of the key
  s_hist[tid] = 0u;
  if (tid == 0) s_ncand = 0u;
  sync();
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (tid + 256 * i < E) atomicAdd(&s_hist[key[i] >> 24], 1u);
  sync();
  if (w == 0) warp_find_bin_from_top(s_hist, static_cast<unsigned>(k), &s_sel[0], &s_sel[1]);
  sync();
  const unsigned b1 = s_sel[0], above1 = s_sel[1];
  // pass 2: the second byte, within that bin
  s_hist[tid] = 0u;
  sync();
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (tid + 256 * i < E && (key[i] >> 24) == b1) atomicAdd(&s_hist[(key[i] >> 16) & 255u], 1u);
  sync();
  if (w == 0) warp_find_bin_from_top(s_hist, static_cast<unsigned>(k) - above1, &s_sel[2], &s_sel[3]);
  sync();
  const unsigned thr = (b1 << 8) | s_sel[2];
  const unsigned ncand = above1 + s_sel[3] + s_hist[s_sel[2]];
  if (ncand > 64u) return false;  // the same for every thread: all read the same shared values
  // collect the candidates (slot order does not matter: ranks decide)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = tid + 256 * i;
    if (e < E && (key[i] >> 16) >= thr) {
      const unsigned slot = atomicAdd(&s_ncand, 1u);
      s_ckey[slot] = (static_cast<uint64_t>(key[i]) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(e));
    }
  }
  sync();
  if (w == 0) {
    for (unsigned r = lane; r < ncand; r += 32) {
      const uint64_t kk = s_ckey[r];
      int rank = 0;
      for (unsigned q = 0; q < ncand; ++q) rank += (s_ckey[q] > kk) ? 1 : 0;
      if (rank < k) {
        const int e = static_cast<int>(~static_cast<uint32_t>(kk & 0xffffffffu));
        out_idx[rank] = e;
        if (out_w != nullptr) out_w[rank] = softmax_weight(s_l[e], M, S);
      }
    }
  }
  return true;
}

// Top-k by k rounds of arg-max (the general case, any ties): warp w takes the
// experts e with (e / 32) % 8 == w and finds its local top-k; warp 0 merges
// the 8 local lists. Weights exp(l - M) / S (out_w may be null).
template <class Sync = CtaSync>
__device__ __forceinline__ void cta_topk_rounds_256(const float* s_l, int E, int k, float M, float S,
                                                    int32_t* out_idx, float* out_w, Sync sync = Sync()) {
  __shared__ float s_cv[8][16];
  __shared__ int s_ci[8][16];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  float v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = 256 * i + 32 * w + lane;
    v[i] = (e < E) ? s_l[e] : -INFINITY;
  }
  // k rounds of warp arg-max by (logit desc, index asc): a lane's values are in
  // ascending expert order, so a strict '>' keeps its lowest index among equal
  // values; across lanes the largest order key wins, then the lowest index
  uint32_t taken = 0u;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = 256 * i + 32 * w + lane;
      if (e < E && !((taken >> i) & 1u) && (bi < 0 || v[i] > bv)) {
        bv = v[i];
        bi = e;
      }
    }
    const uint32_t key = bi < 0 ? 0u : float_order_key(bv);
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
    const uint32_t win =
        __reduce_min_sync(0xffffffffu, (bi >= 0 && key == kmax) ? static_cast<uint32_t>(bi) : 0xffffffffu);
    const int wi = static_cast<int>(win);  // 0xffffffff (-1) when this warp has no expert left
    if (wi >= 0 && (wi & 31) == lane) taken |= 1u << (wi >> 8);
    const float wv = __shfl_sync(0xffffffffu, bv, wi >= 0 ? (wi & 31) : 0);
    if (lane == 0) {
      s_cv[w][j] = wi >= 0 ? wv : -INFINITY;
      s_ci[w][j] = wi >= 0 ? wi : 0x7fffffff;
    }
  }
  sync();

  // merge
  if (w == 0) {
    // candidates: lane holds entries lane, lane + 32, ... of the 8 x k list
    float cv[4];
    int ci[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int slot = lane + 32 * r;
      const int q = slot / 16, j = slot % 16;
      const bool ok = q < 8 && j < k;
      cv[r] = ok ? s_cv[q][j] : -INFINITY;
      ci[r] = ok ? s_ci[q][j] : 0x7fffffff;
    }
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff, br = -1;
#pragma unroll
      for (int r = 0; r < 4; ++r)
        if (ci[r] != 0x7fffffff && (bi == 0x7fffffff || cv[r] > bv || (cv[r] == bv && ci[r] < bi))) {
          bv = cv[r];
          bi = ci[r];
          br = r;
        }
      const uint32_t key = br < 0 ? 0u : float_order_key(bv);
      const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
      const uint32_t win =
          __reduce_min_sync(0xffffffffu, (br >= 0 && key == kmax) ? static_cast<uint32_t>(bi) : 0xffffffffu);
      const int wb = static_cast<int>(win);
      const int owner = __reduce_min_sync(0xffffffffu, (br >= 0 && bi == wb) ? static_cast<uint32_t>(lane) : 32u);
      const float wv = __shfl_sync(0xffffffffu, bv, owner & 31);
      if (lane == owner) {
#pragma unroll
        for (int r = 0; r < 4; ++r)
          if (r == br) ci[r] = 0x7fffffff;  // taken
      }
      if (lane == 0) {
        out_idx[j] = wb;
        if (out_w != nullptr) out_w[j] = softmax_weight(wv, M, S);
      }
    }
  }
}

// Softmax over one token's E <= 1024 final logits, held in shared memory, and
// their top-k by (logit desc, index asc), by 256 threads (threads 0..255 of
// the CTA, all of which must call it; `sync` is their barrier). Writes
// out_idx[0..k) and out_w[0..k) = exp(l - M) / S.
template <class Sync = CtaSync>
__device__ __forceinline__ void cta_softmax_topk_256(const float* s_l, int E, int k, int32_t* out_idx, float* out_w,
                                                     Sync sync = Sync()) {
  float M, S;
  cta_softmax_stats_256(s_l, E, &M, &S, sync);
  if (!cta_topk_histogram_256(s_l, E, k, M, S, out_idx, out_w, sync))
    cta_topk_rounds_256(s_l, E, k, M, S, out_idx, out_w, sync);
}

// Small-T router, second half, one block of 256 threads per token:
//  1. thread i owns experts i, i + 256, ...: l = plane 0 + plane 1 + ... (in
//     ascending chunk order) + bias, kept in shared memory;
//  2. softmax and top-k of those logits (cta_softmax_topk_256).
__global__ void __launch_bounds__(256)
    router_reduce_topk_kernel(const float* __restrict__ lg, int nsplit, const float* __restrict__ bias, int T, int E,
                              int k, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  __shared__ float s_l[1024];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t n = static_cast<int64_t>(T) * E;
  // 1. ordered sums of the chunk partials
  float acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = tid + 256 * i;
    acc[i] = (e < E) ? __ldcs(lg + static_cast<int64_t>(t) * E + e) : 0.0f;
  }
  for (int c0 = 1; c0 < nsplit; c0 += 8) {
    float p[8][4];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = tid + 256 * i;
        p[u][i] = (c0 + u < nsplit && e < E) ? __ldcs(lg + (c0 + u) * n + static_cast<int64_t>(t) * E + e) : 0.0f;
      }
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (c0 + u < nsplit) acc[i] = __fadd_rn(acc[i], p[u][i]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = tid + 256 * i;
    if (e < E) s_l[e] = (bias != nullptr) ? __fadd_rn(acc[i], __ldg(bias + e)) : acc[i];
  }
  __syncthreads();

  cta_softmax_topk_256(s_l, E, k, topk_idx + static_cast<int64_t>(t) * k, topk_w + static_cast<int64_t>(t) * k);
}

}  // namespace moe
