// C ABI of the MoE layer forward pass (declarations and contracts in
// include/moe.h). Host code only validates arguments, carves workspaces,
// encodes TMA descriptors and enqueues kernels; every step of the pass runs in
// the kernels included below. No call allocates, frees or synchronises
// (except moe_get_device_error, a documented debug read).
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "moe.h"

#include "common.cuh"
#include "ep.cuh"
#include "expert_gemm.cuh"
#include "latent.cuh"
#include "mx_gemm.cuh"
#include "mx_prep.cuh"
#include "mx_quant.cuh"
#include "one_token.cuh"
#include "permute.cuh"
#include "ptx.cuh"
#include "qb.cuh"
#include "router.cuh"
#include "router_stream.cuh"
#include "router_tc.cuh"

namespace {

using namespace moe;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  bool fused_ffn = false;  // the one-launch feed-forward fits one CTA on every SM (a cooperative launch)
  bool one_token = false;  // so does the one-launch one-token layer
  int pair_grid = 0;       // CTAs of the CTA-pair gate/up kernel (two per cluster); 0: not available
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Per-device one-time set-up: SM count and the dynamic shared-memory limits of
// the GEMM kernels. Returns MOE_ERR_CUDA if the device cannot be queried.
moe_status_t device_setup(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& di = g_devices[dev];
  if (!di.ready) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(grouped_gemm_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<0>::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(grouped_gemm_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<2>::kSmemBytes) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(grouped_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<1>::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(grouped_gemm_kernel<0, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<0>::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(grouped_gemm_kernel<2, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<2>::kSmemBytes) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(router_one_token_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             router_one_smem_bytes()) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(router_stream_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             router_stream_smem_bytes(1)) != cudaSuccess ||
        cudaFuncSetAttribute(router_stream_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             router_stream_smem_bytes(4)) != cudaSuccess ||
        cudaFuncSetAttribute(router_stream_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             router_stream_smem_bytes(16)) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(router_screen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kScrSmemBytes) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    int coop = 0, per_sm = 0;
    if (cudaFuncSetAttribute(grouped_ffn_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kFusedSmemBytes) != cudaSuccess ||
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, grouped_ffn_fused_kernel, kGemmThreads,
                                                      kFusedSmemBytes) != cudaSuccess)
      return MOE_ERR_CUDA;
    di.fused_ffn = coop != 0 && per_sm >= 1;
    int per_sm1 = 0;
    if (cudaFuncSetAttribute(moe_one_token_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kOneTokenSmemBytes) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm1, moe_one_token_kernel, kGemmThreads,
                                                      kOneTokenSmemBytes) != cudaSuccess)
      return MOE_ERR_CUDA;
    di.one_token = coop != 0 && per_sm1 >= 1;
    // the CTA-pair gate/up kernel: clusters of two CTAs, as many as fit
    di.pair_grid = 0;
    if (cudaFuncSetAttribute(grouped_gemm_pair_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kPairSmemBytes) == cudaSuccess &&
        cudaFuncSetAttribute(grouped_gemm_pair_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kPairSmemBytes) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(sms - sms % 2));
      cfg.blockDim = dim3(kGemmThreads);
      cfg.dynamicSmemBytes = kPairSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_pair_kernel<0>, &cfg) == cudaSuccess && clusters > 0)
        di.pair_grid = 2 * (clusters < sms / 2 ? clusters : sms / 2);
    }
    cudaGetLastError();  // a device without cluster launches only loses the pair kernel
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return MOE_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    di.num_sms = sms;
    di.ready = true;
  }
  *num_sms = di.num_sms;
  return MOE_OK;
}

inline size_t align256(size_t n) { return (n + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

// ------------------------------------------------------------------ router

enum RouterVariant {
  kRouterFullBig = 0,
  kRouterSplitBig = 1,
  kRouterSplitSmall = 2,
  kRouterSplitTiny = 3,
  kRouterTensorCore = 4,
  kRouterStream = 5
};

// Tokens from which the tensor-core screen + exact re-check router is used.
constexpr int kRouterTcMinTokens = 256;

struct RoutePlan {
  RouterVariant variant;
  int nchunks;
  size_t ws_bytes;
  // tensor-core variant: K split of the screen and workspace offsets
  int nsplit = 1, kb_per_split = 0, nparts = 0;
  size_t off_A = 0, off_wt32 = 0, off_hi = 0, off_lo = 0, off_part = 0, off_wnorm = 0, off_xnorm = 0, off_xc = 0,
         off_ovf = 0;
  // few-token variant: chunk partials, final logits, tickets
  size_t off_logits = 0, off_tickets = 0;
};

RoutePlan route_plan(int T, int d, int E) {
  RoutePlan p;
  p.nchunks = ceil_div(d, kRouterChunk);
  const int64_t big_tiles = ceil_div64(T, 128) * ceil_div64(E, 64);
  if (T >= kRouterTcMinTokens && d % 64 == 0 && d <= 8192 && E >= 16) {
    p.variant = kRouterTensorCore;
    // K split of the screen (one CTA per SM: 197 KB of shared memory): the
    // split count minimising waves x K blocks per CTA on a 148-SM part plus the
    // cost of each extra partial plane (written by the screen, read by the
    // reduce: 8 bytes per (token, expert) at about 6.5 TB/s), with a K block
    // taken as about a microsecond; every split keeps at least 8 K blocks
    const int KB = d / kRtBK;
    const int64_t tiles = ceil_div64(T, kScrT) * ceil_div64(E, kScrE);
    const double plane_cost = static_cast<double>(T) * E * 8.0 / 6.5e6;  // in K-block times
    int ns = 1;
    double best = 1e300;
    for (int cand = 1; cand <= (KB / 8 > 0 ? KB / 8 : 1); ++cand) {
      const double cost = static_cast<double>(ceil_div64(tiles * cand, 148)) * ceil_div(KB, cand) + cand * plane_cost;
      if (cost < best) {
        best = cost;
        ns = cand;
      }
    }
    p.kb_per_split = ceil_div(KB, ns);
    p.nsplit = ceil_div(KB, p.kb_per_split);  // every split non-empty
    p.nparts = ceil_div(d, 256);
    size_t at = 0;
    auto take = [&](size_t bytes) {
      const size_t here = at;
      at += align256(bytes);
      return here;
    };
    p.off_A = take(static_cast<size_t>(p.nsplit) * T * E * 4);
    p.off_wt32 = take(static_cast<size_t>(E) * 128 * 64 * 4);
    p.off_hi = take(static_cast<size_t>(E) * d * 2);
    p.off_lo = take(static_cast<size_t>(E) * d * 2);
    p.off_part = take(static_cast<size_t>(p.nparts) * E * 8);
    p.off_wnorm = take(static_cast<size_t>(E + 1) * 4);
    p.off_xnorm = take(static_cast<size_t>(T) * 4);
    p.off_ovf = take(static_cast<size_t>(T + 1) * 4);
    p.ws_bytes = at;
    return p;
  }
  if (T <= kRsMaxTokens && E % 4 == 0) {
    // one launch: every chunk of W_router in flight at once, reductions by the last CTAs
    p.variant = kRouterStream;
    const int G = ceil_div(E, kRsExperts);
    size_t at = align256(static_cast<size_t>(p.nchunks) * T * E * sizeof(float));
    p.off_logits = at;
    at += align256(static_cast<size_t>(T) * E * sizeof(float));
    p.off_tickets = at;
    at += align256(static_cast<size_t>(G + 1) * sizeof(unsigned int));
    p.ws_bytes = at;
    return p;
  }
  if (p.nchunks > 1 && T <= 8)
    p.variant = kRouterSplitTiny;
  else if (p.nchunks > 1 && T <= 32)
    p.variant = kRouterSplitSmall;
  else if (p.nchunks > 1 && big_tiles < 296)
    p.variant = kRouterSplitBig;
  else
    p.variant = kRouterFullBig;
  const int64_t planes = (p.variant == kRouterFullBig) ? 1 : p.nchunks;
  p.ws_bytes = align256(static_cast<size_t>(planes) * T * E * sizeof(float));
  return p;
}

// CTAs of the CTA-pair gate/up kernel on the current device (0: none).
int device_pair_grid() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> lock(g_mutex);
  return g_devices[dev].ready ? g_devices[dev].pair_grid : 0;
}

bool shape_ok(int T, int d, int E, int k) {
  return T >= 1 && d >= 64 && d % 64 == 0 && d <= 32768 && E >= 1 && k >= 1 && k <= E &&
         static_cast<int64_t>(T) * k < (int64_t(1) << 31);
}

bool encode_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
                const cuuint32_t* box);
bool router_w_map(CUtensorMap* map, const float* W, int d, int E);

moe_status_t launch_route_tc(const RoutePlan& plan, const moe_bf16_t* x, const float* W_router, const float* bias,
                             int T, int d, int E, int k, int32_t* idx, float* w, void* ws, cudaStream_t stream) {
  int sms = 0;
  const moe_status_t st = device_setup(&sms);
  if (st != MOE_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* A = reinterpret_cast<float*>(base + plan.off_A);
  float* wt32 = reinterpret_cast<float*>(base + plan.off_wt32);
  uint16_t* hi = reinterpret_cast<uint16_t*>(base + plan.off_hi);
  uint16_t* lo = reinterpret_cast<uint16_t*>(base + plan.off_lo);
  double* part = reinterpret_cast<double*>(base + plan.off_part);
  float* wnorm = reinterpret_cast<float*>(base + plan.off_wnorm);
  float* xnorm = reinterpret_cast<float*>(base + plan.off_xnorm);
  int32_t* ovf = reinterpret_cast<int32_t*>(base + plan.off_ovf);
  const int C = ceil_div(d, 128);
  CUtensorMap mX, mHi, mLo;
  {
    const cuuint64_t dx[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T)};
    const cuuint64_t sx[1] = {static_cast<cuuint64_t>(d) * 2};
    const cuuint32_t bx[2] = {64, 128};
    const cuuint64_t dw[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(E)};
    if (!encode_map(&mX, x, 2, dx, sx, bx) || !encode_map(&mHi, hi, 2, dw, sx, bx) || !encode_map(&mLo, lo, 2, dw, sx, bx))
      return MOE_ERR_INVALID_ARG;
  }
  router_prep_kernel<<<dim3(ceil_div(E, 32), plan.nparts), dim3(32, 8), 0, stream>>>(W_router, d, E, hi, lo, part);
  router_interleave_kernel<<<dim3(ceil_div(E, 32), 32), dim3(32, 8), 0, stream>>>(W_router, d, E, C, wt32);
  router_wnorm_kernel<<<1, 1024, 0, stream>>>(part, plan.nparts, E, wnorm);
  router_xnorm_kernel<<<static_cast<unsigned>(ceil_div64(T, 8)), 256, 0, stream>>>(reinterpret_cast<const uint4*>(x),
                                                                                   T, d / 8, xnorm, ovf);
  router_screen_kernel<<<dim3(ceil_div(T, kScrT), ceil_div(E, kScrE), plan.nsplit), kRtThreads, kScrSmemBytes,
                         stream>>>(mX, mHi, mLo, T, d, E, plan.kb_per_split, A);
  // add the K-split planes in order and the bias: A = plane 0
  router_reduce_partials_kernel<<<static_cast<unsigned>(ceil_div64(static_cast<int64_t>(T) * E, 256)), 256, 0,
                                  stream>>>(A, plan.nsplit, bias, T, E);
  const bool full = (d % 128) == 0;
  const uint16_t* xb = reinterpret_cast<const uint16_t*>(x);
#define MOE_RECHECK(MAXV, FULL)                                                                                   \
  router_recheck_kernel<MAXV, FULL><<<T, kRcWarps * 32, 0, stream>>>(A, xb, wt32, bias, xnorm, wnorm, T, d, E, k, idx, \
                                                                     w, ovf)
  if (E <= 256) {
    if (full) MOE_RECHECK(8, true); else MOE_RECHECK(8, false);
  } else {
    if (full) MOE_RECHECK(32, true); else MOE_RECHECK(32, false);
  }
#undef MOE_RECHECK
  router_fallback_kernel<<<T, 128, 0, stream>>>(ovf, xb, wt32, bias, d, E, k, idx, w);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// disp (one-token steps in moe_forward only): when the fused one-token router
// runs, it also writes these dispatch tables and *dispatched is set.
moe_status_t launch_route(const moe_bf16_t* x, const float* W_router, const float* bias, int T, int d, int E, int k,
                          int32_t* idx, float* w, void* ws, cudaStream_t stream,
                          const RouteDispatch* disp = nullptr, bool* dispatched = nullptr) {
  if (dispatched != nullptr) *dispatched = false;
  const RoutePlan plan = route_plan(T, d, E);
  if (plan.variant == kRouterTensorCore) return launch_route_tc(plan, x, W_router, bias, T, d, E, k, idx, w, ws, stream);
  float* lg = static_cast<float*>(ws);
  RouterVariant variant = plan.variant;
  if (variant == kRouterStream && !aligned16(W_router)) variant = T <= 8 ? kRouterSplitTiny : kRouterSplitSmall;
  if (variant == kRouterStream) {
    int sms = 0;
    const moe_status_t st = device_setup(&sms);
    if (st != MOE_OK) return st;
    uint8_t* base = static_cast<uint8_t*>(ws);
    float* logits = reinterpret_cast<float*>(base + plan.off_logits);
    unsigned int* tickets = reinterpret_cast<unsigned int*>(base + plan.off_tickets);
    const int G = ceil_div(E, kRsExperts);
    if (T == 1 &&
        cudaMemsetAsync(tickets, 0, static_cast<size_t>(G + 1) * sizeof(unsigned int), stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    const dim3 grid(G, plan.nchunks);
    const uint16_t* xb = reinterpret_cast<const uint16_t*>(x);
    const RouteDispatch none = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0};
    CUtensorMap wmap;
    if (T == 1 && d <= kR1MaxD && router_w_map(&wmap, W_router, d, E)) {
      // one CTA per 8 experts over all of d: no cross-CTA chunk sums
      router_one_token_kernel<<<static_cast<unsigned>(ceil_div(E, kR1Experts)), 256, router_one_smem_bytes(),
                                stream>>>(wmap, xb, bias, d, E, k, logits, tickets, idx, w,
                                          disp != nullptr ? *disp : none);
      if (dispatched != nullptr && disp != nullptr) *dispatched = true;
    } else if (T == 1) {
      router_stream_kernel<1><<<grid, kRsThreads, router_stream_smem_bytes(1), stream>>>(
          xb, W_router, bias, T, d, E, k, lg, logits, tickets, idx, w, disp != nullptr ? *disp : none);
      if (dispatched != nullptr && disp != nullptr) *dispatched = true;
    } else if (T <= 4) {
      router_stream_kernel<4><<<grid, kRsThreads, router_stream_smem_bytes(4), stream>>>(
          xb, W_router, bias, T, d, E, k, lg, logits, tickets, idx, w, none);
    } else {
      router_stream_kernel<16><<<grid, kRsThreads, router_stream_smem_bytes(16), stream>>>(
          xb, W_router, bias, T, d, E, k, lg, logits, tickets, idx, w, none);
    }
    if (T > 1) router_reduce_topk_kernel<<<T, 256, 0, stream>>>(lg, plan.nchunks, bias, T, E, k, idx, w);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  switch (variant) {
    case kRouterTensorCore:
    case kRouterStream:
      break;
    case kRouterFullBig: {
      dim3 grid(ceil_div(E, 64), ceil_div(T, 64), 1);
      router_logits_kernel<64, 64, 4, 4, false><<<grid, 256, 0, stream>>>(x, W_router, bias, T, d, E, lg);
      break;
    }
    case kRouterSplitBig: {
      dim3 grid(ceil_div(E, 64), ceil_div(T, 128), plan.nchunks);
      router_logits_kernel<128, 64, 8, 4, true><<<grid, 256, 0, stream>>>(x, W_router, nullptr, T, d, E, lg);
      break;
    }
    case kRouterSplitSmall: {
      dim3 grid(ceil_div(E, 64), ceil_div(T, 32), plan.nchunks);
      router_logits_kernel<32, 64, 2, 4, true><<<grid, 256, 0, stream>>>(x, W_router, nullptr, T, d, E, lg);
      break;
    }
    case kRouterSplitTiny: {
      dim3 grid(ceil_div(E, 128), 1, plan.nchunks);
      router_logits_kernel<8, 128, 2, 4, true><<<grid, 128, 0, stream>>>(x, W_router, nullptr, T, d, E, lg);
      break;
    }
  }
  if (variant != kRouterFullBig) {
    // ordered sum of the chunk partials, bias, softmax and top-k: one block per token
    router_reduce_topk_kernel<<<T, 256, 0, stream>>>(lg, plan.nchunks, bias, T, E, k, idx, w);
  } else {
    const unsigned blocks = static_cast<unsigned>(ceil_div64(T, 8));
    if (E <= 256)
      router_topk_kernel<8><<<blocks, 256, 0, stream>>>(lg, T, E, k, idx, w);
    else
      router_topk_kernel<32><<<blocks, 256, 0, stream>>>(lg, T, E, k, idx, w);
  }
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ----------------------------------------------------------------- permute

size_t permute_ws(int T, int E, int k) {
  const int64_t nblk = ceil_div64(static_cast<int64_t>(T) * k, kPairsPerBlock);
  return align256(static_cast<size_t>(nblk) * E * sizeof(int32_t));
}

moe_status_t launch_permute(const moe_bf16_t* x, const int32_t* idx, int T, int d, int E, int k, int32_t* offsets,
                            int32_t* perm_token, int32_t* inv_perm, moe_bf16_t* x_perm, void* ws,
                            cudaStream_t stream) {
  const int64_t n_pairs = static_cast<int64_t>(T) * k;
  const int nblk = static_cast<int>(ceil_div64(n_pairs, kPairsPerBlock));
  int32_t* block_hist = static_cast<int32_t*>(ws);
  const size_t sm = static_cast<size_t>(E) * sizeof(int32_t);
  permute_hist_kernel<<<nblk, 256, sm, stream>>>(idx, n_pairs, E, block_hist);
  permute_scan_kernel<<<1, 1024, 0, stream>>>(block_hist, nblk, E, offsets);
  permute_scatter_kernel<<<nblk, 32, sm, stream>>>(idx, n_pairs, E, k, block_hist, perm_token, inv_perm);
  if (x_perm != nullptr)  // token-major: each row of x is read once and written k times
    permute_copy_tokens_kernel<<<static_cast<unsigned>(T), 128, 0, stream>>>(
        reinterpret_cast<const uint4*>(x), inv_perm, k, d / 8, reinterpret_cast<uint4*>(x_perm));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// -------------------------------------------------------------- expert FFN

// Stream-K for a grouped GEMM whose output tiles (an upper bound from Tk and
// E) fill at most kStreamKMaxWaves waves of one CTA per SM of a 148-SM part:
// with that few tiles, whole-tile scheduling leaves SMs idle (a 64-tile
// one-token step uses 64 of 148 SMs; 448 tiles leave a fourth wave of 4), so
// the (tile, K block) units are split evenly over kStreamKCtas CTAs instead.
constexpr int kStreamKCtas = 148;
constexpr int kStreamKMaxWaves = 4;

// Workspace of the expert FFN: the two tile-prefix arrays, then (only when
// stream-K is possible for this Tk and E, i.e. min(E, Tk) <= the tile limit)
// the partials (two slots per CTA) and the tickets (one per tile and epilogue warp).
size_t ffn_split_part_bytes() {
  return align256(static_cast<size_t>(2 * kStreamKCtas) * kSplitPartFloats * sizeof(float));
}
size_t ffn_split_ticket_bytes() {
  return align256(static_cast<size_t>(kStreamKMaxWaves * kStreamKCtas) * kGemmEpiWarps * sizeof(unsigned));
}
bool ffn_split_possible(int Tk, int E) { return (E < Tk ? E : Tk) <= kStreamKMaxWaves * kStreamKCtas; }
size_t ffn_prefix_bytes(int E) { return align256(static_cast<size_t>(E + 1) * sizeof(int32_t)); }
size_t ffn_ws(int Tk, int E) {
  size_t b = 2 * ffn_prefix_bytes(E);
  if (ffn_split_possible(Tk, E)) b += ffn_split_part_bytes() + ffn_split_ticket_bytes();
  return b;
}

// W_router [d][E] fp32 (E contiguous) in boxes of kR1Experts experts x
// kR1BoxRows rows, unswizzled, for the one-token router.
bool router_w_map(CUtensorMap* map, const float* W, int d, int E) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(E), static_cast<cuuint64_t>(d)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(E) * 4};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kR1Experts), static_cast<cuuint32_t>(kR1BoxRows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(W), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
                const cuuint32_t* box) {
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
                              const_cast<void*>(base), dims, strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Weights W[E][K][N] (N contiguous): boxes of 64 features x 64 K rows of one expert.
bool weight_map(CUtensorMap* map, const moe_bf16_t* W, int E, int K, int N) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(E)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(N) * 2, static_cast<cuuint64_t>(N) * K * 2};
  const cuuint32_t box[3] = {64, 64, 1};
  return encode_map(map, W, 3, dims, strides, box);
}

// Activations A[rows][K] (K contiguous): boxes of 64 K x `box_rows` rows.
bool act_map(CUtensorMap* map, const moe_bf16_t* A, int rows, int K, int box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  return encode_map(map, A, 2, dims, strides, box);
}

struct FfnPlan {
  CUtensorMap mA0, mB0, mBs0, mA1, mB1, mBs1;
  GemmParams p0, p1;
  // gate/up on CTA pairs (pairs0, 256-row blocks; p0 with 256-feature tiles)
  bool pairs0 = false;
  int pair_grid = 0;
  int grid0, grid1;
  int mode0;  // gate/up: 0 256-row blocks, 2 128-row blocks
  int mode1;  // down: 1 (128-row blocks)
  int act = 0;  // gate/up GLU: 0 SwiGLU, 1 SiTU-GLU (p0.beta1, p0.beta2)
  int rows;                   // Tk: rows of x_perm, h and y_perm
  int split_ticket_words;     // stream-K tickets the schedule kernel clears (0: none)
  unsigned int* ticket_buf;   // where they are
};

moe_status_t plan_ffn(const moe_bf16_t* x_perm, const int32_t* offsets, const moe_bf16_t* Wgu, const moe_bf16_t* Wd,
                      int Tk, int d, int E, int f, moe_bf16_t* h, moe_bf16_t* y_perm, void* ws, int num_sms,
                      FfnPlan* fp) {
  if (!weight_map(&fp->mA0, Wgu, E, d, 2 * f) || !act_map(&fp->mB0, x_perm, Tk, d, kGemmBoxRows) ||
      !act_map(&fp->mBs0, x_perm, Tk, d, kGemmSmallBox) || !weight_map(&fp->mA1, Wd, E, f, d) ||
      !act_map(&fp->mB1, h, Tk, f, kGemmBoxRows) || !act_map(&fp->mBs1, h, Tk, f, kGemmSmallBox))
    return MOE_ERR_INVALID_ARG;
  int32_t* prefix0 = static_cast<int32_t*>(ws);
  int32_t* prefix1 = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + ffn_prefix_bytes(E));
  fp->rows = Tk;
  const int64_t min_e_tk = E < Tk ? E : Tk;
  GemmParams& p0 = fp->p0;
  p0.expert_offsets = offsets;
  p0.tile_prefix = prefix0;
  p0.E = E;
  p0.K = d;
  p0.n_feat = f;
  p0.n_feat_tiles = ceil_div(f, kGemmBMF);
  p0.a1_offset = f;
  p0.out = h;
  // 256-row blocks pay off only when experts average more than 128 rows
  fp->mode0 = (static_cast<int64_t>(Tk) > static_cast<int64_t>(E) * 128) ? 0 : 2;
  fp->mode1 = 1;
  const int64_t tiles0 = (ceil_div64(Tk, gemm_block_rows(fp->mode0)) + min_e_tk) * p0.n_feat_tiles;
  const bool stream_ok = ffn_split_possible(Tk, E);
  uint8_t* split_base = static_cast<uint8_t*>(ws) + 2 * ffn_prefix_bytes(E);
  float* part = stream_ok ? reinterpret_cast<float*>(split_base) : nullptr;
  unsigned int* tickets = stream_ok ? reinterpret_cast<unsigned int*>(split_base + ffn_split_part_bytes()) : nullptr;
  p0.b_fixed_row = -1;
  p0.stream_k = (stream_ok && fp->mode0 == 2 && tiles0 <= kStreamKMaxWaves * kStreamKCtas) ? 1 : 0;
  p0.part = p0.stream_k ? part : nullptr;
  p0.tickets = p0.stream_k ? tickets : nullptr;
  fp->grid0 = p0.stream_k ? (kStreamKCtas < num_sms ? kStreamKCtas : num_sms)
                          : static_cast<int>(tiles0 < num_sms ? tiles0 : num_sms);
  GemmParams& p1 = fp->p1;
  p1 = p0;
  p1.b_fixed_row = -1;
  p1.tile_prefix = prefix1;
  p1.K = f;
  p1.n_feat = d;
  p1.n_feat_tiles = ceil_div(d, 2 * kGemmBMF);
  p1.a1_offset = kGemmBMF;
  p1.out = y_perm;
  const int64_t tiles1 = (ceil_div64(Tk, gemm_block_rows(fp->mode1)) + min_e_tk) * p1.n_feat_tiles;
  p1.stream_k = (stream_ok && tiles1 <= kStreamKMaxWaves * kStreamKCtas) ? 1 : 0;
  p1.part = p1.stream_k ? part : nullptr;
  p1.tickets = p1.stream_k ? tickets : nullptr;
  fp->grid1 = p1.stream_k ? (kStreamKCtas < num_sms ? kStreamKCtas : num_sms)
                          : static_cast<int>(tiles1 < num_sms ? tiles1 : num_sms);
  // the tickets start at zero: the schedule kernel clears them (both GEMMs
  // share them; each tile's last contributor puts its tickets back to zero)
  const int64_t max_tiles = (p0.stream_k ? tiles0 : 0) > (p1.stream_k ? tiles1 : 0) ? (p0.stream_k ? tiles0 : 0)
                                                                                      : (p1.stream_k ? tiles1 : 0);
  fp->split_ticket_words = static_cast<int>(max_tiles) * kGemmEpiWarps;
  fp->ticket_buf = tickets;
  // experts average more than 128 rows (256-row blocks): the gate/up GEMM
  // runs on CTA pairs
  fp->pair_grid = device_pair_grid();
  fp->pairs0 = fp->mode0 == 0 && fp->pair_grid >= 2;
  return MOE_OK;
}

void launch_schedule(const FfnPlan& fp, cudaStream_t stream) {
  gemm_schedule_kernel<<<1, 1024, 0, stream>>>(fp.p0.expert_offsets, fp.p0.E, fp.rows, gemm_block_rows(fp.mode0),
                                               gemm_block_rows(fp.mode1), const_cast<int32_t*>(fp.p0.tile_prefix),
                                               const_cast<int32_t*>(fp.p1.tile_prefix), fp.ticket_buf,
                                               fp.split_ticket_words);
}
// The gate/up GEMM on CTA pairs (clusters of two): p0 as it stands at launch
// (callers set the GLU's caps after planning), with 256-feature tiles.
void launch_gemm_gate_up_pairs(const FfnPlan& fp, cudaStream_t stream) {
  GemmParams ph = fp.p0;
  ph.n_feat_tiles = ceil_div(ph.n_feat, 2 * kGemmBMF);
  ph.stream_k = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(fp.pair_grid));
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kPairSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (fp.act == 1)
    cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel<1>, fp.mA0, fp.mB0, ph);
  else
    cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel<0>, fp.mA0, fp.mB0, ph);
}
void launch_gemm_gate_up(const FfnPlan& fp, cudaStream_t stream) {
  if (fp.pairs0) {
    launch_gemm_gate_up_pairs(fp, stream);
    return;
  }
  if (fp.act == 1) {
    if (fp.mode0 == 0)
      grouped_gemm_kernel<0, 1><<<fp.grid0, kGemmThreads, GemmCfg<0>::kSmemBytes, stream>>>(fp.mA0, fp.mB0, fp.mBs0,
                                                                                             fp.p0);
    else
      grouped_gemm_kernel<2, 1><<<fp.grid0, kGemmThreads, GemmCfg<2>::kSmemBytes, stream>>>(fp.mA0, fp.mB0, fp.mBs0,
                                                                                             fp.p0);
    return;
  }
  if (fp.mode0 == 0)
    grouped_gemm_kernel<0><<<fp.grid0, kGemmThreads, GemmCfg<0>::kSmemBytes, stream>>>(fp.mA0, fp.mB0, fp.mBs0, fp.p0);
  else
    grouped_gemm_kernel<2><<<fp.grid0, kGemmThreads, GemmCfg<2>::kSmemBytes, stream>>>(fp.mA0, fp.mB0, fp.mBs0, fp.p0);
}
void launch_gemm_down(const FfnPlan& fp, cudaStream_t stream) {
  grouped_gemm_kernel<1><<<fp.grid1, kGemmThreads, GemmCfg<1>::kSmemBytes, stream>>>(fp.mA1, fp.mB1, fp.mBs1, fp.p1);
}

bool device_fused_ffn() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_mutex);
  return g_devices[dev].ready && g_devices[dev].fused_ffn;
}
bool device_one_token() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_mutex);
  return g_devices[dev].ready && g_devices[dev].one_token;
}

// Both GEMMs in one cooperative launch of min(148, SMs) CTAs (one per SM), so
// that every CTA whose down chunks wait for another CTA's h rows is resident.
// claim: the chunk counter (zero at launch).
moe_status_t launch_ffn_fused(FfnPlan& fp, unsigned int* h_ready, unsigned int* claim, int num_sms,
                              cudaStream_t stream) {
  const int grid = kStreamKCtas < num_sms ? kStreamKCtas : num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kFusedSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, grouped_ffn_fused_kernel, fp.mA0, fp.mBs0, fp.mA1, fp.mBs1, fp.p0,
                                           fp.p1, h_ready, claim);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t launch_ffn(const moe_bf16_t* x_perm, const int32_t* offsets, const moe_bf16_t* Wgu, const moe_bf16_t* Wd,
                        int Tk, int d, int E, int f, moe_bf16_t* h, moe_bf16_t* y_perm, void* ws, int num_sms,
                        cudaStream_t stream) {
  FfnPlan fp;
  const moe_status_t st = plan_ffn(x_perm, offsets, Wgu, Wd, Tk, d, E, f, h, y_perm, ws, num_sms, &fp);
  if (st != MOE_OK) return st;
  launch_schedule(fp, stream);
  launch_gemm_gate_up(fp, stream);
  launch_gemm_down(fp, stream);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// --------------------------------------------------------------- unpermute

template <int K>
void launch_unpermute_k(const moe_bf16_t* y_perm, const int32_t* inv_perm, const float* w, int T, int d,
                        moe_bf16_t* out, cudaStream_t stream) {
  const int vpr = d / 8;
  const int64_t n = static_cast<int64_t>(T) * vpr;
  unpermute_kernel<K><<<static_cast<unsigned>(ceil_div64(n, 256)), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(y_perm), inv_perm, w, T, vpr, reinterpret_cast<uint4*>(out));
}

moe_status_t launch_unpermute(const moe_bf16_t* y_perm, const int32_t* inv_perm, const float* w, int T, int d, int k,
                              moe_bf16_t* out, cudaStream_t stream) {
  switch (k) {
#define MOE_UNPERMUTE_CASE(K) \
  case K: launch_unpermute_k<K>(y_perm, inv_perm, w, T, d, out, stream); break;
    MOE_UNPERMUTE_CASE(1) MOE_UNPERMUTE_CASE(2) MOE_UNPERMUTE_CASE(3) MOE_UNPERMUTE_CASE(4)
    MOE_UNPERMUTE_CASE(5) MOE_UNPERMUTE_CASE(6) MOE_UNPERMUTE_CASE(7) MOE_UNPERMUTE_CASE(8)
    MOE_UNPERMUTE_CASE(9) MOE_UNPERMUTE_CASE(10) MOE_UNPERMUTE_CASE(11) MOE_UNPERMUTE_CASE(12)
    MOE_UNPERMUTE_CASE(13) MOE_UNPERMUTE_CASE(14) MOE_UNPERMUTE_CASE(15) MOE_UNPERMUTE_CASE(16)
#undef MOE_UNPERMUTE_CASE
    default: return MOE_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ----------------------------------------------------------------- forward

struct ForwardLayout {
  size_t route, idx, w, offsets, perm_token, inv_perm, x_perm, h, y_perm, perm_ws, ffn_ws, fused_ws, total;
};

// Steps in which no expert can hold more than this many rows (T <= 32) run
// both GEMMs in one cooperative launch (grouped_ffn_fused_kernel).
constexpr int kFusedMaxTokens = kGemmSmallBox;
bool ffn_fused_shape(int T) { return T <= kFusedMaxTokens; }

// The fused launch's down GEMM has its own tickets (one per tile and epilogue
// warp) and partial slots, plus the h_ready counters [E] and the chunk
// counter. They sit right after the gate/up GEMM's tickets, which end the
// feed-forward workspace, so one zeroing pass clears both GEMMs' tickets and
// the counters: [tickets0][tickets1][h_ready][claim][part1]. Each GEMM's
// partials are kFusedSlots compact slots (2 x 32 rows x 128 features fp32),
// which fill exactly the stream-K partial area of the two-launch path.
size_t fused_ticket_words() { return static_cast<size_t>(kStreamKMaxWaves * kStreamKCtas) * kGemmEpiWarps; }
size_t fused_counter_words(int E) { return fused_ticket_words() + static_cast<size_t>(E) + 1; }
static_assert(static_cast<size_t>(kFusedSlots) * 2 * kGemmSmallBox * kGemmBMF <=
                  static_cast<size_t>(2 * kStreamKCtas) * kSplitPartFloats,
              "fused partial slots");
static_assert(kFusedSlots / 2 <= kStreamKMaxWaves * kStreamKCtas,
              "a GEMM cut into chunks has at most kFusedSlots / 2 tiles, each with its tickets");
size_t fused_ws(int E) { return align256(fused_counter_words(E) * sizeof(unsigned)) + ffn_split_part_bytes(); }

ForwardLayout forward_layout(int T, int d, int E, int k, int f) {
  ForwardLayout L;
  const size_t Tk = static_cast<size_t>(T) * k;
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t here = at;
    at += align256(bytes);
    return here;
  };
  L.route = take(route_plan(T, d, E).ws_bytes);
  L.idx = take(Tk * sizeof(int32_t));
  L.w = take(Tk * sizeof(float));
  L.offsets = take((static_cast<size_t>(E) + 1) * sizeof(int32_t));
  L.perm_token = take(Tk * sizeof(int32_t));
  L.inv_perm = take(Tk * sizeof(int32_t));
  L.x_perm = take(Tk * d * 2);
  L.h = take(Tk * f * 2);
  L.y_perm = take(Tk * d * 2);
  L.perm_ws = take(permute_ws(T, E, k));
  L.ffn_ws = take(ffn_ws(T * k, E));
  L.fused_ws = ffn_fused_shape(T) ? take(fused_ws(E)) : 0;
  L.total = at;
  return L;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
  }
  return "MOE_ERR_UNKNOWN";
}

int moe_version(void) { return 100; }

size_t moe_route_workspace_size(int T, int d, int E) {
  if (T < 1 || d < 1 || E < 1) return 0;
  return route_plan(T, d, E).ws_bytes;
}

moe_status_t moe_route(const moe_bf16_t* x, const float* W_router, const float* router_bias, int T, int d, int E,
                       int k, int32_t* topk_idx, float* topk_w, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream) {
  if (!x || !W_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(T, d, E, k) || !aligned16(x)) return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK || E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (!workspace || !aligned256(workspace) || workspace_bytes < route_plan(T, d, E).ws_bytes) return MOE_ERR_WORKSPACE;
  return launch_route(x, W_router, router_bias, T, d, E, k, topk_idx, topk_w, workspace, stream);
}

size_t moe_permute_workspace_size(int T, int E, int k) {
  if (T < 1 || E < 1 || k < 1) return 0;
  return permute_ws(T, E, k);
}

moe_status_t moe_permute(const moe_bf16_t* x, const int32_t* topk_idx, int T, int d, int E, int k,
                         int32_t* expert_offsets, int32_t* perm_token, int32_t* inv_perm, moe_bf16_t* x_perm,
                         void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!topk_idx || !expert_offsets || !perm_token || !inv_perm) return MOE_ERR_INVALID_ARG;
  if (x_perm != nullptr && (x == nullptr || !aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(T, d, E, k)) return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK || E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (!workspace || !aligned256(workspace) || workspace_bytes < permute_ws(T, E, k)) return MOE_ERR_WORKSPACE;
  return launch_permute(x, topk_idx, T, d, E, k, expert_offsets, perm_token, inv_perm, x_perm, workspace, stream);
}

size_t moe_expert_ffn_workspace_size(int Tk, int E) {
  if (Tk < 0 || E < 1) return 0;
  return ffn_ws(Tk, E);
}

moe_status_t moe_expert_ffn(const moe_bf16_t* x_perm, const int32_t* expert_offsets, const moe_bf16_t* W_gate_up,
                            const moe_bf16_t* W_down, int Tk, int d, int E, int f, moe_bf16_t* h, moe_bf16_t* y_perm,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!x_perm || !expert_offsets || !W_gate_up || !W_down || !h || !y_perm) return MOE_ERR_INVALID_ARG;
  if (Tk < 1 || d < 64 || d % 64 || f < 64 || f % 64 || d > 32768 || f > 32768 || E < 1) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_perm) || !aligned16(W_gate_up) || !aligned16(W_down) || !aligned16(h) || !aligned16(y_perm))
    return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (!workspace || !aligned256(workspace) || workspace_bytes < ffn_ws(Tk, E)) return MOE_ERR_WORKSPACE;
  int sms = 0;
  const moe_status_t st = device_setup(&sms);
  if (st != MOE_OK) return st;
  return launch_ffn(x_perm, expert_offsets, W_gate_up, W_down, Tk, d, E, f, h, y_perm, workspace, sms, stream);
}

moe_status_t moe_unpermute(const moe_bf16_t* y_perm, const int32_t* inv_perm, const float* topk_w, int T, int d, int k,
                           moe_bf16_t* out, cudaStream_t stream) {
  if (!y_perm || !inv_perm || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  if (T < 1 || d < 64 || d % 64 || d > 32768 || k < 1 || !aligned16(y_perm) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  return launch_unpermute(y_perm, inv_perm, topk_w, T, d, k, out, stream);
}

size_t moe_forward_workspace_size(int T, int d, int E, int k, int f) {
  if (T < 1 || d < 1 || E < 1 || k < 1 || f < 1) return 0;
  return forward_layout(T, d, E, k, f).total;
}

}  // extern "C"

namespace {

// One token, the whole layer in one cooperative launch (moe_one_token_kernel,
// one CTA per SM; the router needs ceil(E / 8) of them). fp is the fused
// feed-forward's plan with its tickets set. Returns MOE_ERR_UNSUPPORTED, with
// nothing enqueued, when the shape or the device does not allow it.
moe_status_t launch_one_token(const moe_bf16_t* x, const float* W_router, const float* bias, int d, int E, int k,
                              FfnPlan& fp, unsigned int* h_ready, uint8_t* ws, const ForwardLayout& L, int sms,
                              moe_bf16_t* out, cudaStream_t stream) {
  const RoutePlan plan = route_plan(1, d, E);
  const int grid = kStreamKCtas < sms ? kStreamKCtas : sms;
  if (plan.variant != kRouterStream || d > kR1MaxD || k > kOneTokenMaxK || !aligned16(W_router) ||
      ceil_div(E, kR1Experts) > grid || !device_one_token())
    return MOE_ERR_UNSUPPORTED;
  CUtensorMap wmap;
  if (!router_w_map(&wmap, W_router, d, E) || !act_map(&fp.mBs0, x, 1, d, kGemmSmallBox)) return MOE_ERR_UNSUPPORTED;
  fp.p0.b_fixed_row = 0;  // every gate/up tile's token operand is x itself
  uint8_t* rws = ws + L.route;
  unsigned int* sync = reinterpret_cast<unsigned int*>(rws + plan.off_tickets);
  if (cudaMemsetAsync(sync, 0, 2 * sizeof(unsigned int), stream) != cudaSuccess) return MOE_ERR_CUDA;
  OneTokenArgs a;
  a.x = reinterpret_cast<const uint16_t*>(x);
  a.bias = bias;
  a.d = d;
  a.E = E;
  a.k = k;
  a.logits = reinterpret_cast<float*>(rws + plan.off_logits);
  a.sync = sync;
  a.topk_idx = reinterpret_cast<int32_t*>(ws + L.idx);
  a.topk_w = reinterpret_cast<float*>(ws + L.w);
  a.inv_perm = reinterpret_cast<int32_t*>(ws + L.inv_perm);
  a.zero_buf = fp.ticket_buf;
  a.zero_n = fp.split_ticket_words;
  a.h_ready = h_ready;
  a.claim = h_ready + E;
  a.out = reinterpret_cast<uint16_t*>(out);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kOneTokenSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  nvtxRangePushA("moe.one_token");
  const cudaError_t e =
      cudaLaunchKernelEx(&cfg, moe_one_token_kernel, wmap, fp.mA0, fp.mBs0, fp.mA1, fp.mBs1, fp.p0, fp.p1, a);
  nvtxRangePop();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t forward_impl(const moe_bf16_t* x, const float* W_router, const float* router_bias,
                          const moe_bf16_t* W_gate_up, const moe_bf16_t* W_down, int T, int d, int E, int k, int f,
                          moe_bf16_t* out, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                          cudaEvent_t* ev) {
  if (!x || !W_router || !W_gate_up || !W_down || !out) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(T, d, E, k) || f < 64 || f % 64 || f > 32768) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(W_gate_up) || !aligned16(W_down) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK || E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  const ForwardLayout L = forward_layout(T, d, E, k, f);
  if (!workspace || !aligned256(workspace) || workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
  int sms = 0;
  moe_status_t st = device_setup(&sms);
  if (st != MOE_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
  float* w = reinterpret_cast<float*>(ws + L.w);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* perm_token = reinterpret_cast<int32_t*>(ws + L.perm_token);
  int32_t* inv_perm = reinterpret_cast<int32_t*>(ws + L.inv_perm);
  moe_bf16_t* x_perm = reinterpret_cast<moe_bf16_t*>(ws + L.x_perm);
  moe_bf16_t* h = reinterpret_cast<moe_bf16_t*>(ws + L.h);
  moe_bf16_t* y_perm = reinterpret_cast<moe_bf16_t*>(ws + L.y_perm);
  const int Tk = T * k;
  FfnPlan fp;
  st = plan_ffn(x_perm, offsets, W_gate_up, W_down, Tk, d, E, f, h, y_perm, ws + L.ffn_ws, sms, &fp);
  if (st != MOE_OK) return st;
  // few tokens: both GEMMs in one cooperative launch, the down phase with its
  // own tickets and partial slots; the zeroing that clears the gate/up
  // tickets (router or dispatch kernel) covers the down tickets and h_ready too
  unsigned int* h_ready = nullptr;
  const bool fused = ffn_fused_shape(T) && device_fused_ffn() && fp.ticket_buf != nullptr &&
                     reinterpret_cast<uint8_t*>(fp.ticket_buf) + ffn_split_ticket_bytes() == ws + L.fused_ws;
  if (fused) {
    unsigned int* tickets1 = fp.ticket_buf + fused_ticket_words();
    h_ready = tickets1 + fused_ticket_words();
    fp.p0.tickets = fp.ticket_buf;
    fp.p0.part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(fp.ticket_buf) - ffn_split_part_bytes());
    fp.p1.tickets = tickets1;
    fp.p1.part = reinterpret_cast<float*>(ws + L.fused_ws + align256(fused_counter_words(E) * sizeof(unsigned)));
    fp.p0.part_rows = kGemmSmallBox;  // no tile of a step of <= 32 tokens has more rows
    fp.p1.part_rows = kGemmSmallBox;
    fp.split_ticket_words = static_cast<int>(fused_ticket_words() + fused_counter_words(E));
  }
  // one token (untimed calls): router, dispatch, both GEMMs and the combine in one launch
  if (T == 1 && fused && ev == nullptr) {
    st = launch_one_token(x, W_router, router_bias, d, E, k, fp, h_ready, ws, L, sms, out, stream);
    if (st != MOE_ERR_UNSUPPORTED) return st;
  }
  // stage boundaries: events (timed calls) and NVTX ranges named for the
  // stage, which profilers show around the stage's launches (no cost without one)
  static const char* const kStage[MOE_TIMED_STAGES] = {"moe.route", "moe.dispatch", "moe.gate_up", "moe.down",
                                                       "moe.combine"};
  struct NvtxStage {  // closes a range left open by an early return
    bool open = false;
    ~NvtxStage() {
      if (open) nvtxRangePop();
    }
  } nv;
  auto mark = [&](int i) {
    if (ev) cudaEventRecord(ev[i], stream);
    if (i % 2 == 0) {
      nvtxRangePushA(kStage[i / 2]);
      nv.open = true;
    } else {
      nvtxRangePop();
      nv.open = false;
    }
  };
  mark(0);
  // one token: the router's last CTA also writes the dispatch tables, and the
  // gate/up GEMM reads its token operand straight from x (every tile is that
  // one row), so neither the dispatch kernel nor the row copy runs
  const RouteDispatch disp = {offsets, perm_token, inv_perm, const_cast<int32_t*>(fp.p0.tile_prefix),
                              const_cast<int32_t*>(fp.p1.tile_prefix), fp.ticket_buf, fp.split_ticket_words};
  bool dispatched = false;
  st = launch_route(x, W_router, router_bias, T, d, E, k, idx, w, ws + L.route, stream, T == 1 ? &disp : nullptr,
                    &dispatched);
  if (st != MOE_OK) return st;
  mark(1);
  mark(2);
  if (dispatched) {
    if (act_map(&fp.mB0, x, 1, d, kGemmBoxRows) && act_map(&fp.mBs0, x, 1, d, kGemmSmallBox)) {
      fp.p0.b_fixed_row = 0;
    } else {  // the maps of the permuted copy stay; make the copy
      permute_copy_rows_kernel<<<static_cast<unsigned>(ceil_div64(Tk, 8)), 256, 0, stream>>>(
          reinterpret_cast<const uint4*>(x), T, perm_token, Tk, d / 8, reinterpret_cast<uint4*>(x_perm));
    }
  } else if (Tk <= kSmallDispatchPairs) {
    // one block: counts, offsets, stable scatter and both GEMM tile prefixes; then the row copy
    dispatch_small_kernel<<<1, 1024, 0, stream>>>(idx, Tk, E, k, gemm_block_rows(fp.mode0), gemm_block_rows(fp.mode1),
                                                  offsets, perm_token, inv_perm,
                                                  const_cast<int32_t*>(fp.p0.tile_prefix),
                                                  const_cast<int32_t*>(fp.p1.tile_prefix), fp.ticket_buf,
                                                  fp.split_ticket_words);
    permute_copy_rows_kernel<<<static_cast<unsigned>(ceil_div64(Tk, 8)), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(x), T, perm_token, Tk, d / 8, reinterpret_cast<uint4*>(x_perm));
  } else {
    st = launch_permute(x, idx, T, d, E, k, offsets, perm_token, inv_perm, x_perm, ws + L.perm_ws, stream);
    if (st != MOE_OK) return st;
    launch_schedule(fp, stream);
  }
  mark(3);
  mark(4);
  if (fused) {
    st = launch_ffn_fused(fp, h_ready, h_ready + E, sms, stream);
    if (st != MOE_OK) return st;
  } else {
    launch_gemm_gate_up(fp, stream);
  }
  mark(5);
  mark(6);
  if (!fused) launch_gemm_down(fp, stream);
  mark(7);
  mark(8);
  st = launch_unpermute(y_perm, inv_perm, w, T, d, k, out, stream);
  mark(9);
  if (st != MOE_OK) return st;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

extern "C" {

moe_status_t moe_forward(const moe_bf16_t* x, const float* W_router, const float* router_bias,
                         const moe_bf16_t* W_gate_up, const moe_bf16_t* W_down, int T, int d, int E, int k, int f,
                         moe_bf16_t* out, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return forward_impl(x, W_router, router_bias, W_gate_up, W_down, T, d, E, k, f, out, workspace, workspace_bytes,
                      stream, nullptr);
}

moe_status_t moe_forward_timed(const moe_bf16_t* x, const float* W_router, const float* router_bias,
                               const moe_bf16_t* W_gate_up, const moe_bf16_t* W_down, int T, int d, int E, int k,
                               int f, moe_bf16_t* out, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                               cudaEvent_t* events) {
  if (!events) return MOE_ERR_INVALID_ARG;
  return forward_impl(x, W_router, router_bias, W_gate_up, W_down, T, d, E, k, f, out, workspace, workspace_bytes,
                      stream, events);
}

size_t moe_forward_host_workspace_size(int T, int d, int E, int k, int f) {
  const size_t fw = moe_forward_workspace_size(T, d, E, k, f);
  if (fw == 0) return 0;
  return 2 * align256(static_cast<size_t>(T) * d * sizeof(moe_bf16_t)) + fw;
}

moe_status_t moe_forward_host(const moe_bf16_t* x_host, const float* W_router, const float* router_bias,
                              const moe_bf16_t* W_gate_up, const moe_bf16_t* W_down, int T, int d, int E, int k,
                              int f, moe_bf16_t* out_host, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
  if (!x_host || !W_router || !W_gate_up || !W_down || !out_host) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(T, d, E, k) || f < 64 || f % 64 || f > 32768) return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK || E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  const size_t stage = align256(static_cast<size_t>(T) * d * sizeof(moe_bf16_t));
  const size_t need = moe_forward_host_workspace_size(T, d, E, k, f);
  if (!workspace || !aligned256(workspace) || workspace_bytes < need) return MOE_ERR_WORKSPACE;
  // x and out must be host memory (pageable or page-locked), never device memory
  for (const void* hp : {static_cast<const void*>(x_host), static_cast<const void*>(out_host)}) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, hp) != cudaSuccess) return MOE_ERR_CUDA;
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return MOE_ERR_INVALID_ARG;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  moe_bf16_t* x_dev = reinterpret_cast<moe_bf16_t*>(ws);
  moe_bf16_t* out_dev = reinterpret_cast<moe_bf16_t*>(ws + stage);
  const size_t bytes = static_cast<size_t>(T) * d * sizeof(moe_bf16_t);
  if (cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess) return MOE_ERR_CUDA;
  const moe_status_t st = forward_impl(x_dev, W_router, router_bias, W_gate_up, W_down, T, d, E, k, f, out_dev,
                                       ws + 2 * stage, workspace_bytes - 2 * stage, stream, nullptr);
  if (st != MOE_OK) return st;
  if (cudaMemcpyAsync(out_host, out_dev, bytes, cudaMemcpyDeviceToHost, stream) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"

// ------------------------------------------------ allocation-free router scratch
//
// The scratch of moe_route_noalloc: one fixed array per device, so callers
// that cannot allocate device memory can still route. Host code must not use
// the symbol itself as a pointer (on the host it names a stand-in, not device
// memory); noalloc_route_scratch() looks up the device address once per
// device, with that device current, and the kernels get that address.
static __device__ __align__(256) unsigned char g_route_noalloc_scratch[MOE_ROUTE_NOALLOC_SCRATCH_BYTES];

namespace {

void* g_route_noalloc_ptr[kMaxDevices] = {};
std::mutex g_route_noalloc_mutex;

moe_status_t noalloc_route_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_route_noalloc_mutex);
  if (g_route_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_noalloc_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_route_noalloc_ptr[dev] = p;
  }
  *out = g_route_noalloc_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status_t moe_route_noalloc(const moe_bf16_t* x, const float* W_router, const float* router_bias, int T, int d,
                               int E, int k, int32_t* topk_idx, float* topk_w, cudaStream_t stream) {
  if (!x || !W_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(T, d, E, k) || !aligned16(x)) return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK || E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (route_plan(T, d, E).ws_bytes > MOE_ROUTE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const moe_status_t st = noalloc_route_scratch(&scratch);
  if (st != MOE_OK) return st;
  return launch_route(x, W_router, router_bias, T, d, E, k, topk_idx, topk_w, scratch, stream);
}

moe_status_t moe_mxfp8_quantize(const moe_bf16_t* x, int rows, int cols, uint8_t* codes, uint8_t* scales,
                                cudaStream_t stream) {
  if (!x || !codes || !scales) return MOE_ERR_INVALID_ARG;
  if (rows < 1 || cols < moe::kMxBlock || cols > (1 << 20) || cols % moe::kMxBlock) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes)) return MOE_ERR_INVALID_ARG;
  const int64_t nblocks = static_cast<int64_t>(rows) * (cols / moe::kMxBlock);
  const int64_t grid = ceil_div64(nblocks, 256);
  if (grid > 0x7fffffff) return MOE_ERR_UNSUPPORTED;
  moe::mxfp8_quantize_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(reinterpret_cast<const uint4*>(x),
                                                                               nblocks, codes, scales);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_mxfp4_quantize(const moe_bf16_t* w, int K, int N, uint8_t* codes, uint8_t* scales,
                                cudaStream_t stream) {
  if (!w || !codes || !scales) return MOE_ERR_INVALID_ARG;
  if (K < moe::kMxBlock || K > (1 << 20) || K % moe::kMxBlock || N < 1 || N > (1 << 20)) return MOE_ERR_INVALID_ARG;
  const auto addr = [](const void* p) { return reinterpret_cast<uintptr_t>(p); };
  const bool x4 = N % 4 == 0 && addr(w) % 8 == 0 && addr(codes) % 4 == 0 && addr(scales) % 4 == 0;
  const int64_t groups = static_cast<int64_t>(K / moe::kMxBlock) * (x4 ? N / 4 : N);
  const int64_t grid = ceil_div64(groups, 256);
  if (grid > 0x7fffffff) return MOE_ERR_UNSUPPORTED;
  if (x4)
    moe::mxfp4_quantize_x4_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        reinterpret_cast<const uint2*>(w), K, N / 4, reinterpret_cast<uint32_t*>(codes),
        reinterpret_cast<uint32_t*>(scales));
  else
    moe::mxfp4_quantize_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(w, K, N, codes, scales);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"

// ------------------------------------------------------- MX expert FFN path

namespace {

std::mutex g_mx_mutex;
bool g_mx_ready[kMaxDevices] = {};

// Shared-memory limits of the MX GEMMs (once per device, on first MX use only).
moe_status_t mx_setup(int* num_sms) {
  moe_status_t st = device_setup(num_sms);
  if (st != MOE_OK) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mx_mutex);
  if (!g_mx_ready[dev]) {
    if (cudaFuncSetAttribute(mx_grouped_gemm_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kMxSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(mx_grouped_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kMxSmemBytes) != cudaSuccess)
      return MOE_ERR_CUDA;
    g_mx_ready[dev] = true;
  }
  return MOE_OK;
}

bool encode_map_typed(CUtensorMap* map, CUtensorMapDataType type, const void* base, int rank, const cuuint64_t* dims,
                      const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, type, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides_bytes,
                              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Packed E2M1 weights Wq[E][rows][K / 2]: boxes of 128 K x 128 rows of one
// expert, unpacked to one byte per element in shared memory.
bool mx_weight_map(CUtensorMap* map, const uint8_t* wq, int E, int rows, int K) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(E)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) / 2, static_cast<cuuint64_t>(rows) * K / 2};
  const cuuint32_t box[3] = {128, 128, 1};
  return encode_map_typed(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, wq, 3, dims, strides, box);
}

// E4M3 token rows [rows][K]: boxes of 128 K x box_rows rows.
bool mx_token_map(CUtensorMap* map, const uint8_t* q, int rows, int K, int box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
  return encode_map_typed(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, 2, dims, strides, box);
}

bool mx_shape_ok(int d, int f) { return d % 256 == 0 && f % 128 == 0 && f >= 128 && f <= 32768; }

inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

struct MxLayout {
  size_t route, idx, w, offsets, perm_token, inv_perm, xq, sfx, hq, sfh, y, perm_ws, pre0, pre1, part, tickets, total;
  int64_t tiles_max;
  bool split0, split1;  // stream-K for the gate/up and the down GEMM
};

// Stream-K for an MX GEMM whose tile count (an upper bound) fills at most four
// waves of one CTA per SM on a 148-SM part, as for the bf16 GEMMs.
constexpr int kMxSplitCtas = 148;
constexpr int64_t kMxSplitMaxTiles = 4 * kMxSplitCtas;

MxLayout mx_layout(int T, int d, int E, int k, int f) {
  MxLayout L;
  const size_t Tk = static_cast<size_t>(T) * k;
  L.tiles_max = ceil_div64(static_cast<int64_t>(Tk), kMxTileRows) + (E < static_cast<int64_t>(Tk) ? E : Tk);
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t here = at;
    at += align256(bytes);
    return here;
  };
  L.route = take(route_plan(T, d, E).ws_bytes);
  L.idx = take(Tk * sizeof(int32_t));
  L.w = take(Tk * sizeof(float));
  L.offsets = take((static_cast<size_t>(E) + 1) * sizeof(int32_t));
  L.perm_token = take(Tk * sizeof(int32_t));
  L.inv_perm = take(Tk * sizeof(int32_t));
  L.xq = take(Tk * d);
  L.sfx = take(static_cast<size_t>(L.tiles_max) * (d / 128) * kMxAtomBytes);
  L.hq = take(Tk * f);
  L.sfh = take(static_cast<size_t>(L.tiles_max) * (f / 128) * kMxAtomBytes);
  L.y = take(Tk * d * 2);
  L.perm_ws = take(permute_ws(T, E, k));
  L.pre0 = take((static_cast<size_t>(E) + 1) * sizeof(int32_t));
  L.pre1 = take((static_cast<size_t>(E) + 1) * sizeof(int32_t));
  L.split0 = L.tiles_max * (f / 128) <= kMxSplitMaxTiles;
  L.split1 = L.tiles_max * (d / 256) <= kMxSplitMaxTiles;
  const bool split = L.split0 || L.split1;
  L.part = take(split ? static_cast<size_t>(2 * kMxSplitCtas) * kMxPartFloats * sizeof(float) : 0);
  L.tickets = take(split ? static_cast<size_t>(kMxSplitMaxTiles) * 4 * sizeof(unsigned int) : 0);
  L.total = at;
  return L;
}

}  // namespace

extern "C" {

moe_status_t moe_mx_expert_bytes(int E, int d, int f, size_t* wq_gate_up, size_t* sf_gate_up, size_t* wq_down,
                                 size_t* sf_down) {
  if (!wq_gate_up || !sf_gate_up || !wq_down || !sf_down) return MOE_ERR_INVALID_ARG;
  if (E < 1 || d < 256 || d > 32768 || !mx_shape_ok(d, f)) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  const size_t n = static_cast<size_t>(E) * d * f;  // elements of W_down; W_gate_up has 2n
  *wq_gate_up = n;       // 2n codes, two per byte
  *sf_gate_up = n / 16;  // one scale per 32 codes
  *wq_down = n / 2;
  *sf_down = n / 32;
  return MOE_OK;
}

moe_status_t moe_mx_pack_experts(const moe_bf16_t* W_gate_up, const moe_bf16_t* W_down, int E, int d, int f,
                                 uint8_t* wq_gate_up, uint8_t* sf_gate_up, uint8_t* wq_down, uint8_t* sf_down,
                                 cudaStream_t stream) {
  size_t b0, b1, b2, b3;
  const moe_status_t st = moe_mx_expert_bytes(E, d, f, &b0, &b1, &b2, &b3);
  if (st != MOE_OK) return st;
  if (!W_gate_up || !W_down || !wq_gate_up || !sf_gate_up || !wq_down || !sf_down) return MOE_ERR_INVALID_ARG;
  if (!aligned32(wq_gate_up) || !aligned32(wq_down) || !aligned16(sf_gate_up) || !aligned16(sf_down))
    return MOE_ERR_INVALID_ARG;
  const int64_t g0 = static_cast<int64_t>(E) * (d / kMxBlock) * (2 * f);
  const int64_t g1 = static_cast<int64_t>(E) * (f / kMxBlock) * d;
  mx_pack_weights_kernel<<<static_cast<unsigned>(ceil_div64(g0, 256)), 256, 0, stream>>>(W_gate_up, E, d, 2 * f,
                                                                                        wq_gate_up, sf_gate_up);
  mx_pack_weights_kernel<<<static_cast<unsigned>(ceil_div64(g1, 256)), 256, 0, stream>>>(W_down, E, f, d, wq_down,
                                                                                        sf_down);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

size_t moe_forward_mx_workspace_size(int T, int d, int E, int k, int f) {
  if (T < 1 || d < 1 || E < 1 || k < 1 || f < 1 || !mx_shape_ok(d, f)) return 0;
  return mx_layout(T, d, E, k, f).total;
}

moe_status_t moe_forward_mx(const moe_bf16_t* x, const float* W_router, const float* router_bias,
                            const uint8_t* wq_gate_up, const uint8_t* sf_gate_up, const uint8_t* wq_down,
                            const uint8_t* sf_down, int T, int d, int E, int k, int f, moe_bf16_t* out,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!x || !W_router || !wq_gate_up || !sf_gate_up || !wq_down || !sf_down || !out) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(T, d, E, k) || !mx_shape_ok(d, f)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out) || !aligned32(wq_gate_up) || !aligned32(wq_down) || !aligned16(sf_gate_up) ||
      !aligned16(sf_down))
    return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK || E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  const MxLayout L = mx_layout(T, d, E, k, f);
  if (!workspace || !aligned256(workspace) || workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
  int sms = 0;
  moe_status_t st = mx_setup(&sms);
  if (st != MOE_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
  float* w = reinterpret_cast<float*>(ws + L.w);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* perm_token = reinterpret_cast<int32_t*>(ws + L.perm_token);
  int32_t* inv_perm = reinterpret_cast<int32_t*>(ws + L.inv_perm);
  uint8_t* xq = ws + L.xq;
  uint8_t* sfx = ws + L.sfx;
  uint8_t* hq = ws + L.hq;
  uint8_t* sfh = ws + L.sfh;
  moe_bf16_t* y = reinterpret_cast<moe_bf16_t*>(ws + L.y);
  int32_t* pre0 = reinterpret_cast<int32_t*>(ws + L.pre0);
  int32_t* pre1 = reinterpret_cast<int32_t*>(ws + L.pre1);
  const int Tk = T * k;
  CUtensorMap mA0, mB0, mBs0, mA1, mB1, mBs1;
  if (!mx_weight_map(&mA0, wq_gate_up, E, 2 * f, d) || !mx_token_map(&mB0, xq, Tk, d, kMxTileRows) ||
      !mx_token_map(&mBs0, xq, Tk, d, kMxSmallRows) || !mx_weight_map(&mA1, wq_down, E, d, f) ||
      !mx_token_map(&mB1, hq, Tk, f, kMxTileRows) || !mx_token_map(&mBs1, hq, Tk, f, kMxSmallRows))
    return MOE_ERR_INVALID_ARG;

  // route, then the dispatch tables (counts, offsets, permutation, token tiles
  // of kMxTileRows rows); no bf16 row copy: the rows are copied as MXFP8 below
  // stream-K tickets start at zero: the dispatch step clears them
  unsigned int* tickets = reinterpret_cast<unsigned int*>(ws + L.tickets);
  const int ticket_words =
      static_cast<int>((L.split0 || L.split1) ? static_cast<int64_t>(kMxSplitMaxTiles) * 4 : 0);
  const RouteDispatch disp = {offsets, perm_token, inv_perm, pre0, pre1, tickets, ticket_words};
  bool dispatched = false;
  st = launch_route(x, W_router, router_bias, T, d, E, k, idx, w, ws + L.route, stream, T == 1 ? &disp : nullptr,
                    &dispatched);
  if (st != MOE_OK) return st;
  if (!dispatched) {
    if (Tk <= kSmallDispatchPairs) {
      dispatch_small_kernel<<<1, 1024, 0, stream>>>(idx, Tk, E, k, kMxTileRows, kMxTileRows, offsets, perm_token,
                                                    inv_perm, pre0, pre1, tickets, ticket_words);
    } else {
      st = launch_permute(x, idx, T, d, E, k, offsets, perm_token, inv_perm, nullptr, ws + L.perm_ws, stream);
      if (st != MOE_OK) return st;
      gemm_schedule_kernel<<<1, 1024, 0, stream>>>(offsets, E, Tk, kMxTileRows, kMxTileRows, pre0, pre1, tickets,
                                                   ticket_words);
    }
  }
  {
    // few tokens: one warp per CTA and several CTAs per token (a block per thread)
    const int nblk = d / kMxBlock;
    const bool spread = T < 64;
    const unsigned threads = spread ? 32u : 256u;
    const dim3 grid(static_cast<unsigned>(T), spread ? static_cast<unsigned>(ceil_div(nblk, 32)) : 1u);
    mx_quantize_dispatch_kernel<<<grid, threads, 0, stream>>>(reinterpret_cast<const uint4*>(x), idx, inv_perm,
                                                             offsets, pre0, d, k, E, xq, sfx);
  }

  MxGemmParams p0;
  p0.expert_offsets = offsets;
  p0.tile_prefix = pre0;
  p0.E = E;
  p0.K = d;
  p0.n_feat = f;
  p0.n_feat_tiles = f / 128;
  p0.a1_row = f;
  p0.w_rows = 2 * f;
  p0.sfw = sf_gate_up;
  p0.sft = sfx;
  p0.hq = hq;
  p0.hs = sfh;
  p0.out = nullptr;
  p0.stream_k = L.split0 ? 1 : 0;
  p0.part = reinterpret_cast<float*>(ws + L.part);
  p0.tickets = tickets;
  MxGemmParams p1 = p0;
  p1.K = f;
  p1.n_feat = d;
  p1.n_feat_tiles = d / 256;
  p1.a1_row = 128;
  p1.w_rows = d;
  p1.sfw = sf_down;
  p1.sft = sfh;
  p1.hq = nullptr;
  p1.hs = nullptr;
  p1.out = y;
  p1.stream_k = L.split1 ? 1 : 0;
  // stream-K launches one CTA per SM (at most kMxSplitCtas, the partial slots'
  // count); whole-tile scheduling launches min(tiles, SMs) persistent CTAs
  const int split_grid = sms < kMxSplitCtas ? sms : kMxSplitCtas;
  int64_t g0 = L.tiles_max * p0.n_feat_tiles, g1 = L.tiles_max * p1.n_feat_tiles;
  if (L.split0) g0 = split_grid;
  if (L.split1) g1 = split_grid;
  mx_grouped_gemm_kernel<0><<<static_cast<unsigned>(g0 < sms ? g0 : sms), kMxThreads, kMxSmemBytes, stream>>>(
      mA0, mB0, mBs0, p0);
  mx_grouped_gemm_kernel<1><<<static_cast<unsigned>(g1 < sms ? g1 : sms), kMxThreads, kMxSmemBytes, stream>>>(
      mA1, mB1, mBs1, p1);
  st = launch_unpermute(y, inv_perm, w, T, d, k, out, stream);
  if (st != MOE_OK) return st;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_router_logits(const moe_bf16_t* x, const float* W_router, const float* router_bias, int T, int d,
                               int E, float* logits, cudaStream_t stream) {
  if (!x || !W_router || !logits) return MOE_ERR_INVALID_ARG;
  if (T < 1 || d < 64 || d % 64 || d > 32768 || E < 1 || !aligned16(x)) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS || ceil_div64(T, 64) > 65535) return MOE_ERR_UNSUPPORTED;
  // the whole-chunk-walk variant of the router's logits kernel: final logits
  // (+ bias) in the canonical order, no scratch
  const dim3 grid(ceil_div(E, 64), static_cast<unsigned>(ceil_div64(T, 64)), 1);
  router_logits_kernel<64, 64, 4, 4, false><<<grid, 256, 0, stream>>>(x, W_router, router_bias, T, d, E, logits);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_qb_histogram(const float* logits, const float* bias, int T, int E, int k, float lo, float hi,
                              int bins, float* alpha, uint64_t* H, cudaStream_t stream) {
  if (!logits || !alpha || !H) return MOE_ERR_INVALID_ARG;
  if (T < 1 || E < 2 || k < 1 || k >= E || bins < 1 || !(hi > lo) || !std::isfinite(lo) || !std::isfinite(hi))
    return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK || bins > kQbMaxBins) return MOE_ERR_UNSUPPORTED;
  const float inv_w = static_cast<float>(bins) / (hi - lo);
  if (!std::isfinite(inv_w)) return MOE_ERR_INVALID_ARG;
  const unsigned cut_blocks = static_cast<unsigned>(ceil_div64(T, 8));
  if (E <= 256)
    qb_cutoffs_kernel<8><<<cut_blocks, 256, 0, stream>>>(logits, bias, T, E, k, alpha);
  else
    qb_cutoffs_kernel<32><<<cut_blocks, 256, 0, stream>>>(logits, bias, T, E, k, alpha);
  // about four waves of CTAs on a 148-SM part, each slice at least 32 tokens
  const int gx = ceil_div(E, kQbExpertsPerCta);
  int64_t slices = (4 * 148 + gx - 1) / gx;
  slices = slices < ceil_div64(T, 32) ? slices : ceil_div64(T, 32);
  if (slices < 1) slices = 1;
  const int64_t per = ceil_div64(T, slices);
  const int64_t gy = ceil_div64(T, per);
  if (gy > 65535) return MOE_ERR_UNSUPPORTED;
  qb_histogram_kernel<<<dim3(gx, static_cast<unsigned>(gy)), 256,
                        static_cast<size_t>(kQbExpertsPerCta) * bins * sizeof(uint32_t), stream>>>(
      logits, alpha, T, E, lo, inv_w, bins, static_cast<int>(per), reinterpret_cast<unsigned long long*>(H));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_qb_bias(const uint64_t* H, int E, int bins, float lo, float hi, int64_t m_total, int k,
                         int32_t* bin_out, float* bias_out, cudaStream_t stream) {
  if (!H || !bin_out || !bias_out) return MOE_ERR_INVALID_ARG;
  if (E < 2 || k < 1 || k >= E || bins < 1 || m_total < 1 || m_total > (int64_t(1) << 56) || !(hi > lo) ||
      !std::isfinite(lo) || !std::isfinite(hi))
    return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK || bins > kQbMaxBins) return MOE_ERR_UNSUPPORTED;
  int64_t r = (m_total * k + E - 1) / E;
  r = r < 1 ? 1 : (r > m_total ? m_total : r);
  const float w = (hi - lo) / static_cast<float>(bins);
  qb_bias_kernel<<<static_cast<unsigned>(ceil_div(E, 8)), 256, 0, stream>>>(
      reinterpret_cast<const unsigned long long*>(H), E, bins, lo, w, static_cast<long long>(r), bin_out, bias_out);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_gather_rows(const moe_bf16_t* src, int64_t n_src, const int32_t* rows, int64_t n_out, int d,
                             moe_bf16_t* out, cudaStream_t stream) {
  if (n_src < 0 || n_out < 0 || d < 8 || d % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (n_out == 0) return MOE_OK;
  if (!rows || !out || (n_src > 0 && !src) || !aligned16(out) || (src && !aligned16(src)))
    return MOE_ERR_INVALID_ARG;
  const int64_t blocks = ceil_div64(n_out, 8);  // 8 warps of 256 threads, warp per row
  if (blocks > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  gather_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(src), n_src, rows, n_out, d / 8, reinterpret_cast<uint4*>(out));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_get_device_error(uint32_t* code, int clear) {
  if (!code) return MOE_ERR_INVALID_ARG;
  unsigned int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, moe::g_device_error, sizeof(v)) != cudaSuccess) return MOE_ERR_CUDA;
  if (clear && v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(moe::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return MOE_ERR_CUDA;
  }
  *code = v;
  return v ? MOE_ERR_DEVICE : MOE_OK;
}

moe_status_t moe_selftest_wait_timeout(int timeout_us, cudaStream_t stream) {
  if (timeout_us < 1 || timeout_us > 1000000) return MOE_ERR_INVALID_ARG;
  moe::selftest_wait_kernel<<<1, 32, 0, stream>>>(static_cast<unsigned long long>(timeout_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"

// ----------------------------------------------------- Stable LatentMoE

namespace {

// A linear layer out = A W on the down-GEMM kernel (mode 1): n experts that
// each take `rows` consecutive rows of A [n rows, K] through their own W [n, K,
// N] into out [n rows, N] (bf16). The expert offsets and token-block prefixes
// are written on the device by launch_linear_schedule.
struct LinearPlan {
  CUtensorMap mA, mB, mBs;
  GemmParams p;
  int grid;
  int32_t* offsets;
  int32_t* prefix0;
  int rows, n;
};

moe_status_t plan_linear(const moe_bf16_t* A, const moe_bf16_t* W, moe_bf16_t* out, int rows, int n, int K, int N,
                         int32_t* offsets, int32_t* prefix0, int32_t* prefix1, int num_sms, LinearPlan* lp) {
  if (!weight_map(&lp->mA, W, n, K, N) || !act_map(&lp->mB, A, n * rows, K, kGemmBoxRows) ||
      !act_map(&lp->mBs, A, n * rows, K, kGemmSmallBox))
    return MOE_ERR_INVALID_ARG;
  GemmParams& p = lp->p;
  p = GemmParams{};
  p.expert_offsets = offsets;
  p.tile_prefix = prefix1;
  p.E = n;
  p.K = K;
  p.n_feat = N;
  p.n_feat_tiles = ceil_div(N, 2 * kGemmBMF);
  p.a1_offset = kGemmBMF;
  p.out = reinterpret_cast<uint16_t*>(out);
  p.stream_k = 0;
  p.b_fixed_row = -1;
  const int64_t tiles = static_cast<int64_t>(n) * ceil_div64(rows, 128) * p.n_feat_tiles;
  lp->grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  lp->offsets = offsets;
  lp->prefix0 = prefix0;
  lp->rows = rows;
  lp->n = n;
  return MOE_OK;
}

void launch_linear_schedule(const LinearPlan& lp, cudaStream_t stream) {
  uniform_offsets_kernel<<<1, 64, 0, stream>>>(lp.rows, lp.n, lp.offsets);
  gemm_schedule_kernel<<<1, 1024, 0, stream>>>(lp.offsets, lp.n, lp.n * lp.rows, 128, 128, lp.prefix0,
                                               const_cast<int32_t*>(lp.p.tile_prefix), nullptr, 0);
}

void launch_linear(const LinearPlan& lp, cudaStream_t stream) {
  grouped_gemm_kernel<1><<<lp.grid, kGemmThreads, GemmCfg<1>::kSmemBytes, stream>>>(lp.mA, lp.mB, lp.mBs, lp.p);
}

constexpr int kLatentMaxShared = 8;

struct LatentLayout {
  size_t route, idx, w, offsets, perm_token, inv_perm, z, z_perm, h, y_perm, n, o, perm_ws, ffn_ws, lin, x_rep, hs,
      ys, sh_offsets, ffn_ws_sh, total;
};

LatentLayout latent_layout(int T, int d, int l, int E, int k, int f, int S, int fs) {
  LatentLayout L{};
  const size_t Tk = static_cast<size_t>(T) * k;
  const size_t ST = static_cast<size_t>(S) * T;
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t here = at;
    at += align256(bytes);
    return here;
  };
  L.route = take(route_plan(T, d, E).ws_bytes);
  L.idx = take(Tk * 4);
  L.w = take(Tk * 4);
  L.offsets = take((static_cast<size_t>(E) + 1) * 4);
  L.perm_token = take(Tk * 4);
  L.inv_perm = take(Tk * 4);
  L.z = take(static_cast<size_t>(T) * l * 2);
  L.z_perm = take(Tk * l * 2);
  L.h = take(Tk * f * 2);
  L.y_perm = take(Tk * l * 2);
  L.n = take(static_cast<size_t>(T) * l * 2);
  L.o = take(static_cast<size_t>(T) * d * 2);
  L.perm_ws = take(permute_ws(T, E, k));
  L.ffn_ws = take(ffn_ws(T * k, E));
  L.lin = take(3 * align256(2 * 4));  // offsets, prefix0, prefix1 of the one-expert projections
  if (S > 0) {
    L.x_rep = take(ST * d * 2);
    L.hs = take(ST * fs * 2);
    L.ys = take(ST * d * 2);
    L.sh_offsets = take((static_cast<size_t>(S) + 1) * 4);
    L.ffn_ws_sh = take(ffn_ws(S * T, S));
  }
  L.total = at;
  return L;
}

bool latent_shape_ok(int T, int d, int l, int E, int k, int f, int S, int fs) {
  const bool dims = d >= 64 && d % 64 == 0 && d <= 32768 && l >= 64 && l % 64 == 0 && l <= 8192 && f >= 64 &&
                    f % 64 == 0 && f <= 32768 && S >= 0 && S <= kLatentMaxShared &&
                    (S == 0 || (fs >= 64 && fs % 64 == 0 && fs <= 32768));
  return dims && shape_ok(T, d, E, k) && static_cast<int64_t>(T) * (S > 0 ? S : 1) < (int64_t(1) << 31);
}

}  // namespace

extern "C" {

size_t moe_latent_workspace_size(int T, int d, int l, int E, int k, int f, int S, int fs) {
  if (!latent_shape_ok(T, d, l, E, k, f, S, fs)) return 0;
  return latent_layout(T, d, l, E, k, f, S, fs).total;
}

moe_status_t moe_latent_forward(const moe_bf16_t* x, const float* W_router, const float* router_bias,
                                const moe_bf16_t* W_dn, const moe_bf16_t* W_up, const moe_bf16_t* W_gate_up,
                                const moe_bf16_t* W_down, const float* gamma, const moe_bf16_t* Ws_gate_up,
                                const moe_bf16_t* Ws_down, int T, int d, int l, int E, int k, int f, int S, int fs,
                                int act, float beta1, float beta2, float eps, moe_bf16_t* out, void* workspace,
                                size_t workspace_bytes, cudaStream_t stream) {
  if (!x || !W_router || !W_dn || !W_up || !W_gate_up || !W_down || !out) return MOE_ERR_INVALID_ARG;
  if (S > 0 && (!Ws_gate_up || !Ws_down)) return MOE_ERR_INVALID_ARG;
  if (!latent_shape_ok(T, d, l, E, k, f, S, fs)) return MOE_ERR_INVALID_ARG;
  if (act != 0 && act != 1) return MOE_ERR_INVALID_ARG;
  if (act == 1 && !(beta1 > 0.0f && beta2 > 0.0f && std::isfinite(beta1) && std::isfinite(beta2)))
    return MOE_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return MOE_ERR_INVALID_ARG;
  for (const void* p : {static_cast<const void*>(x), static_cast<const void*>(W_dn), static_cast<const void*>(W_up),
                        static_cast<const void*>(W_gate_up), static_cast<const void*>(W_down),
                        static_cast<const void*>(out)})
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (S > 0 && (!aligned16(Ws_gate_up) || !aligned16(Ws_down))) return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK || E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  const LatentLayout L = latent_layout(T, d, l, E, k, f, S, fs);
  if (!workspace || !aligned256(workspace) || workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
  int sms = 0;
  moe_status_t st = device_setup(&sms);
  if (st != MOE_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
  float* w = reinterpret_cast<float*>(ws + L.w);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* perm_token = reinterpret_cast<int32_t*>(ws + L.perm_token);
  int32_t* inv_perm = reinterpret_cast<int32_t*>(ws + L.inv_perm);
  moe_bf16_t* z = reinterpret_cast<moe_bf16_t*>(ws + L.z);
  moe_bf16_t* z_perm = reinterpret_cast<moe_bf16_t*>(ws + L.z_perm);
  moe_bf16_t* h = reinterpret_cast<moe_bf16_t*>(ws + L.h);
  moe_bf16_t* y_perm = reinterpret_cast<moe_bf16_t*>(ws + L.y_perm);
  moe_bf16_t* nrm = reinterpret_cast<moe_bf16_t*>(ws + L.n);
  moe_bf16_t* o = reinterpret_cast<moe_bf16_t*>(ws + L.o);
  int32_t* lin_off = reinterpret_cast<int32_t*>(ws + L.lin);
  int32_t* lin_pre0 = reinterpret_cast<int32_t*>(ws + L.lin + align256(8));
  int32_t* lin_pre1 = reinterpret_cast<int32_t*>(ws + L.lin + 2 * align256(8));
  const int Tk = T * k;

  // plans (host only: tensor maps and parameters)
  LinearPlan down_proj, up_proj;
  st = plan_linear(x, W_dn, z, T, 1, d, l, lin_off, lin_pre0, lin_pre1, sms, &down_proj);
  if (st != MOE_OK) return st;
  st = plan_linear(nrm, W_up, o, T, 1, l, d, lin_off, lin_pre0, lin_pre1, sms, &up_proj);
  if (st != MOE_OK) return st;
  FfnPlan fr;
  st = plan_ffn(z_perm, offsets, W_gate_up, W_down, Tk, l, E, f, h, y_perm, ws + L.ffn_ws, sms, &fr);
  if (st != MOE_OK) return st;
  fr.act = act;
  fr.p0.beta1 = beta1;
  fr.p0.beta2 = beta2;
  FfnPlan fsh;
  moe_bf16_t* x_rep = nullptr;
  moe_bf16_t* ys = nullptr;
  if (S > 0) {
    x_rep = reinterpret_cast<moe_bf16_t*>(ws + L.x_rep);
    ys = reinterpret_cast<moe_bf16_t*>(ws + L.ys);
    st = plan_ffn(x_rep, reinterpret_cast<int32_t*>(ws + L.sh_offsets), Ws_gate_up, Ws_down, S * T, d, S, fs,
                  reinterpret_cast<moe_bf16_t*>(ws + L.hs), ys, ws + L.ffn_ws_sh, sms, &fsh);
    if (st != MOE_OK) return st;
    fsh.act = act;
    fsh.p0.beta1 = beta1;
    fsh.p0.beta2 = beta2;
  }

  // 1-3. route on x
  st = launch_route(x, W_router, router_bias, T, d, E, k, idx, w, ws + L.route, stream);
  if (st != MOE_OK) return st;
  // z = x W_dn (one-expert GEMM)
  launch_linear_schedule(down_proj, stream);
  launch_linear(down_proj, stream);
  // dispatch z rows, the routed SiTU-GLU experts on z
  if (Tk <= kSmallDispatchPairs) {
    dispatch_small_kernel<<<1, 1024, 0, stream>>>(idx, Tk, E, k, gemm_block_rows(fr.mode0), gemm_block_rows(fr.mode1),
                                                  offsets, perm_token, inv_perm,
                                                  const_cast<int32_t*>(fr.p0.tile_prefix),
                                                  const_cast<int32_t*>(fr.p1.tile_prefix), fr.ticket_buf,
                                                  fr.split_ticket_words);
    permute_copy_rows_kernel<<<static_cast<unsigned>(ceil_div64(Tk, 8)), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(z), T, perm_token, Tk, l / 8, reinterpret_cast<uint4*>(z_perm));
  } else {
    st = launch_permute(z, idx, T, l, E, k, offsets, perm_token, inv_perm, z_perm, ws + L.perm_ws, stream);
    if (st != MOE_OK) return st;
    launch_schedule(fr, stream);
  }
  launch_gemm_gate_up(fr, stream);
  launch_gemm_down(fr, stream);
  // u = sum_j p_j E_j(z), RMSNorm -> n; o = n W_up
  const int vpr_l = l / 8;
  switch (k) {
#define MOE_LATENT_RMS_CASE(K)                                                                            \
  case K:                                                                                                 \
    combine_rmsnorm_kernel<K><<<static_cast<unsigned>(T), 256, 0, stream>>>(                             \
        reinterpret_cast<const uint4*>(y_perm), inv_perm, w, gamma, eps, T, vpr_l, reinterpret_cast<uint4*>(nrm)); \
    break;
    MOE_LATENT_RMS_CASE(1) MOE_LATENT_RMS_CASE(2) MOE_LATENT_RMS_CASE(3) MOE_LATENT_RMS_CASE(4)
    MOE_LATENT_RMS_CASE(5) MOE_LATENT_RMS_CASE(6) MOE_LATENT_RMS_CASE(7) MOE_LATENT_RMS_CASE(8)
    MOE_LATENT_RMS_CASE(9) MOE_LATENT_RMS_CASE(10) MOE_LATENT_RMS_CASE(11) MOE_LATENT_RMS_CASE(12)
    MOE_LATENT_RMS_CASE(13) MOE_LATENT_RMS_CASE(14) MOE_LATENT_RMS_CASE(15) MOE_LATENT_RMS_CASE(16)
#undef MOE_LATENT_RMS_CASE
    default: return MOE_ERR_UNSUPPORTED;
  }
  launch_linear(up_proj, stream);  // same one-expert tables as the down projection
  // shared experts on x, then out = o + sum_s y_s
  const int64_t nvec = static_cast<int64_t>(T) * d / 8;
  if (S > 0) {
    repeat_rows_kernel<<<static_cast<unsigned>(ceil_div64(nvec, 256)), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(x), nvec, S, reinterpret_cast<uint4*>(x_rep));
    uniform_offsets_kernel<<<1, 64, 0, stream>>>(T, S, const_cast<int32_t*>(fsh.p0.expert_offsets));
    launch_schedule(fsh, stream);
    launch_gemm_gate_up(fsh, stream);
    launch_gemm_down(fsh, stream);
  }
  sum_rows_kernel<<<static_cast<unsigned>(ceil_div64(nvec, 256)), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(o), reinterpret_cast<const uint4*>(ys), S, nvec, reinterpret_cast<uint4*>(out));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
