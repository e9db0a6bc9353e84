// Grouped expert GEMMs on the sm_100a tensor cores (tcgen05 + TMEM, fed by TMA).
//
// Computes every expert's SwiGLU feed-forward on its dispatched rows (the
// routed experts E_i of "Kimi K3: Open Frontier Intelligence", section
// "Operational Execution Flow"; the page names SwiGLU as the regime its GLU
// keeps). Two launches of one kernel template:
//   mode 0 (gate/up):  H[r, j] = SiLU(X[r] . Wgu[e][:, j]) * (X[r] . Wgu[e][:, f + j])
//   mode 1 (down):     Y[r, c] = H[r] . Wd[e][:, c]
// for every row r of expert e (rows offsets[e] .. offsets[e+1]-1).
//
// Orientation ("swap AB"): the weights are the UMMA A operand (M = 128 output
// features per MMA) and the tokens are the B operand (N = the rows of one
// token block of one expert), so an expert with 1..16 rows still issues
// full-height MMAs and each weight byte is read once per token block. D = W^T X^T
// lands in TMEM with one feature per lane and one token per column.
//   A: weight tile [64 K rows x 128 features], N-contiguous in memory
//      -> MN-major operand, two 64-feature boxes, 128-byte swizzle.
//   B: token rows [N rows x 64 K], K-contiguous -> K-major, 128-byte swizzle.
// Every tile carries two A operands and two accumulators side by side in TMEM:
//   mode 0: gate features j0..j0+127 and the matching up features, so one
//           thread holds g and u of the same (feature, token): the SiLU-gate is
//           fused in the epilogue. Token blocks are 256 rows: a block with more
//           than 128 rows issues N = 256 MMAs and uses all 512 TMEM columns,
//           which halves the weight traffic of heavily loaded experts.
//   mode 1: output features n0..n0+127 and n0+128..n0+255 (256 per tile), so
//           each row of H is read once per 256 output features. Token blocks are
//           128 rows.
// TMEM holds two 256-column slots: a tile with N <= 128 uses one slot (the
// epilogue of one tile overlaps the MMAs of the next), a tile with N > 128 both.
//
// Warp roles (320 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer (one lane): smem ring of kStages stages;
//   warp 1      TMEM allocator and MMA issuer (one lane);
//   warps 2..9  epilogue: tcgen05.ld -> fp32 math -> bf16 stores. A warp may
//               read only the TMEM lane quadrant warp % 4, so each quadrant
//               (32 features) has two epilogue warps, which take alternate
//               32-token chunks of the tile: the epilogue's 2-byte stores and
//               GLU math then keep up with the MMAs of the next tile.
// Tiles are (expert, feature block, token block), enumerated from the device
// copy of the expert offsets, so there is no host synchronisation; consecutive
// tiles share a weight tile when an expert has several token blocks.
// Every barrier wait is bounded; on a timeout the kernel records an error code,
// drains what it issued and returns.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kGemmBK = 64;         // K per stage: one 128-byte swizzle row of bf16
constexpr int kGemmBMF = 128;       // output features per A operand (UMMA M)
constexpr int kGemmEpiWarps = 8;                   // two per TMEM lane quadrant
constexpr int kGemmThreads = 64 + 32 * kGemmEpiWarps;
constexpr int kGemmBoxRows = 128;   // rows of the large B box
constexpr int kGemmSmallBox = 32;   // rows of the small B box (tiles of <= 32 rows)
constexpr int kTmemSlotCols = 256;

// Modes: 0 gate/up with 256-row token blocks (3 stages of 64 KB), 2 gate/up
// with 128-row token blocks (4 stages of 48 KB: more stages in flight when no
// expert fills a 256-row block), 1 down with 128-row blocks (4 stages of
// 48 KB). Mode 0 never takes the stream-K split.
__host__ __device__ constexpr bool gemm_is_gate_up(int mode) { return mode != 1; }
__host__ __device__ constexpr int gemm_block_rows(int mode) { return mode == 0 ? 256 : 128; }

template <int kMode>
struct GemmCfg {
  static constexpr int kABytes = kGemmBK * kGemmBMF * 2;         // 16 KB per A operand
  static constexpr int kAHalf = kABytes / 2;                     // one 64-feature box (8 KB)
  static constexpr int kBRows = gemm_block_rows(kMode);          // 256 / 128
  static constexpr int kBBytes = kBRows * kGemmBK * 2;           // 32 KB (mode 0) / 16 KB
  static constexpr int kStageBytes = 2 * kABytes + kBBytes;      // 64 KB / 48 KB
  static constexpr int kStages = (kBRows == 256) ? 3 : 4;
  static constexpr int kTmemCols = 2 * kTmemSlotCols;            // 512
  static constexpr int kBarrierBytes = 256;
  static constexpr int kTableBytes = 2 * (1024 + 1) * 4 + 8;  // shared copies of tile_prefix and expert_offsets
  static constexpr int kSmemBytes = kStages * kStageBytes + kBarrierBytes + kTableBytes + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

struct GemmParams {
  const int32_t* expert_offsets;  // [E + 1] rows per expert (device)
  const int32_t* tile_prefix;     // [E + 1] token blocks before expert e (device)
  int E;
  int K;             // reduction length (d for mode 0, f for mode 1)
  int n_feat;        // output features (f for mode 0, d for mode 1)
  int n_feat_tiles;  // mode 0: ceil(f / 128); mode 1: ceil(d / 256)
  int a1_offset;     // column of the second A operand: f + j0 (mode 0) or n0 + 128 (mode 1), minus j0 / n0
  uint16_t* out;     // [Tk, n_feat] bf16
  // Stream-K (stream_k != 0; modes 1 and 2): the units (output tile t, K block
  // kb), t-major, are split evenly over the CTAs, CTA c taking units
  // [c * per, (c + 1) * per) with per = ceil(units / gridDim.x), so every SM
  // streams the same number of weight blocks however few tiles there are. A
  // CTA's share is a run of work items, each one tile's K-block range; an item
  // that covers a tile's whole K range is finished as usual, a partial item
  // writes its fp32 accumulators to part[slot] (slot 2c for the CTA's first
  // item, 2c + 1 for its last), and for each 32-feature slice the last of the
  // tile's contributors to finish (a ticket) adds the partials in ascending
  // CTA order, which is ascending K, and finishes the tile. tickets[] start at
  // zero and are put back to zero.
  int stream_k;
  int b_fixed_row;        // >= 0: every tile's token operand starts at this row (one-token steps read x itself)
  float* part;            // [slots][2][part_rows rows][128 features] fp32
  unsigned int* tickets;  // [tiles][kGemmEpiWarps]: one per epilogue warp (32 features x alternate chunks)
  float beta1, beta2;     // SiTU-GLU soft caps (gate/up kernels with kAct = 1 only)
  int part_rows = 128;    // rows of one partial's accumulators (32 when no tile has more)
};

// fp32 elements of one partial: two accumulators, 128 rows x 128 features
constexpr int kSplitPartFloats = 2 * 128 * kGemmBMF;

struct TileInfo {
  int e, nb, row0, nrows, nblocks;  // nblocks: token blocks of expert e
  int t, kb0, kb1;                  // tile index, K-block range [kb0, kb1) of this item
  bool partial;                     // the item covers only part of the tile's K range
  int slot;                         // partial slot of this CTA's item
  // chunked items (the one-launch feed-forward): the tile's partials are the
  // slots chunk_first .. chunk_first + chunk_count - 1, in K order
  int chunk_first = 0, chunk_count = 0;
};

// Tile t -> (expert, feature block, token block), from shared-memory copies of
// the tile prefix (pre[0..E]) and the expert offsets (off[0..E]).
template <int kMode>
__device__ __forceinline__ void decode_tile(const GemmParams& p, const int32_t* pre, const int32_t* off, int t,
                                            TileInfo& ti) {
  constexpr int BR = gemm_block_rows(kMode);
  const int NB = p.n_feat_tiles;
  // owner: the largest e with pre[e] * NB <= t
  int lo = 0, hi = p.E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] * NB <= t)
      lo = mid;
    else
      hi = mid - 1;
  }
  const int e = lo;
  const int tb_count = pre[e + 1] - pre[e];
  const int local = t - pre[e] * NB;
  const int tb = local % tb_count;
  ti.e = e;
  ti.nblocks = tb_count;
  ti.nb = local / tb_count;
  ti.row0 = off[e] + tb * BR;
  ti.nrows = min(BR, off[e + 1] - ti.row0);
  ti.t = t;
}

// Units of stream-K work per CTA (see GemmParams).
__device__ __forceinline__ int stream_k_per(int ntiles, int KB) {
  return (ntiles * KB + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
}

// The it-th work item of this CTA: tiles blockIdx.x, blockIdx.x + gridDim.x,
// ... with their whole K range, or, with stream-K, the tiles its unit range
// touches with the K blocks inside that range.
template <int kMode>
__device__ __forceinline__ bool work_item(const GemmParams& p, const int32_t* pre, const int32_t* off, int it,
                                          TileInfo& ti) {
  const int KB = p.K / kGemmBK;
  const int ntiles = pre[p.E] * p.n_feat_tiles;
  if (!p.stream_k) {
    const int t = static_cast<int>(blockIdx.x) + it * static_cast<int>(gridDim.x);
    if (t >= ntiles) return false;
    decode_tile<kMode>(p, pre, off, t, ti);
    ti.kb0 = 0;
    ti.kb1 = KB;
    ti.partial = false;
    ti.slot = -1;
    return true;
  }
  const int per = stream_k_per(ntiles, KB);
  const int u0 = static_cast<int>(blockIdx.x) * per;
  const int u1 = min(ntiles * KB, u0 + per);
  const int t = u0 / KB + it;
  if (u0 >= u1 || t * KB >= u1) return false;
  decode_tile<kMode>(p, pre, off, t, ti);
  ti.kb0 = max(u0, t * KB) - t * KB;
  ti.kb1 = min(u1, (t + 1) * KB) - t * KB;
  ti.partial = ti.kb0 > 0 || ti.kb1 < KB;
  ti.slot = 2 * static_cast<int>(blockIdx.x) + (it == 0 ? 0 : 1);
  return true;
}

// TMEM slot use of one tile: a tile with more than 128 rows takes both slots.
struct SlotPlan {
  int first, count;
};
__device__ __forceinline__ SlotPlan slot_plan(int nrows, int& next_slot) {
  SlotPlan sp;
  if (nrows > 128) {
    sp.first = 0;
    sp.count = 2;
    next_slot = 0;
  } else {
    sp.first = next_slot;
    sp.count = 1;
    next_slot ^= 1;
  }
  return sp;
}

__device__ __forceinline__ float silu_f32(float a) { return a / (1.0f + expf(-a)); }

// The gate/up epilogue's GLU: kAct 0 SwiGLU, SiLU(g) * u; kAct 1 SiTU-GLU
// (the soft-capped GLU of "Kimi K3: Open Frontier Intelligence", section
// "Operational Execution Flow"; its formula is lost on the page, the reading
// taken is beta1 tanh(SiLU(g) / beta1) * beta2 tanh(u / beta2), bounded by
// beta1 beta2).
template <int kAct>
__device__ __forceinline__ float glu_f32(float g, float u, const GemmParams& p) {
  if (kAct == 0) return silu_f32(g) * u;
  return p.beta1 * tanhf(silu_f32(g) / p.beta1) * (p.beta2 * tanhf(u / p.beta2));
}

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  const __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<const uint16_t*>(&b);
}

// ------------------------------------------------------- pipeline pieces
// One K block of a work item: both A operands (four 64-feature boxes), then the
// token rows (one small box, or one to two 128-row boxes), into stage `st`,
// completing on `bar`.

template <int kMode>
__device__ __forceinline__ uint32_t gemm_b_bytes(const TileInfo& ti) {
  if (ti.nrows <= kGemmSmallBox) return kGemmSmallBox * kGemmBK * 2;
  return static_cast<uint32_t>((ti.nrows + kGemmBoxRows - 1) / kGemmBoxRows) * kGemmBoxRows * kGemmBK * 2;
}

template <int kMode>
__device__ __forceinline__ void gemm_load_a(uint8_t* st, const CUtensorMap* tmA, uint64_t* bar, const GemmParams& p,
                                            const TileInfo& ti, int k0, uint64_t pol_w) {
  using Cfg = GemmCfg<kMode>;
  const int f0 = ti.nb * (gemm_is_gate_up(kMode) ? kGemmBMF : 2 * kGemmBMF);
  const int f1 = f0 + p.a1_offset;
  tma_load_3d(st, tmA, bar, f0, k0, ti.e, pol_w);
  tma_load_3d(st + Cfg::kAHalf, tmA, bar, f0 + 64, k0, ti.e, pol_w);
  tma_load_3d(st + Cfg::kABytes, tmA, bar, f1, k0, ti.e, pol_w);
  tma_load_3d(st + Cfg::kABytes + Cfg::kAHalf, tmA, bar, f1 + 64, k0, ti.e, pol_w);
}

template <int kMode>
__device__ __forceinline__ void gemm_load_b(uint8_t* st, const CUtensorMap* tmB, const CUtensorMap* tmBs,
                                            uint64_t* bar, const GemmParams& p, int row0, int nrows, int k0,
                                            uint64_t pol_x) {
  using Cfg = GemmCfg<kMode>;
  uint8_t* bdst = st + 2 * Cfg::kABytes;
  if (nrows <= kGemmSmallBox) {
    tma_load_2d(bdst, tmBs, bar, k0, p.b_fixed_row >= 0 ? p.b_fixed_row : row0, pol_x);
  } else {
    const int nbox = (nrows + kGemmBoxRows - 1) / kGemmBoxRows;
    for (int b = 0; b < nbox; ++b)
      tma_load_2d(bdst + b * kGemmBoxRows * kGemmBK * 2, tmB, bar, k0, row0 + b * kGemmBoxRows, pol_x);
  }
}

// The shared-memory ring and TMEM state of one CTA's pipeline.
struct GemmRing {
  uint8_t* smem;
  uint64_t* full_bar;
  uint64_t* empty_bar;
  uint64_t* acc_full_bar;   // [2] one per TMEM slot
  uint64_t* acc_empty_bar;  // [2]
  volatile int* abort_flag;
  uint32_t tmem_base;
};

// MMA issuer, one work item: waits for its TMEM slot(s) to be free, then for
// each K block for the stage to be full, issues the stage's MMAs (two A
// operands into two accumulators) and frees the stage; finally marks the
// accumulators complete. Returns false if a wait gave up.
template <int kMode>
__device__ __forceinline__ bool gemm_mma_item(const GemmRing& r, const TileInfo& ti, int& s, uint32_t& ph,
                                              uint32_t (&uses)[2], int& next_slot, bool& any) {
  using Cfg = GemmCfg<kMode>;
  constexpr int S = Cfg::kStages;
  const uint32_t n_mma = static_cast<uint32_t>(max(16, (ti.nrows + 15) & ~15));
  const uint32_t idesc = umma_idesc_bf16_f32(128u, n_mma, 1u, 0u);
  const SlotPlan sp = slot_plan(ti.nrows, next_slot);
  for (int j = 0; j < sp.count; ++j) {
    const int sl = sp.first + j;
    if (!mbar_wait_bounded(&r.acc_empty_bar[sl], (uses[sl] & 1u) ^ 1u, kWaitLimitNs, r.abort_flag)) {
      record_device_error(2u /* MOE_DEVERR_WAIT_TIMEOUT_MMA */);
      *r.abort_flag = 1;
      return false;
    }
  }
  tc_fence_after_sync();
  // accumulator 0 at the slot start; accumulator 1 after N columns (128 or 256)
  const uint32_t d0 = r.tmem_base + static_cast<uint32_t>(sp.first * kTmemSlotCols);
  const uint32_t d1 = d0 + (sp.count == 2 ? 256u : 128u);
  for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
    if (!mbar_wait_bounded(&r.full_bar[s], ph, kWaitLimitNs, r.abort_flag)) {
      record_device_error(2u /* MOE_DEVERR_WAIT_TIMEOUT_MMA */);
      *r.abort_flag = 1;
      return false;
    }
    tc_fence_after_sync();
    const uint32_t a_addr = smem_u32(r.smem + s * Cfg::kStageBytes);
    const uint32_t b_addr = a_addr + 2 * Cfg::kABytes;
#pragma unroll
    for (int kk = 0; kk < kGemmBK / 16; ++kk) {
      const uint64_t bdesc = umma_smem_desc_sw128(b_addr + kk * 32, 16, 1024);
      const uint64_t adesc0 = umma_smem_desc_sw128(a_addr + kk * 2048, Cfg::kAHalf, 1024);
      const uint64_t adesc1 = umma_smem_desc_sw128(a_addr + Cfg::kABytes + kk * 2048, Cfg::kAHalf, 1024);
      const uint32_t accum = (kb > ti.kb0 || kk > 0) ? 1u : 0u;
      tc_mma_bf16(d0, adesc0, bdesc, idesc, accum);
      tc_mma_bf16(d1, adesc1, bdesc, idesc, accum);
    }
    tc_commit(&r.empty_bar[s]);  // stage s is free once these MMAs have read it
    any = true;
    if (++s == S) {
      s = 0;
      ph ^= 1u;
    }
  }
  for (int j = 0; j < sp.count; ++j) {
    tc_commit(&r.acc_full_bar[sp.first + j]);  // accumulators complete
    ++uses[sp.first + j];
  }
  return true;
}

// One count per (gate/up tile, epilogue warp) once that warp's 32-feature
// slice of h is stored, published with release semantics for a CTA that will
// read h with TMA loads (the fused one-launch feed-forward below).
__device__ __forceinline__ void signal_h_slice(unsigned int* ready, int e, int lane) {
  fence_proxy_async_global();
  __threadfence();
  __syncwarp();
  if (lane == 0) atomicAdd(ready + e, 1u);
}

// Epilogue warp (q, h): TMEM lanes 32q..32q+31 (features) and the 32-token
// chunks h, h + 2, ... of the tile's columns. One work item: waits for the
// accumulators, then either stores the finished rows (mode 0/2: h =
// SiLU(g) * u; mode 1: the two 128-feature halves of y), or, for a stream-K
// partial item, writes its fp32 partials and, if it is the last of the tile's
// contributors for this warp's rows, adds them in K order and stores the
// rows. With kSignal, a finished gate/up slice is counted in ready[e].
// Returns false if a wait gave up.
constexpr int kGemmEpiHalves = kGemmEpiWarps / 4;
template <int kMode, bool kSignal, int kAct = 0>
__device__ __forceinline__ bool gemm_epilogue_item(const GemmRing& r, const GemmParams& p, const int32_t* pre,
                                                   const TileInfo& ti, int q, int h, int lane, uint32_t (&uses)[2],
                                                   int& next_slot, unsigned int* ready) {
  const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
  const SlotPlan sp = slot_plan(ti.nrows, next_slot);
  for (int j = 0; j < sp.count; ++j) {
    const int sl = sp.first + j;
    if (!mbar_wait_bounded(&r.acc_full_bar[sl], uses[sl] & 1u, kWaitLimitNs, r.abort_flag)) {
      record_device_error(3u /* MOE_DEVERR_WAIT_TIMEOUT_EPILOGUE */);
      *r.abort_flag = 1;
      return false;
    }
  }
  tc_fence_after_sync();
  const uint32_t t0 = r.tmem_base + lane_base + static_cast<uint32_t>(sp.first * kTmemSlotCols);
  const uint32_t t1 = t0 + (sp.count == 2 ? 256u : 128u);
  const int fa = ti.nb * (gemm_is_gate_up(kMode) ? kGemmBMF : 2 * kGemmBMF) + q * 32 + lane;
  const int fb = fa + kGemmBMF;  // mode 1: the second 128 output features
  const bool fa_ok = fa < p.n_feat;
  const bool fb_ok = !gemm_is_gate_up(kMode) && fb < p.n_feat;
  if (gemm_block_rows(kMode) == 128 && ti.partial) {
    // stream-K partial item: fp32 accumulators to part[slot]; the TMEM
    // slot is free as soon as it is read
    const int fl = q * 32 + lane;
    const int64_t slot_floats = 2 * static_cast<int64_t>(p.part_rows) * kGemmBMF;
    float* mine = p.part + ti.slot * slot_floats;
    for (int c0 = 32 * h; c0 < ti.nrows; c0 += 32 * kGemmEpiHalves) {
      uint32_t g[32], u[32];
      tmem_ld_32x32b_x32(t0 + static_cast<uint32_t>(c0), g);
      tmem_ld_32x32b_x32(t1 + static_cast<uint32_t>(c0), u);
      tmem_ld_wait();
      const int nv = min(32, ti.nrows - c0);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (i < nv) {
          __stcg(mine + (c0 + i) * kGemmBMF + fl, __uint_as_float(g[i]));
          __stcg(mine + (p.part_rows + c0 + i) * kGemmBMF + fl, __uint_as_float(u[i]));
        }
      }
    }
    tc_fence_before_sync();
    __syncwarp();
    for (int j = 0; j < sp.count; ++j) {
      if (lane == 0) mbar_arrive(&r.acc_empty_bar[sp.first + j]);
      ++uses[sp.first + j];
    }
    // the tile's contributors: CTAs c_first..c_last (stream-K; slot 2c for a
    // CTA's first item, 2c + 1 for its last) or, for a chunked item, chunks
    // chunk_first..; per (tile, warp), the last one to finish adds their
    // partials in that order (K order) for this warp's rows
    int c_first, c_last, per = 0;
    const int KB = p.K / kGemmBK;
    if (ti.chunk_count > 0) {
      c_first = ti.chunk_first;
      c_last = ti.chunk_first + ti.chunk_count - 1;
    } else {
      per = stream_k_per(pre[p.E] * p.n_feat_tiles, KB);
      c_first = (ti.t * KB) / per;
      c_last = ((ti.t + 1) * KB - 1) / per;
    }
    __threadfence();
    __syncwarp();
    unsigned int tk = 0u;
    const int wslot = ti.t * kGemmEpiWarps + h * 4 + q;
    if (lane == 0) tk = atomicAdd(&p.tickets[wslot], 1u);
    tk = __shfl_sync(0xffffffffu, tk, 0);
    if (tk == static_cast<unsigned int>(c_last - c_first)) {
      __threadfence();
      for (int c0 = 32 * h; c0 < ti.nrows; c0 += 32 * kGemmEpiHalves) {
        const int c1 = min(c0 + 32, ti.nrows);
        for (int i = c0; i < c1; ++i) {
          // the contributors' partials, eight loads in flight at a time, added
          // one after another in contributor order
          float gs = 0.0f, us = 0.0f;
          for (int cb = c_first; cb <= c_last; cb += 8) {
            float gv[8], uv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int c = cb + j;
              if (c <= c_last) {
                const int slot = ti.chunk_count > 0 ? c : 2 * c + ((ti.t == (c * per) / KB) ? 0 : 1);
                const float* src = p.part + slot * slot_floats;
                gv[j] = __ldcg(src + i * kGemmBMF + fl);
                uv[j] = __ldcg(src + (p.part_rows + i) * kGemmBMF + fl);
              }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int c = cb + j;
              if (c <= c_last) {
                gs = (c == c_first) ? gv[j] : __fadd_rn(gs, gv[j]);
                us = (c == c_first) ? uv[j] : __fadd_rn(us, uv[j]);
              }
            }
          }
          uint16_t* orow = p.out + static_cast<int64_t>(ti.row0 + i) * p.n_feat;
          if (gemm_is_gate_up(kMode)) {
            if (fa_ok) orow[fa] = bf16_bits(glu_f32<kAct>(gs, us, p));
          } else {
            if (fa_ok) orow[fa] = bf16_bits(gs);
            if (fb_ok) orow[fb] = bf16_bits(us);
          }
        }
      }
      if (lane == 0) p.tickets[wslot] = 0u;
      if (kSignal) signal_h_slice(ready, ti.e, lane);
    }
    return true;
  }
  for (int c0 = 32 * h; c0 < ti.nrows; c0 += 32 * kGemmEpiHalves) {
    uint32_t g[32], u[32];
    tmem_ld_32x32b_x32(t0 + static_cast<uint32_t>(c0), g);
    tmem_ld_32x32b_x32(t1 + static_cast<uint32_t>(c0), u);
    tmem_ld_wait();
    uint16_t* orow = p.out + static_cast<int64_t>(ti.row0 + c0) * p.n_feat;
    const int nv = min(32, ti.nrows - c0);
    if (gemm_is_gate_up(kMode)) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (fa_ok && i < nv)
          orow[static_cast<int64_t>(i) * p.n_feat + fa] =
              bf16_bits(glu_f32<kAct>(__uint_as_float(g[i]), __uint_as_float(u[i]), p));
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (i < nv) {
          if (fa_ok) orow[static_cast<int64_t>(i) * p.n_feat + fa] = bf16_bits(__uint_as_float(g[i]));
          if (fb_ok) orow[static_cast<int64_t>(i) * p.n_feat + fb] = bf16_bits(__uint_as_float(u[i]));
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncwarp();
  for (int j = 0; j < sp.count; ++j) {
    if (lane == 0) mbar_arrive(&r.acc_empty_bar[sp.first + j]);
    ++uses[sp.first + j];
  }
  if (kSignal) signal_h_slice(ready, ti.e, lane);
  return true;
}

template <int kMode, int kAct = 0>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmBs, const GemmParams p) {
  using Cfg = GemmCfg<kMode>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + S * Cfg::kStageBytes);
  uint64_t* empty_bar = full_bar + S;
  uint64_t* acc_full_bar = empty_bar + S;      // [2] one per TMEM slot
  uint64_t* acc_empty_bar = acc_full_bar + 2;  // [2]
  uint64_t* drain_bar = acc_empty_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem + S * Cfg::kStageBytes + Cfg::kBarrierBytes);
  int32_t* s_off = s_pre + (p.E + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
    s_pre[i] = __ldg(p.tile_prefix + i);
    s_off[i] = __ldg(p.expert_offsets + i);
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full_bar[b], 1);
      mbar_init(&acc_empty_bar[b], kGemmEpiWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmBs);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const GemmRing ring{smem, full_bar, empty_bar, acc_full_bar, acc_empty_bar, abort_flag, *tmem_slot};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // weights of an expert with one token block are read once: evict first;
      // with several blocks the neighbouring tiles re-read them: normal priority
      const uint64_t pol_w_once = l2_policy_evict_first();
      const uint64_t pol_w_shared = l2_policy_evict_normal();
      const uint64_t pol_x = l2_policy_evict_last();  // activations: re-read per feature block
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      bool ok = true;
      TileInfo ti;
      for (int it = 0; ok && work_item<kMode>(p, s_pre, s_off, it, ti); ++it) {
        const uint64_t pol_w = (ti.nblocks == 1) ? pol_w_once : pol_w_shared;
        const uint32_t tx = 2 * Cfg::kABytes + gemm_b_bytes<kMode>(ti);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, kWaitLimitNs, abort_flag)) {
            record_device_error(1u /* MOE_DEVERR_WAIT_TIMEOUT_PRODUCER */);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* st = smem + s * Cfg::kStageBytes;
          mbar_arrive_expect_tx(&full_bar[s], tx);
          const int k0 = kb * kGemmBK;
          gemm_load_a<kMode>(st, &tmA, &full_bar[s], p, ti, k0, pol_w);
          gemm_load_b<kMode>(st, &tmB, &tmBs, &full_bar[s], p, ti.row0, ti.nrows, k0, pol_x);
          ++issued;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        // drain: wait (bounded) for the loads still in flight into the ring
        for (int i = 0; i < S && i < issued; ++i) {
          s = (s == 0) ? S - 1 : s - 1;
          if (s == S - 1) ph ^= 1u;
          mbar_wait_bounded(&full_bar[s], ph, kWaitLimitNs, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t uses[2] = {0u, 0u};  // completed uses of each TMEM slot
      int next_slot = 0;
      bool any = false;
      TileInfo ti;
      for (int it = 0; work_item<kMode>(p, s_pre, s_off, it, ti); ++it)
        if (!gemm_mma_item<kMode>(ring, ti, s, ph, uses, next_slot, any)) break;
      if (any) {
        // make sure no MMA is still running before TMEM is released
        tc_commit(drain_bar);
        mbar_wait_bounded(drain_bar, 0u, kWaitLimitNs, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;         // TMEM lane quadrant this warp may access
    const int h = (warp - 2) >> 2;  // its share of the token chunks
    uint32_t uses[2] = {0u, 0u};
    int next_slot = 0;
    TileInfo ti;
    for (int it = 0; work_item<kMode>(p, s_pre, s_off, it, ti); ++it)
      if (!gemm_epilogue_item<kMode, false, kAct>(ring, p, s_pre, ti, q, h, lane, uses, next_slot, nullptr)) break;
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(ring.tmem_base, Cfg::kTmemCols);
  }
}

// ------------------------------------------- gate/up on CTA pairs
//
// The gate/up GEMM when experts average more than 128 rows (256-row token
// blocks; the skewed loads, whose heavily loaded experts make the tensor core
// the limit). A cluster of two CTAs (one TPC) shares each MMA (tcgen05
// .cta_group::2, M = 256): a pair tile is 256 gate features and the 256
// matching up features of one expert times one token block of up to 256
// rows, N = the block's rows rounded up to 16. CTA r (rank in the pair) loads
// gate and up features f0 + 128 r .. f0 + 128 r + 127 and token rows
// row0 + r N/2 .. of each 64-wide K block: 48 KB per stage per SM, 8.4 MFLOP
// of its MMA work on a full block (the single-CTA 256-row kernel loads 64 KB
// for the same work), and four stages in flight instead of three for the
// weight-streaming tiles of lightly loaded experts. Each CTA's TMEM receives
// its 128 features x N tokens of both accumulators, so each CTA's epilogue
// finishes its own features. The even CTA (rank 0) posts the stage's expected
// bytes (both CTAs' loads complete on its barrier), issues the MMAs, and
// frees the stage in both CTAs with one multicast commit; both CTAs' epilogue
// warps arrive on its accumulator-empty barrier. No load uses cluster
// multicast. Token blocks: the schedule kernel's 256-row prefix (prefix0).
constexpr int kPairStages = 4;
constexpr int kPairABytes = 128 * kGemmBK * 2;                     // one A operand half: 16 KB
constexpr int kPairBBytes = 128 * kGemmBK * 2;                     // 128 token rows: 16 KB
constexpr int kPairStageBytes = 2 * kPairABytes + kPairBBytes;     // 48 KB
constexpr int kPairSmemBytes = kPairStages * kPairStageBytes + 256 + 2 * (1024 + 1) * 4 + 8 + 1024;
static_assert(kPairSmemBytes <= 232448, "shared memory per CTA");

template <int kAct>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const GemmParams p) {
  constexpr int S = kPairStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + S * kPairStageBytes);
  uint64_t* empty_bar = full_bar + S;
  uint64_t* acc_full_bar = empty_bar + S;
  uint64_t* acc_empty_bar = acc_full_bar + 1;
  uint64_t* drain_bar = acc_empty_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem + S * kPairStageBytes + 256);
  int32_t* s_off = s_pre + (p.E + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs
  const int pair = static_cast<int>(blockIdx.x) >> 1, npairs = static_cast<int>(gridDim.x) >> 1;
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
    s_pre[i] = __ldg(p.tile_prefix + i);
    s_off[i] = __ldg(p.expert_offsets + i);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(acc_full_bar, 1);
    mbar_init(acc_empty_bar, 2 * kGemmEpiWarps);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrive or load
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int NP = p.n_feat_tiles;  // pair tiles per token block: ceil(f / 256)
  const int KB = p.K / kGemmBK;
  const int ntiles = s_pre[p.E] * NP;
  // pair tile t -> expert, 256-feature block, 256-row token block
  auto decode = [&](int t, int& e, int& np, int& row0, int& nrows) {
    int lo = 0, hi = p.E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] * NP <= t)
        lo = mid;
      else
        hi = mid - 1;
    }
    e = lo;
    const int tbc = s_pre[e + 1] - s_pre[e];
    const int local = t - s_pre[e] * NP;
    np = local / tbc;
    row0 = s_off[e] + (local % tbc) * 256;
    nrows = min(256, s_off[e + 1] - row0);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_normal();  // a heavy expert's weights serve several token blocks
      const uint64_t pol_x = l2_policy_evict_last();
      uint32_t full_lead[S];
#pragma unroll
      for (int s = 0; s < S; ++s) full_lead[s] = smem_peer_u32(&full_bar[s], 0);
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      bool ok = true;
      for (int t = pair; ok && t < ntiles; t += npairs) {
        int e, np, row0, nrows;
        decode(t, e, np, row0, nrows);
        const int f0 = np * 256 + static_cast<int>(rank) * 128;
        const int half_n = max(16, (nrows + 15) & ~15) / 2;  // token rows of each CTA's B half
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, kWaitLimitNs, abort_flag)) {
            record_device_error(1u /* MOE_DEVERR_WAIT_TIMEOUT_PRODUCER */);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kPairStageBytes;
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * kPairStageBytes);
          const int k0 = kb * kGemmBK;
          tma_load_3d_pair(st, &tmA, full_lead[s], f0, k0, e, pol_w);
          tma_load_3d_pair(st + kPairABytes / 2, &tmA, full_lead[s], f0 + 64, k0, e, pol_w);
          tma_load_3d_pair(st + kPairABytes, &tmA, full_lead[s], p.a1_offset + f0, k0, e, pol_w);
          tma_load_3d_pair(st + kPairABytes + kPairABytes / 2, &tmA, full_lead[s], p.a1_offset + f0 + 64, k0, e,
                           pol_w);
          tma_load_2d_pair(st + 2 * kPairABytes, &tmB, full_lead[s], k0, row0 + static_cast<int>(rank) * half_n,
                           pol_x);
          ++issued;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      (void)issued;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && rank == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t uses = 0;
      bool any = false, ok = true;
      for (int t = pair; ok && t < ntiles; t += npairs) {
        int e, np, row0, nrows;
        decode(t, e, np, row0, nrows);
        const uint32_t idesc = umma_idesc_bf16_f32(256u, static_cast<uint32_t>(max(16, (nrows + 15) & ~15)), 1u, 0u);
        if (!mbar_wait_bounded(acc_empty_bar, (uses & 1u) ^ 1u, kWaitLimitNs, abort_flag)) {
          record_device_error(2u /* MOE_DEVERR_WAIT_TIMEOUT_MMA */);
          *abort_flag = 1;
          break;
        }
        tc_fence_after_sync();
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&full_bar[s], ph, kWaitLimitNs, abort_flag)) {
            record_device_error(2u /* MOE_DEVERR_WAIT_TIMEOUT_MMA */);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(smem + s * kPairStageBytes);
          const uint32_t b_addr = a_addr + 2 * kPairABytes;
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk) {
            const uint64_t bdesc = umma_smem_desc_sw128(b_addr + kk * 32, 16, 1024);
            const uint64_t adesc0 = umma_smem_desc_sw128(a_addr + kk * 2048, kPairABytes / 2, 1024);
            const uint64_t adesc1 = umma_smem_desc_sw128(a_addr + kPairABytes + kk * 2048, kPairABytes / 2, 1024);
            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
            tc_mma_bf16_pair(tmem_base, adesc0, bdesc, idesc, accum);
            tc_mma_bf16_pair(tmem_base + 256u, adesc1, bdesc, idesc, accum);
          }
          tc_commit_pair_mc(&empty_bar[s], 0x3);  // stage s is free in both CTAs
          any = true;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(acc_full_bar, 0x3);  // both CTAs' accumulators complete
        ++uses;
      }
      if (any) {
        tc_commit_pair_mc(drain_bar, 0x1);
        mbar_wait_bounded(drain_bar, 0u, kWaitLimitNs, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t acc_empty_lead = smem_peer_u32(acc_empty_bar, 0);
    uint32_t uses = 0;
    for (int t = pair; t < ntiles; t += npairs) {
      int e, np, row0, nrows;
      decode(t, e, np, row0, nrows);
      if (!mbar_wait_bounded(acc_full_bar, uses & 1u, kWaitLimitNs, abort_flag)) {
        record_device_error(3u /* MOE_DEVERR_WAIT_TIMEOUT_EPILOGUE */);
        *abort_flag = 1;
        break;
      }
      tc_fence_after_sync();
      const int fa = np * 256 + static_cast<int>(rank) * 128 + q * 32 + lane;
      const bool fa_ok = fa < p.n_feat;
      const uint32_t t0 = tmem_base + lane_base;
      for (int c0 = 32 * h; c0 < nrows; c0 += 32 * kGemmEpiHalves) {
        uint32_t g[32], u[32];
        tmem_ld_32x32b_x32(t0 + static_cast<uint32_t>(c0), g);
        tmem_ld_32x32b_x32(t0 + 256u + static_cast<uint32_t>(c0), u);
        tmem_ld_wait();
        uint16_t* orow = p.out + static_cast<int64_t>(row0 + c0) * p.n_feat;
        const int nv = min(32, nrows - c0);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (fa_ok && i < nv)
            orow[static_cast<int64_t>(i) * p.n_feat + fa] =
                bf16_bits(glu_f32<kAct>(__uint_as_float(g[i]), __uint_as_float(u[i]), p));
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_lead);
      ++uses;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its pair may still use its barriers or TMEM
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// ------------------------------------------- one launch for both GEMMs
//
// For steps in which no expert has more than 32 rows (T <= 32), the gate/up
// GEMM (mode 2) and the down GEMM (mode 1) run in one persistent cooperative
// launch whose CTAs take their work from a shared queue: chunk ids are handed
// out one at a time (a CTA's own index first, then by an atomic counter), the
// gate/up chunks before the down chunks of the same expert, both in
// expert-major tile order (with 64 or more experts with rows the down chunks
// of expert i - L follow the gate/up chunks of expert i; see the claim order
// in fused_cta_run). A chunk is one tile's K-block range
// [j * ck, (j + 1) * ck); a GEMM with few tiles cuts each of them into up to
// kFusedTargetChunks / tiles chunks (about four per SM) so that every SM stays busy, one with many
// tiles hands out whole tiles. Because the queue is shared, a CTA that streams
// its weights faster simply takes more chunks: no SM waits at the end of the
// gate/up chunks for a slower one, and the experts' h tiles are finished in
// expert order, well before the down chunks that read them are handed out.
//
// A chunk's fp32 accumulators go to the partial slot of its chunk id; the
// last chunk of a tile to finish (a ticket per tile and epilogue warp) adds
// the tile's partials in chunk order, which is ascending K, and stores the
// rows. Which CTA takes which chunk depends on timing, but every sum is taken
// in the fixed order, so results are deterministic. A down chunk of expert e
// needs all of e's h rows: each epilogue warp that finishes its slice of an h
// tile counts it in h_ready[e], and the producer loads a down chunk's token
// rows (h) only once h_ready[e] reaches kGemmEpiWarps * (gate/up feature
// tiles); its weight boxes do not depend on h, so the producer issues them at
// once and keeps up to a ring of stages whose token rows are still pending.
// The producer lane claims the chunks and passes each id to the MMA lane and
// the epilogue warps through a small shared-memory queue (kFusedQueue
// entries, one mbarrier pair each). The launch is cooperative (every CTA resident), so
// a wait on another CTA always ends; it is bounded anyway, recording
// MOE_DEVERR_WAIT_TIMEOUT_DEPENDENCY. The claim counter, the tickets and
// h_ready start at zero (the dispatch step clears them).

// Partial slots per GEMM: one per chunk, of 2 x 32 rows x 128 features fp32.
// A tile is cut into at most kFusedMaxCpt chunks (the partials its last chunk
// adds).
constexpr int kFusedSlots = 2 * 148 * (128 / kGemmSmallBox);
constexpr int kFusedMaxCpt = 16;
constexpr int kFusedTargetChunks = 4 * 148;  // per GEMM: about four chunks per SM
constexpr int kFusedQueue = 16;
constexpr int kFusedBarrierBytes = 512;
constexpr int kFusedAuxBars = 12;
// The claim order's lag L (below): half the experts with rows when there are
// at least kFusedLagMin of them, else all of them (no interleaving), the
// better of the two as measured on one-token, 8-token and 32-token steps.
constexpr int kFusedLagMin = 64;
constexpr int kFusedSmemBytes = GemmCfg<1>::kStages * GemmCfg<1>::kStageBytes + kFusedBarrierBytes +
                                kFusedQueue * 4 + 3 * (1024 + 1) * 4 + 8 + 1024;
static_assert(GemmCfg<1>::kStageBytes == GemmCfg<2>::kStageBytes && GemmCfg<1>::kStages == GemmCfg<2>::kStages,
              "the fused launch runs mode 2 and mode 1 chunks in one ring");
static_assert(kFusedSmemBytes <= 232448, "shared memory per CTA");
static_assert((2 * GemmCfg<1>::kStages + 5 + 2 * kFusedQueue + kFusedAuxBars) * 8 + 8 <= kFusedBarrierBytes,
              "fused barriers");

// How one GEMM of the fused launch is cut into chunks (the same in every CTA).
struct FusedPlan {
  int KB;      // K blocks per tile
  int ck;      // K blocks per chunk
  int cpt;     // chunks per tile
  int chunks;  // tiles * cpt
};
__device__ __forceinline__ FusedPlan fused_plan(const GemmParams& p, int tiles) {
  FusedPlan f;
  f.KB = p.K / kGemmBK;
  int cpt = tiles > 0 ? kFusedTargetChunks / tiles : 1;
  cpt = max(1, min(min(cpt, kFusedMaxCpt), f.KB));
  f.ck = (f.KB + cpt - 1) / cpt;
  f.cpt = (f.KB + f.ck - 1) / f.ck;  // no empty chunk
  f.chunks = tiles * f.cpt;
  return f;
}

// Chunk c of one GEMM -> its work item.
template <int kMode>
__device__ __forceinline__ void fused_chunk(const GemmParams& p, const int32_t* pre, const int32_t* off,
                                            const FusedPlan& f, int c, TileInfo& ti) {
  const int t = c / f.cpt, j = c - (c / f.cpt) * f.cpt;
  decode_tile<kMode>(p, pre, off, t, ti);
  ti.kb0 = j * f.ck;
  ti.kb1 = min(f.KB, ti.kb0 + f.ck);
  ti.partial = f.cpt > 1;
  ti.slot = c;
  ti.chunk_first = t * f.cpt;
  ti.chunk_count = f.cpt;
}

// One CTA's state in the chunk-queue feed-forward: the stage ring, its
// mbarriers, the chunk queue and the shared tables (tile prefixes of both
// GEMMs and the expert offsets, E + 1 entries each).
struct FusedCta {
  uint8_t* smem;  // 1024-aligned: the ring (kStages stages), then the barriers and tables
  uint64_t* full_bar;
  uint64_t* empty_bar;
  uint64_t* acc_full_bar;
  uint64_t* acc_empty_bar;
  uint64_t* drain_bar;
  uint64_t* q_full;   // [Q] the producer has written entry i
  uint64_t* q_empty;  // [Q] the MMA lane and every epilogue warp have read it
  uint64_t* aux_bar;  // [kFusedAuxBars] free for the caller (the one-token router's W ring)
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  volatile int* s_chunk;
  int32_t* s_pre0;
  int32_t* s_pre1;
  int32_t* s_off;
};

__device__ __forceinline__ FusedCta fused_cta_layout(uint8_t* smem_raw, int E) {
  using Cfg = GemmCfg<1>;
  constexpr int S = Cfg::kStages;
  FusedCta c;
  c.smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  c.full_bar = reinterpret_cast<uint64_t*>(c.smem + S * Cfg::kStageBytes);
  c.empty_bar = c.full_bar + S;
  c.acc_full_bar = c.empty_bar + S;
  c.acc_empty_bar = c.acc_full_bar + 2;
  c.drain_bar = c.acc_empty_bar + 2;
  c.q_full = c.drain_bar + 1;
  c.q_empty = c.q_full + kFusedQueue;
  c.aux_bar = c.q_empty + kFusedQueue;
  c.tmem_slot = reinterpret_cast<uint32_t*>(c.aux_bar + kFusedAuxBars);
  c.abort_flag = reinterpret_cast<volatile int*>(c.tmem_slot + 1);
  c.s_chunk = reinterpret_cast<volatile int*>(c.smem + S * Cfg::kStageBytes + kFusedBarrierBytes);
  c.s_pre0 = reinterpret_cast<int32_t*>(c.smem + S * Cfg::kStageBytes + kFusedBarrierBytes + kFusedQueue * 4);
  c.s_pre1 = c.s_pre0 + (E + 1);
  c.s_off = c.s_pre1 + (E + 1);
  return c;
}

// Barrier initialisation (thread 0), tensor-map prefetch (warp 0) and the TMEM
// allocation (warp 1); the caller then fences and synchronises the CTA.
__device__ __forceinline__ void fused_cta_setup(const FusedCta& c, const CUtensorMap* tmA0, const CUtensorMap* tmBs0,
                                                const CUtensorMap* tmA1, const CUtensorMap* tmBs1) {
  using Cfg = GemmCfg<1>;
  constexpr int S = Cfg::kStages;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&c.full_bar[s], 1);
      mbar_init(&c.empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&c.acc_full_bar[b], 1);
      mbar_init(&c.acc_empty_bar[b], kGemmEpiWarps);
    }
    mbar_init(c.drain_bar, 1);
    for (int i = 0; i < kFusedQueue; ++i) {
      mbar_init(&c.q_full[i], 1);
      mbar_init(&c.q_empty[i], 1 + kGemmEpiWarps);
    }
    for (int i = 0; i < kFusedAuxBars; ++i) mbar_init(&c.aux_bar[i], 1);
    *c.abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(tmA0);
    tma_prefetch_desc(tmBs0);
    tma_prefetch_desc(tmA1);
    tma_prefetch_desc(tmBs1);
  }
  if (warp == 1) {
    tmem_alloc(c.tmem_slot, GemmCfg<1>::kTmemCols);
    tmem_relinquish();
  }
}

// The CTA's part of the feed-forward: claims chunks until the queue is empty
// (producer lane of warp 0), issues their MMAs (lane 0 of warp 1) and runs
// their epilogues (warps 2..9). The shared tables must be loaded.
__device__ __forceinline__ void fused_cta_run(const FusedCta& fc, const CUtensorMap* tmA0, const CUtensorMap* tmBs0,
                                              const CUtensorMap* tmA1, const CUtensorMap* tmBs1, const GemmParams& p0,
                                              const GemmParams& p1, unsigned int* __restrict__ h_ready,
                                              unsigned int* __restrict__ claim) {
  using Cfg = GemmCfg<1>;
  constexpr int S = Cfg::kStages;
  constexpr int Q = kFusedQueue;
  uint8_t* smem = fc.smem;
  uint64_t* full_bar = fc.full_bar;
  uint64_t* empty_bar = fc.empty_bar;
  uint64_t* drain_bar = fc.drain_bar;
  uint64_t* q_full = fc.q_full;
  uint64_t* q_empty = fc.q_empty;
  volatile int* abort_flag = fc.abort_flag;
  volatile int* s_chunk = fc.s_chunk;
  const int32_t* s_pre0 = fc.s_pre0;
  const int32_t* s_pre1 = fc.s_pre1;
  const int32_t* s_off = fc.s_off;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const GemmRing ring{smem, full_bar, empty_bar, fc.acc_full_bar, fc.acc_empty_bar, abort_flag, *fc.tmem_slot};
  const unsigned int h_target = static_cast<unsigned int>(kGemmEpiWarps * p0.n_feat_tiles);
  const FusedPlan f0 = fused_plan(p0, s_pre0[p0.E] * p0.n_feat_tiles);
  const FusedPlan f1 = fused_plan(p1, s_pre1[p0.E] * p1.n_feat_tiles);
  const int total = f0.chunks + f1.chunks;
  // Claim order. Every expert with rows has one token block in each GEMM (no
  // step of this launch gives an expert more than 32 rows), so it has G
  // gate/up and D down chunks. The gate/up chunks of the first L experts come
  // first; then, for each later expert i, its gate/up chunks followed by the
  // down chunks of expert i - L; then the down chunks of the last L experts.
  // A down chunk is thus claimed L experts' worth of work after the gate/up
  // chunks whose h rows it reads, instead of right behind the last of them.
  const int nsel = s_pre0[p0.E];
  const int G = nsel > 0 ? f0.chunks / nsel : 0;
  const int D = nsel > 0 ? f1.chunks / nsel : 0;
  const int L = nsel >= kFusedLagMin ? (nsel + 1) / 2 : nsel;
  const int seg_a = L * G, seg_b = (nsel - L) * (G + D);
  // claim id -> work item of the gate/up (true) or the down GEMM
  auto decode = [&](int c, TileInfo& ti) -> bool {
    int gate_up = 1, loc = c;
    if (c >= seg_a && c < seg_a + seg_b) {
      const int i = (c - seg_a) / (G + D), r = (c - seg_a) - i * (G + D);
      gate_up = r < G;
      loc = gate_up ? (L + i) * G + r : i * D + (r - G);
    } else if (c >= seg_a + seg_b) {
      gate_up = 0;
      loc = (nsel - L) * D + (c - seg_a - seg_b);
    }
    if (gate_up) {
      fused_chunk<2>(p0, s_pre0, s_off, f0, loc, ti);
      return true;
    }
    fused_chunk<1>(p1, s_pre1, s_off, f1, loc, ti);
    return false;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();  // every expert has one token block: weights read once
      const uint64_t pol_x = l2_policy_evict_last();
      constexpr uint32_t kTx = 2 * Cfg::kABytes + kGemmSmallBox * kGemmBK * 2;  // every tile fits the small box
      int s = 0;
      uint32_t ph = 0;
      int qi = 0;
      uint32_t qph = 0;
      int issued = 0;
      bool ok = true;
      // down stages whose weight boxes are issued and whose h rows are not yet:
      // a FIFO of (stage, K offset, first row, expert), at most S long
      int q_stage[S], q_k0[S], q_row[S], q_e[S];
      int q_head = 0, q_n = 0;
      int ready_e = -1;  // an expert whose h is known complete
      auto h_is_ready = [&](int e) -> bool {
        if (e == ready_e) return true;
        if (ld_acquire_gpu(h_ready + e) >= h_target) {
          ready_e = e;
          return true;
        }
        return false;
      };
      // issue the pending h loads in order; with `block`, wait (bounded) for
      // each one's expert. After an abort they are issued without waiting, so
      // that every stage's barrier completes and the drain below ends.
      auto flush = [&](bool block) {
        while (q_n > 0) {
          const int e = q_e[q_head];
          if (!*abort_flag && !h_is_ready(e)) {
            if (!block) return;
            const uint64_t t0 = global_timer_ns();
            while (!h_is_ready(e)) {
              if (*abort_flag) break;
              if (global_timer_ns() - t0 > kWaitLimitNs) {
                record_device_error(7u /* MOE_DEVERR_WAIT_TIMEOUT_DEPENDENCY */);
                *abort_flag = 1;
                break;
              }
            }
          }
          fence_proxy_async_global();
          const int st_i = q_stage[q_head];
          gemm_load_b<1>(smem + st_i * Cfg::kStageBytes, tmBs1, tmBs1, &full_bar[st_i], p1, q_row[q_head], 1,
                         q_k0[q_head], pol_x);
          q_head = (q_head + 1) % S;
          --q_n;
        }
      };
      // a CTA's first chunk is its own index (no atomic round trip before the
      // first loads); later ones come from the counter, from gridDim.x on
      bool first_claim = true;
      while (ok) {
        const unsigned int id = first_claim ? blockIdx.x : gridDim.x + atomicAdd(claim, 1u);
        first_claim = false;
        const int c = id < static_cast<unsigned int>(total) ? static_cast<int>(id) : -1;
        // hand the id to the MMA lane and the epilogue warps
        if (!mbar_wait_bounded(&q_empty[qi], qph ^ 1u, kWaitLimitNs, abort_flag)) {
          record_device_error(1u /* MOE_DEVERR_WAIT_TIMEOUT_PRODUCER */);
          ok = false;
          break;
        }
        s_chunk[qi] = c;
        mbar_arrive(&q_full[qi]);
        if (++qi == Q) {
          qi = 0;
          qph ^= 1u;
        }
        if (c < 0) break;
        TileInfo ti;
        const bool down = !decode(c, ti);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (q_n == S) flush(true);  // the ring holds only stages waiting for h
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, kWaitLimitNs, abort_flag)) {
            record_device_error(1u /* MOE_DEVERR_WAIT_TIMEOUT_PRODUCER */);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * Cfg::kStageBytes;
          mbar_arrive_expect_tx(&full_bar[s], kTx);
          const int k0 = kb * kGemmBK;
          if (!down) {
            gemm_load_a<2>(st, tmA0, &full_bar[s], p0, ti, k0, pol_w);
            gemm_load_b<2>(st, tmBs0, tmBs0, &full_bar[s], p0, ti.row0, 1, k0, pol_x);
          } else {
            gemm_load_a<1>(st, tmA1, &full_bar[s], p1, ti, k0, pol_w);
            const int qj = (q_head + q_n) % S;
            q_stage[qj] = s;
            q_k0[qj] = k0;
            q_row[qj] = ti.row0;
            q_e[qj] = ti.e;
            ++q_n;
            flush(false);
          }
          ++issued;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) *abort_flag = 1;
      flush(true);
      if (!ok) {
        for (int i = 0; i < S && i < issued; ++i) {
          s = (s == 0) ? S - 1 : s - 1;
          if (s == S - 1) ph ^= 1u;
          mbar_wait_bounded(&full_bar[s], ph, kWaitLimitNs, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int qi = 0;
      uint32_t qph = 0;
      uint32_t uses[2] = {0u, 0u};
      int next_slot = 0;
      bool any = false;
      while (true) {
        if (!mbar_wait_bounded(&q_full[qi], qph, kWaitLimitNs, abort_flag)) {
          if (!*abort_flag) record_device_error(2u /* MOE_DEVERR_WAIT_TIMEOUT_MMA */);
          *abort_flag = 1;
          break;
        }
        const int c = s_chunk[qi];
        mbar_arrive(&q_empty[qi]);
        if (++qi == Q) {
          qi = 0;
          qph ^= 1u;
        }
        if (c < 0) break;
        TileInfo ti;
        const bool ok = decode(c, ti) ? gemm_mma_item<2>(ring, ti, s, ph, uses, next_slot, any)
                                      : gemm_mma_item<1>(ring, ti, s, ph, uses, next_slot, any);
        if (!ok) break;
      }
      if (any) {
        tc_commit(drain_bar);
        mbar_wait_bounded(drain_bar, 0u, kWaitLimitNs, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    int qi = 0;
    uint32_t qph = 0;
    uint32_t uses[2] = {0u, 0u};
    int next_slot = 0;
    while (true) {
      if (!mbar_wait_bounded(&q_full[qi], qph, kWaitLimitNs, abort_flag)) {
        if (!*abort_flag) record_device_error(3u /* MOE_DEVERR_WAIT_TIMEOUT_EPILOGUE */);
        *abort_flag = 1;
        break;
      }
      const int c = s_chunk[qi];
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_empty[qi]);
      if (++qi == Q) {
        qi = 0;
        qph ^= 1u;
      }
      if (c < 0) break;
      TileInfo ti;
      const bool ok = decode(c, ti)
                          ? gemm_epilogue_item<2, true>(ring, p0, s_pre0, ti, q, h, lane, uses, next_slot, h_ready)
                          : gemm_epilogue_item<1, false>(ring, p1, s_pre1, ti, q, h, lane, uses, next_slot, nullptr);
      if (!ok) break;
    }
  }
}

__device__ __forceinline__ void fused_cta_teardown(const FusedCta& fc) {
  tc_fence_before_sync();
  __syncthreads();
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after_sync();
    tmem_dealloc(*fc.tmem_slot, GemmCfg<1>::kTmemCols);
  }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_ffn_fused_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmBs0,
                             const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmBs1,
                             const GemmParams p0, const GemmParams p1, unsigned int* __restrict__ h_ready,
                             unsigned int* __restrict__ claim) {
  extern __shared__ uint8_t smem_raw[];
  const FusedCta fc = fused_cta_layout(smem_raw, p0.E);
  for (int i = threadIdx.x; i <= p0.E; i += blockDim.x) {
    fc.s_pre0[i] = __ldg(p0.tile_prefix + i);
    fc.s_pre1[i] = __ldg(p1.tile_prefix + i);
    fc.s_off[i] = __ldg(p0.expert_offsets + i);
  }
  fused_cta_setup(fc, &tmA0, &tmBs0, &tmA1, &tmBs1);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  fused_cta_run(fc, &tmA0, &tmBs0, &tmA1, &tmBs1, p0, p1, h_ready, claim);
  fused_cta_teardown(fc);
}

// Token blocks per expert for both GEMMs:
//   prefix0[e] = sum_{e' < e} ceil(count_e' / rows0)  (gate/up, rows0 = 256 or 128)
//   prefix1[e] = sum_{e' < e} ceil(count_e' / rows1)  (down, rows1 = 128)
// The MOE_CHECKS build first checks the offsets (offsets[0] = 0, never
// decreasing, offsets[E] <= rows_total); on bad ones it records
// MOE_DEVERR_INDEX_CHECK and schedules no tile at all.
__global__ void __launch_bounds__(1024)
    gemm_schedule_kernel(const int32_t* __restrict__ offsets, int E, int rows_total, int rows0, int rows1,
                         int32_t* __restrict__ prefix0, int32_t* __restrict__ prefix1, unsigned int* __restrict__ zero_buf,
                         int zero_n) {
  __shared__ int32_t warp_sums[2][32];
  const int e = threadIdx.x;
  for (int i = e; i < zero_n; i += 1024) zero_buf[i] = 0u;  // K-split tickets of the gate/up GEMM
  int32_t cnt = (e < E) ? (offsets[e + 1] - offsets[e]) : 0;
  if (kIndexChecks) {
    const bool bad = (e < E && cnt < 0) || (e == 0 && offsets[0] != 0) || (e == E - 1 && offsets[E] > rows_total);
    if (__syncthreads_or(bad)) {
      if (e == 0) index_ok(false);
      cnt = 0;
    }
  }
  const int32_t nb[2] = {(cnt + rows0 - 1) / rows0, (cnt + rows1 - 1) / rows1};
  const int lane = e & 31, w = e >> 5;
  int32_t incl[2];
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    incl[m] = nb[m];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl[m], o);
      if (lane >= o) incl[m] += y;
    }
    if (lane == 31) warp_sums[m][w] = incl[m];
  }
  __syncthreads();
  if (w < 2) {
    const int m = w;
    const int32_t ws = warp_sums[m][lane];
    int32_t wincl = ws;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, wincl, o);
      if (lane >= o) wincl += y;
    }
    warp_sums[m][lane] = wincl - ws;
  }
  __syncthreads();
  if (e < E) {
    int32_t* outs[2] = {prefix0, prefix1};
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int32_t excl = warp_sums[m][w] + incl[m] - nb[m];
      outs[m][e] = excl;
      if (e == E - 1) outs[m][E] = excl + nb[m];
    }
  }
}

// A wait that nothing will ever satisfy, bounded by `limit_ns`: checks that
// bounded waits end and report instead of hanging.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait_bounded(&bar, 0u, limit_ns, nullptr)) record_device_error(4u /* MOE_DEVERR_SELFTEST_TIMEOUT */);
  }
}

}  // namespace moe
