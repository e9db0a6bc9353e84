// Grouped expert GEMMs in the MX serving format: MXFP4 (E2M1) expert weights
// times MXFP8 (E4M3) token rows on the block-scaled sm_100a tensor cores
// (tcgen05.mma kind::mxf8f6f4, E8M0 scales per 32 K elements), for the
// serving format of "Kimi K3: Open Frontier Intelligence", section "Systems
// Optimization, Load Balancing, and Post-Training Alignment" applied to the
// routed experts of its section "Operational Execution Flow":
//   mode 0 (gate/up): h[r, j] = SiLU(x[r] . Wgu[e][:, j]) * (x[r] . Wgu[e][:, f + j]),
//                     stored as MXFP8 along j (codes + per-tile scale atoms),
//                     the down projection's token operand;
//   mode 1 (down):    y[r, c] = h[r] . Wd[e][:, c], stored bf16.
// Operand layouts are those of mx_prep.cuh.
//
// The structure follows the bf16 kernel (expert_gemm.cuh): swap AB (weights
// are the M = 128 operand, a tile's token rows the N operand), two A operands
// and two accumulators per tile (mode 0: gate and up features j0..j0+127;
// mode 1: output features n0..n0+127 and n0+128..n0+255), persistent CTAs
// over (expert, feature block, token block) tiles, warp 0 TMA producer, warp 1
// MMA issuer, warps 2..5 epilogue, and every wait bounded.
// What changes:
//   - a stage covers 128 K elements: per A operand a 16U4 TMA box that reads
//     64 bytes of packed codes per weight row and leaves them in shared memory
//     with one byte per element (the tensor core's layout for 4-bit operands
//     next to 8-bit ones); the token box is 128 E4M3 bytes per row, 112 rows,
//     or 16 rows for tiles of at most 16 (decode steps);
//   - each stage also brings three 512-byte scale atoms (both A operands and
//     the token tile) by bulk copy; the MMA issuer moves them into TMEM with
//     tcgen05.cp before the stage's four MMAs (K = 32 each), whose scale IDs
//     pick the byte of the block;
//   - token tiles are kMxTileRows = 112 rows, so that two accumulator pairs
//     (2 x 2 x 112 columns) and the scale columns fit in the 512 TMEM columns;
//   - the gate/up epilogue quantises h to MXFP8 itself: a block is 32
//     consecutive features, which are the 32 lanes of one epilogue warp, so the
//     block maximum is one warp reduction per token column.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "expert_gemm.cuh"  // silu_f32, bf16_bits, SlotPlan
#include "mx_prep.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kMxBK = 128;        // K elements per stage
constexpr int kMxThreads = 192;
constexpr int kMxStages = 4;
constexpr int kMxABytes = 128 * kMxBK;            // 16 KB in shared memory (one byte per element)
constexpr int kMxATx = 128 * kMxBK / 2;           // 8 KB read from memory (packed)
constexpr int kMxBBytes = 128 * kMxBK;            // room for 128 token rows of 128 bytes
constexpr int kMxBTx = kMxTileRows * kMxBK;       // 112 rows are loaded
constexpr int kMxSmallRows = 16;                  // token box of tiles with <= 16 rows (decode)
constexpr int kMxBTxSmall = kMxSmallRows * kMxBK;
constexpr int kMxSfOff = 2 * kMxABytes + kMxBBytes;  // three atoms after the operands
constexpr int kMxStageBytes = kMxSfOff + 3 * kMxAtomBytes + 512;  // 50 KB (1024-aligned)
constexpr int kMxSlotCols = 2 * kMxTileRows;      // 224: two accumulators of one tile
constexpr int kMxSfCol = 2 * kMxSlotCols;         // 448: scale columns (A0, A1, B at +0, +8, +16)
constexpr int kMxTmemCols = 512;
constexpr int kMxBarrierBytes = 256;
constexpr int kMxTableBytes = 2 * (1024 + 1) * 4 + 8;
constexpr int kMxSmemBytes = kMxStages * kMxStageBytes + kMxBarrierBytes + kMxTableBytes + 1024;
static_assert(kMxStageBytes % 1024 == 0, "stages stay 1024-byte aligned");
static_assert(kMxSmemBytes <= 232448, "shared memory per CTA");
static_assert(kMxSfCol + 20 <= kMxTmemCols, "TMEM columns");

struct MxGemmParams {
  const int32_t* expert_offsets;  // [E + 1]
  const int32_t* tile_prefix;     // [E + 1] token tiles (kMxTileRows rows) before expert e
  int E;
  int K;             // d (mode 0) or f (mode 1); multiple of 128
  int n_feat;        // f (mode 0) or d (mode 1)
  int n_feat_tiles;  // mode 0: f / 128; mode 1: d / 256
  int a1_row;        // weight row of the second A operand minus the first: f (mode 0) or 128 (mode 1)
  int w_rows;        // rows of one expert's packed weight: 2f (mode 0) or d (mode 1)
  const uint8_t* sfw;  // weight scale atoms [E][w_rows / 128][K / 128][512]
  const uint8_t* sft;  // token scale atoms [tiles][K / 128][512]
  uint8_t* hq;         // mode 0: h codes [Tk][f]
  uint8_t* hs;         // mode 0: h scale atoms [tiles][f / 128][512]
  uint16_t* out;       // mode 1: y [Tk][d] bf16
  // Stream-K, as in the bf16 kernel: with few output tiles the (tile, K
  // chunk) units are split evenly over the CTAs; a CTA's first and last items
  // may cover part of a tile's K range and leave fp32 partials in part[slot]
  // (slot 2c for CTA c's first item, 2c + 1 for its last); per (tile, epilogue
  // warp) the last contributor (a ticket) adds them in CTA order, which is K
  // order, and finishes the tile. tickets[] start at zero and are put back.
  int stream_k;
  float* part;            // [2 * gridDim.x][2][kMxTileRows][128] fp32
  unsigned int* tickets;  // [tiles][4]
};

constexpr int kMxPartFloats = 2 * kMxTileRows * 128;

struct MxTile {
  int e, nb, row0, nrows, nblocks, tile;  // tile: global token-tile index (prefix[e] + block)
  int t, kb0, kb1;                        // output tile index, K-chunk range [kb0, kb1) of this item
  bool partial;                           // the item covers only part of the tile's K range
  int slot;                               // partial slot of this CTA's item
};

__device__ __forceinline__ bool mx_tile(const MxGemmParams& p, const int32_t* pre, const int32_t* off, int t,
                                        MxTile& ti) {
  const int NB = p.n_feat_tiles;
  if (t >= pre[p.E] * NB) return false;
  int lo = 0, hi = p.E - 1;  // the largest e with pre[e] * NB <= t
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
  ti.row0 = off[e] + tb * kMxTileRows;
  ti.nrows = min(kMxTileRows, off[e + 1] - ti.row0);
  ti.tile = pre[e] + tb;
  return true;
}

__device__ __forceinline__ int mx_stream_k_per(int ntiles, int KC) {
  return (ntiles * KC + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
}

// The it-th work item of this CTA: whole tiles blockIdx.x + it * gridDim.x, or
// with stream-K the tiles its unit range touches, with their K chunks inside it.
__device__ __forceinline__ bool mx_work_item(const MxGemmParams& p, const int32_t* pre, const int32_t* off, int it,
                                             MxTile& ti) {
  const int KC = p.K / kMxBK;
  if (!p.stream_k) {
    const int t = static_cast<int>(blockIdx.x) + it * static_cast<int>(gridDim.x);
    if (!mx_tile(p, pre, off, t, ti)) return false;
    ti.t = t;
    ti.kb0 = 0;
    ti.kb1 = KC;
    ti.partial = false;
    ti.slot = -1;
    return true;
  }
  const int ntiles = pre[p.E] * p.n_feat_tiles;
  const int per = mx_stream_k_per(ntiles, KC);
  const int u0 = static_cast<int>(blockIdx.x) * per;
  const int u1 = min(ntiles * KC, u0 + per);
  const int t = u0 / KC + it;
  if (u0 >= u1 || t * KC >= u1) return false;
  mx_tile(p, pre, off, t, ti);
  ti.t = t;
  ti.kb0 = max(u0, t * KC) - t * KC;
  ti.kb1 = min(u1, (t + 1) * KC) - t * KC;
  ti.partial = ti.kb0 > 0 || ti.kb1 < KC;
  ti.slot = 2 * static_cast<int>(blockIdx.x) + (it == 0 ? 0 : 1);
  return true;
}

// Finishes token row i (0-based in the tile) from this lane's two fp32 sums:
// mode 0 h = SiLU(g) * u, quantised to MXFP8 over the warp's 32 features (one
// block), codes to hq and the scale into the tile's atom; mode 1 the two bf16
// outputs. Warp-uniform: every lane of the warp calls it for the same i.
template <int kMode>
__device__ __forceinline__ void mx_finish_row(const MxGemmParams& p, const MxTile& ti, int q, int lane, int i, float g,
                                              float u) {
  if (kMode == 0) {
    const int feat = ti.nb * 128 + q * 32 + lane;
    const float h = silu_f32(g) * u;
    const uint32_t amax = __reduce_max_sync(0xffffffffu, __float_as_uint(h) & 0x7fffffffu);
    const int sc = mx_scale_exponent(__uint_as_float(amax), 8);
    const uint32_t code = mx_e4m3_code(h, mx_inverse_scale(sc));
    p.hq[static_cast<int64_t>(ti.row0 + i) * p.n_feat + feat] = static_cast<uint8_t>(code);
    if (lane == 0)
      p.hs[(static_cast<int64_t>(ti.tile) * (p.n_feat / 128) + ti.nb) * kMxAtomBytes + mx_atom_offset(i, q)] =
          static_cast<uint8_t>(sc + 127);
  } else {
    const int fa = ti.nb * 256 + q * 32 + lane;
    uint16_t* orow = p.out + static_cast<int64_t>(ti.row0 + i) * p.n_feat;
    orow[fa] = bf16_bits(g);
    orow[fa + 128] = bf16_bits(u);
  }
}

// Columns c0 .. c0 + 31 of both accumulators of a tile (only c0 .. c0 + 15 for
// the last chunk of a 112-column accumulator, so no read reaches past it).
__device__ __forceinline__ void mx_ld_chunk(uint32_t t0, uint32_t t1, int c0, uint32_t (&g)[32], uint32_t (&u)[32]) {
  if (c0 + 32 <= kMxTileRows) {
    tmem_ld_32x32b_x32(t0 + static_cast<uint32_t>(c0), g);
    tmem_ld_32x32b_x32(t1 + static_cast<uint32_t>(c0), u);
  } else {
    tmem_ld_32x32b_x16(t0 + static_cast<uint32_t>(c0), g);
    tmem_ld_32x32b_x16(t1 + static_cast<uint32_t>(c0), u);
  }
  tmem_ld_wait();
}

template <int kMode>
__global__ void __launch_bounds__(kMxThreads, 1)
    mx_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmBs, const MxGemmParams p) {
  constexpr int S = kMxStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + S * kMxStageBytes);
  uint64_t* empty_bar = full_bar + S;
  uint64_t* acc_full_bar = empty_bar + S;      // [2] one per TMEM slot
  uint64_t* acc_empty_bar = acc_full_bar + 2;  // [2]
  uint64_t* drain_bar = acc_empty_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem + S * kMxStageBytes + kMxBarrierBytes);
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
      mbar_init(&acc_empty_bar[b], 4);
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
    tmem_alloc(tmem_slot, kMxTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int KC = p.K / kMxBK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w_once = l2_policy_evict_first();
      const uint64_t pol_w_shared = l2_policy_evict_normal();
      const uint64_t pol_x = l2_policy_evict_last();
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      bool ok = true;
      MxTile ti;
      for (int it = 0; ok && mx_work_item(p, s_pre, s_off, it, ti); ++it) {
        const int ra0 = ti.nb * (kMode == 0 ? 128 : 256);
        const int ra1 = ra0 + p.a1_row;
        const uint64_t pol_w = (ti.nblocks == 1) ? pol_w_once : pol_w_shared;
        const int64_t wtiles = static_cast<int64_t>(ti.e) * (p.w_rows / 128);
        const uint8_t* sfa0 = p.sfw + (wtiles + ra0 / 128) * KC * kMxAtomBytes;
        const uint8_t* sfa1 = p.sfw + (wtiles + ra1 / 128) * KC * kMxAtomBytes;
        const uint8_t* sfb = p.sft + static_cast<int64_t>(ti.tile) * KC * kMxAtomBytes;
        // a tile of at most 16 rows loads a 16-row token box (its MMAs have N = 16)
        const bool small = ti.nrows <= kMxSmallRows;
        const CUtensorMap* mb = small ? &tmBs : &tmB;
        const uint32_t tx = 2 * kMxATx + (small ? kMxBTxSmall : kMxBTx) + 3 * kMxAtomBytes;
        for (int kc = ti.kb0; kc < ti.kb1; ++kc) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, kWaitLimitNs, abort_flag)) {
            record_device_error(1u /* MOE_DEVERR_WAIT_TIMEOUT_PRODUCER */);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kMxStageBytes;
          mbar_arrive_expect_tx(&full_bar[s], tx);
          const int k0 = kc * kMxBK;
          tma_load_3d(st, &tmA, &full_bar[s], k0, ra0, ti.e, pol_w);
          tma_load_3d(st + kMxABytes, &tmA, &full_bar[s], k0, ra1, ti.e, pol_w);
          tma_load_2d(st + 2 * kMxABytes, mb, &full_bar[s], k0, ti.row0, pol_x);
          uint8_t* sf = st + kMxSfOff;
          bulk_load(sf, sfa0 + static_cast<int64_t>(kc) * kMxAtomBytes, kMxAtomBytes, &full_bar[s], pol_w);
          bulk_load(sf + kMxAtomBytes, sfa1 + static_cast<int64_t>(kc) * kMxAtomBytes, kMxAtomBytes, &full_bar[s],
                    pol_w);
          bulk_load(sf + 2 * kMxAtomBytes, sfb + static_cast<int64_t>(kc) * kMxAtomBytes, kMxAtomBytes,
                    &full_bar[s], pol_x);
          ++issued;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
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
      uint32_t uses[2] = {0u, 0u};
      int next_slot = 0;
      bool ok = true;
      bool any = false;
      const uint32_t t_sfa0 = tmem_base + kMxSfCol, t_sfa1 = t_sfa0 + 8u, t_sfb = t_sfa0 + 16u;
      MxTile ti;
      for (int it = 0; ok && mx_work_item(p, s_pre, s_off, it, ti); ++it) {
        const uint32_t n_mma = static_cast<uint32_t>(max(16, (ti.nrows + 15) & ~15));
        const int sl = next_slot;
        next_slot ^= 1;
        if (!mbar_wait_bounded(&acc_empty_bar[sl], (uses[sl] & 1u) ^ 1u, kWaitLimitNs, abort_flag)) {
          record_device_error(2u /* MOE_DEVERR_WAIT_TIMEOUT_MMA */);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(sl * kMxSlotCols);
        const uint32_t d1 = d0 + static_cast<uint32_t>(kMxTileRows);
        for (int kc = ti.kb0; kc < ti.kb1; ++kc) {
          if (!mbar_wait_bounded(&full_bar[s], ph, kWaitLimitNs, abort_flag)) {
            record_device_error(2u /* MOE_DEVERR_WAIT_TIMEOUT_MMA */);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(smem + s * kMxStageBytes);
          const uint32_t b_addr = a_addr + 2 * kMxABytes;
          const uint32_t sf_addr = a_addr + kMxSfOff;
          tc_cp_32x128b_warpx4(t_sfa0, umma_smem_desc_noswizzle(sf_addr, 128, 128));
          tc_cp_32x128b_warpx4(t_sfa1, umma_smem_desc_noswizzle(sf_addr + kMxAtomBytes, 128, 128));
          tc_cp_32x128b_warpx4(t_sfb, umma_smem_desc_noswizzle(sf_addr + 2 * kMxAtomBytes, 128, 128));
#pragma unroll
          for (int kk = 0; kk < kMxBK / 32; ++kk) {
            const uint32_t idesc = umma_idesc_mx_e2m1_e4m3(128u, n_mma, static_cast<uint32_t>(kk),
                                                           static_cast<uint32_t>(kk));
            const uint32_t id = static_cast<uint32_t>(kk) << 30;  // scale byte of this K block
            const uint64_t adesc0 = umma_smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t adesc1 = umma_smem_desc_sw128(a_addr + kMxABytes + kk * 32, 16, 1024);
            const uint64_t bdesc = umma_smem_desc_sw128(b_addr + kk * 32, 16, 1024);
            const uint32_t accum = (kc > ti.kb0 || kk > 0) ? 1u : 0u;
            tc_mma_mx(d0, adesc0, bdesc, idesc, t_sfa0 | id, t_sfb | id, accum);
            tc_mma_mx(d1, adesc1, bdesc, idesc, t_sfa1 | id, t_sfb | id, accum);
          }
          tc_commit(&empty_bar[s]);
          any = true;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full_bar[sl]);
        ++uses[sl];
      }
      if (any) {
        tc_commit(drain_bar);
        mbar_wait_bounded(drain_bar, 0u, kWaitLimitNs, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    uint32_t uses[2] = {0u, 0u};
    int next_slot = 0;
    MxTile ti;
    for (int it = 0; mx_work_item(p, s_pre, s_off, it, ti); ++it) {
      const int sl = next_slot;
      next_slot ^= 1;
      if (!mbar_wait_bounded(&acc_full_bar[sl], uses[sl] & 1u, kWaitLimitNs, abort_flag)) {
        record_device_error(3u /* MOE_DEVERR_WAIT_TIMEOUT_EPILOGUE */);
        *abort_flag = 1;
        break;
      }
      tc_fence_after_sync();
      const uint32_t t0 = tmem_base + lane_base + static_cast<uint32_t>(sl * kMxSlotCols);
      const uint32_t t1 = t0 + static_cast<uint32_t>(kMxTileRows);
      if (ti.partial) {
        // stream-K partial item: fp32 accumulators to part[slot]; the TMEM
        // slot is free as soon as they are read
        const int fl = q * 32 + lane;
        float* mine = p.part + static_cast<int64_t>(ti.slot) * kMxPartFloats;
        for (int c0 = 0; c0 < ti.nrows; c0 += 32) {
          uint32_t g[32], u[32];
          mx_ld_chunk(t0, t1, c0, g, u);
          const int nv = min(32, ti.nrows - c0);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (i < nv) {
              __stcg(mine + (c0 + i) * 128 + fl, __uint_as_float(g[i]));
              __stcg(mine + (kMxTileRows + c0 + i) * 128 + fl, __uint_as_float(u[i]));
            }
          }
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty_bar[sl]);
        ++uses[sl];
        // contributors of tile t are CTAs c_first..c_last; per (tile, warp) the
        // last to finish adds their partials in CTA order (K order)
        const int per = mx_stream_k_per(s_pre[p.E] * p.n_feat_tiles, KC);
        const int c_first = (ti.t * KC) / per, c_last = ((ti.t + 1) * KC - 1) / per;
        __threadfence();
        __syncwarp();
        unsigned int tk = 0u;
        if (lane == 0) tk = atomicAdd(&p.tickets[ti.t * 4 + q], 1u);
        tk = __shfl_sync(0xffffffffu, tk, 0);
        if (tk == static_cast<unsigned int>(c_last - c_first)) {
          __threadfence();
          for (int i = 0; i < ti.nrows; ++i) {
            float gs = 0.0f, us = 0.0f;
            for (int c = c_first; c <= c_last; ++c) {
              const int slot = 2 * c + ((ti.t == (c * per) / KC) ? 0 : 1);
              const float* src = p.part + static_cast<int64_t>(slot) * kMxPartFloats;
              const float gv = __ldcg(src + i * 128 + fl);
              const float uv = __ldcg(src + (kMxTileRows + i) * 128 + fl);
              gs = (c == c_first) ? gv : __fadd_rn(gs, gv);
              us = (c == c_first) ? uv : __fadd_rn(us, uv);
            }
            mx_finish_row<kMode>(p, ti, q, lane, i, gs, us);
          }
          if (lane == 0) p.tickets[ti.t * 4 + q] = 0u;
        }
        continue;
      }
      for (int c0 = 0; c0 < ti.nrows; c0 += 32) {
        uint32_t g[32], u[32];
        mx_ld_chunk(t0, t1, c0, g, u);
        const int nv = min(32, ti.nrows - c0);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i < nv) mx_finish_row<kMode>(p, ti, q, lane, c0 + i, __uint_as_float(g[i]), __uint_as_float(u[i]));
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty_bar[sl]);
      ++uses[sl];
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kMxTmemCols);
  }
}

}  // namespace moe
