// tc_swap.cuh -- the expert GEMMs in weight-row ("swap-AB") form, for groups
// with few rows (decode, and FP8 batches of a few thousand tokens over 512
// experts, where an expert sees tens of rows).
//
// The row-tiled kernel of tc_gemm.cuh would spend a 128-row activation tile on
// a group of ~2..64 rows.  Here the weights are the MMA's M = 128 operand and
// a chunk of kNCH token rows of the group is its N operand:
//     D[n, j] = sum_c W_g[n, c] * X[r0 + j, c],  n in a 128-row weight tile,
// so almost all shared memory holds weight bytes in flight and the tensor
// core does no work on absent rows.  Tiles are (group, 128 weight rows,
// kNCH-row token chunk); the chunks of one weight tile are adjacent in the
// list, so a large group (the shared expert) re-reads that tile from L2.
//
// Warp roles: warp 0 TMA producer; warp 1 TMEM owner + MMA issuer (dual:
// gate and up accumulators side by side, two MMAs sharing the token tile);
// warps 2..9 epilogue, one thread per weight row (output feature) walking the
// token columns.  E4M3 weights take the kernel of tc_swap8.cuh, which shares
// the tile list and the epilogue defined here.
#pragma once
#include "tc_gemm.cuh"

namespace moe {

constexpr int kNCH = 64;  // token rows per tile: the MMA's N

template <bool DUAL>
struct SwapCfg {
  static constexpr int NB = DUAL ? 256 : 128;  // weight rows per stage (gate then up, or one tile)
  static constexpr int W_BYTES = NB * 128;      // bf16 weight rows of 128 bytes
  static constexpr int X_BYTES = kNCH * 128;    // token rows of 128 bytes
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
  static constexpr int STAGES = DUAL ? 5 : 8;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr int EPI_WARPS = 8;  // two warps per TMEM lane quarter, one per token half
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int ACC_COLS = (DUAL ? 2 : 1) * kNCH;
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  static constexpr int BAR_BYTES = (2 * STAGES + 5) * 8 + 16;
  static constexpr int SCHED_INTS = 2 * (512 + 2);
  static constexpr int SMEM_BYTES = 1024 + RING_BYTES + BAR_BYTES + SCHED_INTS * 4;
  static_assert(TMEM_COLS == 128 || TMEM_COLS == 256, "TMEM columns");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

struct SwapTile {
  int g, rows, c0, n0, kblocks, N;
  int64_t row0;
};

// TILE_ROWS: weight rows per tile (128; 256 for the E4M3 down GEMM, whose
// tile is two 128-row halves sharing the token chunk).
template <int TILE_ROWS = 128>
__device__ __forceinline__ SwapTile decode_swap(const TcGemmArgs& p, const int32_t* s_pre, const int32_t* s_offs,
                                                int tile) {
  SwapTile t;
  int lo = 0, hi = p.E + 1;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_pre[mid] <= tile) lo = mid; else hi = mid;
  }
  t.g = lo;
  const int r0 = s_offs[t.g];
  t.rows = s_offs[t.g + 1] - r0;
  const int chc = (t.rows + kNCH - 1) / kNCH;
  const int local = tile - s_pre[t.g];
  t.c0 = (local % chc) * kNCH;
  t.n0 = (local / chc) * TILE_ROWS;
  t.row0 = (int64_t)r0 + t.c0;
  const bool sh = t.g == p.E;
  t.N = sh ? p.N_s : p.N_r;
  t.kblocks = ((sh ? p.K_s : p.K_r) + kBK - 1) / kBK;
  return t;
}

// Epilogue of a weight-row GEMM, run by EPI_WARPS warps numbered from 2: one
// thread per weight row (= TMEM lane, output feature), walking the kNCH token
// columns of each finished tile; with 8 warps two warps share a lane quarter
// and take one 32-token half each.
// DUAL with SwiGLU: gate and up accumulators of one 128-row weight tile;
// DUAL with SlotStore / Store: the accumulators of the two 128-row halves of a
// 256-row weight tile (output features n0 .. n0 + 255).
template <bool DUAL, int EPI, int EPI_WARPS, int ACC_BUFS = 2>
__device__ __forceinline__ void swap_epilogue(const TcGemmArgs& p, const int32_t* s_pre, const int32_t* s_offs,
                                              int total, uint32_t tmem_base, uint64_t* tfull, uint64_t* tempty,
                                              volatile int* abort_flag, unsigned tcode, int warp, int lane) {
  constexpr int ACC_COLS = (DUAL ? 2 : 1) * kNCH;
  constexpr bool HALVES = DUAL && EPI != kTcSwiGLU;
  constexpr int TILE_ROWS = HALVES ? 256 : 128;
  constexpr int EG = EPI_WARPS / 4;
  const int eg = (warp - 2) / 4;  // with 8 warps: which 32-token half this warp writes
  const int q = warp & 3;
  const int nl = q * 32 + lane;  // weight row within the tile = TMEM lane
  int acc = 0;
  uint32_t acc_phase = 0;
  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    const SwapTile t = decode_swap<TILE_ROWS>(p, s_pre, s_offs, tile);
    // per-column data of the chunk: lane j holds token columns j and j + 32
    int64_t dst_lo = -1, dst_hi = -1;
    float w_lo = 0.f, w_hi = 0.f;
    if (EPI == kTcSlotStore) {
      const int64_t ra = t.row0 + lane, rb = t.row0 + 32 + lane;
      if (t.c0 + lane < t.rows && ra < p.rows_cap) {
        dst_lo = __ldg(p.row_dst + ra);
        w_lo = __ldg(p.row_w + ra);
        if (dst_lo >= 0 && !in_range(dst_lo, p.ys_rows, p.status, kSiteSlotRow)) dst_lo = -1;
      }
      if (t.c0 + 32 + lane < t.rows && rb < p.rows_cap) {
        dst_hi = __ldg(p.row_dst + rb);
        w_hi = __ldg(p.row_w + rb);
        if (dst_hi >= 0 && !in_range(dst_hi, p.ys_rows, p.status, kSiteSlotRow)) dst_hi = -1;
      }
    }
    if (!__all_sync(0xffffffffu, mbar_wait(tfull + acc, acc_phase, abort_flag, p.status, tcode | 4)))
      break;  // the warp stops as one: its TMEM loads are warp-collective
    tc_fence_after();
    const int jmax = min(kNCH, t.rows - t.c0);
#pragma unroll 1
    for (int m = 0; m < (HALVES ? 2 : 1); ++m)
#pragma unroll 1
    for (int half = eg; half < 2 && half * 32 < jmax; half += EG) {  // (jmax is uniform per tile)
      const uint32_t tb = tmem_base + acc * ACC_COLS + ((uint32_t)(q * 32) << 16) + m * kNCH;
      const int n = t.n0 + m * 128 + nl;
      const bool nvalid = n < t.N;
      uint32_t a[32], b[32];
      tmem_ld32(tb + half * 32, a);
      if (DUAL && !HALVES) tmem_ld32(tb + kNCH + half * 32, b);
      tmem_wait_regs(a);
      if (DUAL && !HALVES) tmem_wait_regs(b);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int jj = half * 32 + j;
        const int64_t row = t.row0 + jj;
        if (EPI == kTcSwiGLU) {
          if (nvalid && jj < jmax && row < p.rows_cap)
            p.H[row * p.ldh + n] = __float2bfloat16_rn(silu_f32(__uint_as_float(a[j])) * __uint_as_float(b[j]));
        } else if (EPI == kTcSlotStore) {
          const int64_t dr = __shfl_sync(0xffffffffu, half ? dst_hi : dst_lo, j);
          const float w = __shfl_sync(0xffffffffu, half ? w_hi : w_lo, j);
          if (nvalid && jj < jmax && dr >= 0) p.ys[dr * p.ldy + n] = __float2bfloat16_rn(w * __uint_as_float(a[j]));
        } else {
          if (nvalid && jj < jmax && row < p.rows_cap) p.out[row * p.ldo + n] = __float2bfloat16_rn(__uint_as_float(a[j]));
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(tempty + acc);
    if (++acc == ACC_BUFS) {
      acc = 0;
      acc_phase ^= 1;
    }
  }
}

// tmW*: weight maps (box 64 x 128 rows; gate / the single operand = B, up = C);
// tmX*: token-row maps (box 64 x kNCH); _r routed groups, _s the shared group.
template <bool DUAL, int EPI>
__global__ void __launch_bounds__(SwapCfg<DUAL>::THREADS, 1)
    k_gemm_swap(const __grid_constant__ CUtensorMap tmX_r, const __grid_constant__ CUtensorMap tmX_s,
                const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
                const __grid_constant__ CUtensorMap tmC_r, const __grid_constant__ CUtensorMap tmC_s, TcGemmArgs p) {
  using Cfg = SwapCfg<DUAL>;
  constexpr int S = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::RING_BYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem + Cfg::RING_BYTES + Cfg::BAR_BYTES);
  int32_t* s_offs = s_pre + 514;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned tcode = kStatusTimeoutBase | (kKernGemmSwap << 8);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, Cfg::EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX_r);
    prefetch_tmap(&tmX_s);
    prefetch_tmap(&tmB_r);
    prefetch_tmap(&tmB_s);
    if (DUAL) {
      prefetch_tmap(&tmC_r);
      prefetch_tmap(&tmC_s);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  // the tile schedule comes from earlier kernels in the stream: read it once
  // they are done (barrier set-up, tensor-map prefetch and TMEM allocation above
  // overlap the previous kernel's tail under programmatic launch)
  pdl_begin();
  for (int i = threadIdx.x; i < p.E + 2; i += blockDim.x) {
    s_pre[i] = __ldg(p.prefix + i);
    s_offs[i] = __ldg(p.offs + i);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_pre[p.E + 1];

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const SwapTile t = decode_swap(p, s_pre, s_offs, tile);
        const bool sh = t.g == p.E;
        for (int kb = 0; kb < t.kblocks; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1, abort_flag, p.status, tcode | 1)) {
            ok = false;
            break;
          }
          uint64_t* land = full + stage;
          uint8_t* base = smem + stage * Cfg::STAGE_BYTES;
          uint8_t* xdst = base + Cfg::W_BYTES;
          mbar_arrive_expect_tx(land, Cfg::STAGE_BYTES);
          if (sh) tma_load_2d(base, &tmB_s, land, kb * kBK, t.n0, pol_w);
          else tma_load_3d(base, &tmB_r, land, kb * kBK, t.n0, t.g, pol_w);
          if (DUAL) {
            if (sh) tma_load_2d(base + 128 * 128, &tmC_s, land, kb * kBK, t.n0, pol_w);
            else tma_load_3d(base + 128 * 128, &tmC_r, land, kb * kBK, t.n0, t.g, pol_w);
          }
          tma_load_2d(xdst, sh ? &tmX_s : &tmX_r, land, kb * kBK, (int)t.row0, pol_x);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag)
        for (int s = 0; s < S; ++s)
          if (issued >> s & 1u) drain_wait(full + s, last_par >> s & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const SwapTile t = decode_swap(p, s_pre, s_offs, tile);
        // MMA N = the chunk's token rows rounded up to 16: columns past them are
        // neither computed nor read back
        const uint32_t idesc = idesc_bf16(kBM, min(kNCH, (t.rows - t.c0 + 15) & ~15));
        if (!mbar_wait(tempty + acc, acc_phase ^ 1, abort_flag, p.status, tcode | 2)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * Cfg::ACC_COLS;
        for (int kb = 0; kb < t.kblocks; ++kb) {
          if (!mbar_wait(full + stage, phase, abort_flag, p.status, tcode | 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sw = smem_u32(smem + stage * Cfg::STAGE_BYTES);
          const uint32_t sx = sw + Cfg::W_BYTES;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bd = sdesc_sw128(sx + kk * 32);
            const uint32_t accum = (kb | kk) != 0;
            umma_f16(d0, sdesc_sw128(sw + kk * 32), bd, idesc, accum);
            if (DUAL) umma_f16(d0 + kNCH, sdesc_sw128(sw + 128 * 128 + kk * 32), bd, idesc, accum);
          }
          umma_commit(empty + stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(tfull + acc);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      umma_commit(drain);
      drain_wait(drain, 0);
    }
    __syncwarp();
  } else if (warp < 2 + Cfg::EPI_WARPS) {
    swap_epilogue<DUAL, EPI, Cfg::EPI_WARPS>(p, s_pre, s_offs, total, tmem_base, tfull, tempty, abort_flag, tcode,
                                            warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace moe
