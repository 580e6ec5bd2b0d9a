// tc_swap8.cuh -- the weight-row ("swap-AB") expert GEMMs for E4M3 weights
// with one fp32 scale per 128 x 128 block (the FP8 weight format of the
// Qwen3.8-Max report, chapter "06 · Quantification et matériel"; the tile
// schedule and epilogues are those of tc_swap.cuh).
//
// The weights are again the MMA's M = 128 operand, but the MMA reads them from
// tensor memory: converter warps turn each raw E4M3 tile into bf16 values
// bf16(q * s) and write them with tcgen05.st straight into TMEM columns, which
// the next MMAs take as their A operand.  Converted weights never pass through
// shared memory, so the only shared-memory ring is the raw one, and it is deep.
// A raw K block is 128 codes wide: one scale block, one 128-byte row per weight
// row, loaded with 128-byte swizzling so that the converters' one-row-per-
// thread reads spread over all banks.  The token tile (kNCH rows, two 64-wide
// bf16 K atoms) travels in the same raw slot and is the MMA's B operand there.
//
// TMEM (512 columns): two accumulator buffers of ACC_COLS, then A_STAGES slots
// of A_COLS columns (64 columns = 128 bf16 per weight row, gate then up).
//
// Warps: 0 TMA producer; 1 TMEM owner + MMA issuer; 2..5 epilogue (one thread
// per weight row); 6.. converters, NB / 32 of them: converter warp w owns TMEM
// lane quarter w % 4 (the quarter a warp may access) of matrix (w - 6) / 4.
#pragma once
#include "tc_swap.cuh"

namespace moe {

constexpr int kBK8 = 128;  // E4M3 K block: 128 codes, one scale block, one 128-byte row

template <bool DUAL>
struct Swap8Cfg {
  static constexpr int NB = DUAL ? 256 : 128;     // weight rows per K block: gate then up, or one tile
  static constexpr int X_BYTES = 2 * kNCH * 128;  // token tile: two 64-wide bf16 K atoms
  static constexpr int RAW_BYTES = NB * kBK8 + X_BYTES;
  static constexpr int RAW_STAGES = DUAL ? 4 : 6;
  static constexpr int RING_BYTES = RAW_STAGES * RAW_BYTES;
  static constexpr int EPI_WARPS = 4;
  static constexpr int CONV_WARPS = NB / 32;
  static constexpr int THREADS = 64 + 32 * (EPI_WARPS + CONV_WARPS);
  static constexpr int ACC_COLS = (DUAL ? 2 : 1) * kNCH;
  static constexpr int ACC_BUFS = 2;  // accumulator buffers (epilogue of tile i overlaps tile i + 1)
  static constexpr int A_COLS = (DUAL ? 2 : 1) * (kBK8 / 2);
  static constexpr int A_STAGES = DUAL ? 2 : 4;
  static constexpr int TMEM_COLS = 512;
  static constexpr int BAR_BYTES = (2 * RAW_STAGES + 2 * A_STAGES + 5) * 8 + 16;
  static constexpr int SCHED_INTS = 2 * (512 + 2);
  static constexpr int SMEM_BYTES = 1024 + RING_BYTES + BAR_BYTES + SCHED_INTS * 4;
  static_assert(ACC_BUFS * ACC_COLS + A_STAGES * A_COLS <= TMEM_COLS, "TMEM columns");
  static_assert(RAW_BYTES % 1024 == 0 && (NB * kBK8) % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// tmX*: token-row maps (bf16, box 64 x kNCH, 128-byte swizzle); tmB* / tmC*:
// E4M3 weight maps (box 128 codes x 128 rows, 128-byte swizzle), gate (or the
// single operand) and up; _r routed groups [E, N, K], _s the shared group [N, K].
template <bool DUAL, int EPI>
__global__ void __launch_bounds__(Swap8Cfg<DUAL>::THREADS, 1)
    k_gemm_swap8(const __grid_constant__ CUtensorMap tmX_r, const __grid_constant__ CUtensorMap tmX_s,
                 const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
                 const __grid_constant__ CUtensorMap tmC_r, const __grid_constant__ CUtensorMap tmC_s, TcGemmArgs p) {
  using Cfg = Swap8Cfg<DUAL>;
  constexpr int R = Cfg::RAW_STAGES, A = Cfg::A_STAGES;
  // DUAL with a SlotStore / Store epilogue (the down GEMM): the two matrices
  // are the two 128-row halves of a 256-row weight tile of one matrix, so each
  // K block's handoffs carry twice the weight bytes; the second half's rows
  // and scales start 128 rows further
  constexpr bool HALVES = DUAL && EPI != kTcSwiGLU;
  constexpr int TILE_ROWS = HALVES ? 256 : 128;
  constexpr int C_ROW = HALVES ? 128 : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + Cfg::RING_BYTES);
  uint64_t* raw_empty = raw_full + R;  // converters done with the weights + MMAs done with the tokens
  uint64_t* a_full = raw_empty + R;    // converted A slot written (one arrival per converter warp)
  uint64_t* a_empty = a_full + A;      // MMAs done reading the A slot
  uint64_t* tfull = a_empty + A;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem + Cfg::RING_BYTES + Cfg::BAR_BYTES);
  int32_t* s_offs = s_pre + 514;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned tcode = kStatusTimeoutBase | (kKernGemmSwap << 8);
  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(raw_full + s, 1);
      mbar_init(raw_empty + s, Cfg::CONV_WARPS + 1);
    }
    for (int s = 0; s < A; ++s) {
      mbar_init(a_full + s, Cfg::CONV_WARPS);
      mbar_init(a_empty + s, 1);
    }
    for (int b = 0; b < Cfg::ACC_BUFS; ++b) {
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
        const SwapTile t = decode_swap<TILE_ROWS>(p, s_pre, s_offs, tile);
        const bool sh = t.g == p.E;
        const int nkb = (sh ? p.K_s : p.K_r) / kBK8;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(raw_empty + stage, phase ^ 1, abort_flag, p.status, tcode | 1)) {
            ok = false;
            break;
          }
          uint64_t* land = raw_full + stage;
          uint8_t* base = smem + stage * Cfg::RAW_BYTES;
          uint8_t* xdst = base + Cfg::NB * kBK8;
          const int k0 = kb * kBK8;
          mbar_arrive_expect_tx(land, Cfg::RAW_BYTES);
          if (sh) tma_load_2d(base, &tmB_s, land, k0, t.n0, pol_w);
          else tma_load_3d(base, &tmB_r, land, k0, t.n0, t.g, pol_w);
          if (DUAL) {
            if (sh) tma_load_2d(base + 128 * kBK8, &tmC_s, land, k0, t.n0 + C_ROW, pol_w);
            else tma_load_3d(base + 128 * kBK8, &tmC_r, land, k0, t.n0 + C_ROW, t.g, pol_w);
          }
          const CUtensorMap* tx = sh ? &tmX_s : &tmX_r;
          tma_load_2d(xdst, tx, land, k0, (int)t.row0, pol_x);
          tma_load_2d(xdst + kNCH * 128, tx, land, k0 + 64, (int)t.row0, pol_x);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == R) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag)
        for (int s = 0; s < R; ++s)
          if (issued >> s & 1u) drain_wait(raw_full + s, last_par >> s & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer (A from TMEM, B = token tile)
      int rstage = 0, astage = 0, acc = 0;
      uint32_t aphase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const SwapTile t = decode_swap<TILE_ROWS>(p, s_pre, s_offs, tile);
        // MMA N = the chunk's token rows rounded up to 16: columns past them are
        // neither computed nor read back
        const uint32_t idesc = idesc_bf16(kBM, min(kNCH, (t.rows - t.c0 + 15) & ~15));
        const int nkb = (t.g == p.E ? p.K_s : p.K_r) / kBK8;
        if (!mbar_wait(tempty + acc, acc_phase ^ 1, abort_flag, p.status, tcode | 2)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * Cfg::ACC_COLS;
        for (int kb = 0; kb < nkb; ++kb) {
          // a_full is arrived by the converters after they saw the raw slot
          // land, so the token tile in that slot has landed too.
          if (!mbar_wait(a_full + astage, aphase, abort_flag, p.status, tcode | 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = tmem_base + Cfg::ACC_BUFS * Cfg::ACC_COLS + astage * Cfg::A_COLS;
          const uint32_t sx = smem_u32(smem + rstage * Cfg::RAW_BYTES + Cfg::NB * kBK8);
#pragma unroll
          for (int kk = 0; kk < kBK8 / 16; ++kk) {
            const uint64_t bd = sdesc_sw128(sx + (kk >> 2) * (kNCH * 128) + (kk & 3) * 32);
            const uint32_t accum = (kb | kk) != 0;
            umma_f16_ta(d0, a0 + kk * 8, bd, idesc, accum);
            if (DUAL) umma_f16_ta(d0 + kNCH, a0 + kBK8 / 2 + kk * 8, bd, idesc, accum);
          }
          umma_commit(a_empty + astage);
          umma_commit(raw_empty + rstage);
          if (++astage == A) {
            astage = 0;
            aphase ^= 1;
          }
          if (++rstage == R) rstage = 0;
        }
        if (!ok) break;
        umma_commit(tfull + acc);
        if (++acc == Cfg::ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      umma_commit(drain);
      drain_wait(drain, 0);
    }
    __syncwarp();
  } else if (warp < 2 + Cfg::EPI_WARPS) {
    swap_epilogue<DUAL, EPI, Cfg::EPI_WARPS, Cfg::ACC_BUFS>(p, s_pre, s_offs, total, tmem_base, tfull, tempty, abort_flag, tcode,
                                            warp, lane);
  } else {
    // ------------------------------------------------ E4M3 -> bf16 converters, raw smem -> TMEM
    const int mat = (warp - 2 - Cfg::EPI_WARPS) >> 2;  // 0: gate (or the single operand), 1: up
    const int q = warp & 3;
    const int r = q * 32 + lane;  // weight row within the 128-row tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    int rstage = 0, astage = 0;
    uint32_t rphase = 0, aphase = 0;
    bool stop = false;
    for (int tile = blockIdx.x; tile < total && !stop; tile += gridDim.x) {
      const SwapTile t = decode_swap<TILE_ROWS>(p, s_pre, s_offs, tile);
      const bool sh = t.g == p.E;
      const int nkb = (sh ? p.K_s : p.K_r) / kBK8;
      // the tile's 128 rows are one scale row block: one fp32 scale per K block
      // (a second half past the matrix's last row reads zeros and no scale)
      const float* sbase = mat == 0 ? (sh ? p.sc_b_s : p.sc_b_r) : (sh ? p.sc_c_s : p.sc_c_r);
      const int rb0 = t.n0 + mat * C_ROW;
      const bool rin = rb0 < t.N;
      const float* srow = sbase + ((sh ? 0 : (int64_t)t.g * (t.N / 128)) + rb0 / 128) * (int64_t)nkb;
      float s_cur = rin ? __ldg(srow) : 0.f;
      float s_nxt = rin && nkb > 1 ? __ldg(srow + 1) : 0.f;
      for (int kb = 0; kb < nkb; ++kb) {
        const bool ok = mbar_wait(raw_full + rstage, rphase, abort_flag, p.status, tcode | 5) &&
                        mbar_wait(a_empty + astage, aphase ^ 1, abort_flag, p.status, tcode | 7);
        if (!__all_sync(0xffffffffu, ok)) {  // the warp goes on, or stops, as one
          stop = true;
          break;
        }
        tc_fence_after();
        const uint8_t* src = smem + rstage * Cfg::RAW_BYTES + (mat * 128 + r) * kBK8;
        uint32_t o[64];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4 v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j)  // 16-byte chunk c of the row sits at chunk c ^ (row & 7)
            v[j] = *reinterpret_cast<const uint4*>(src + (((h * 4 + j) ^ (r & 7)) << 4));
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint2 a = e4m3x4_scaled_bf16(v[j].x, s_cur);
            const uint2 b = e4m3x4_scaled_bf16(v[j].y, s_cur);
            const uint2 c = e4m3x4_scaled_bf16(v[j].z, s_cur);
            const uint2 d = e4m3x4_scaled_bf16(v[j].w, s_cur);
            uint32_t* w = o + 32 * h + 8 * j;
            w[0] = a.x;
            w[1] = a.y;
            w[2] = b.x;
            w[3] = b.y;
            w[4] = c.x;
            w[5] = c.y;
            w[6] = d.x;
            w[7] = d.y;
          }
        }
        tmem_st64(tmem_base + lane_off + Cfg::ACC_BUFS * Cfg::ACC_COLS + astage * Cfg::A_COLS + mat * (kBK8 / 2),
                  o);
        // raw weight bytes consumed: order these generic reads before the TMA's refill
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(a_full + astage);
          mbar_arrive(raw_empty + rstage);
        }
        s_cur = s_nxt;
        s_nxt = rin && kb + 2 < nkb ? __ldg(srow + kb + 2) : 0.f;
        if (++astage == A) {
          astage = 0;
          aphase ^= 1;
        }
        if (++rstage == R) {
          rstage = 0;
          rphase ^= 1;
        }
      }
    }
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
