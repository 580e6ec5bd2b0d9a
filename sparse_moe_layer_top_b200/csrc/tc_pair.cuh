// tc_pair.cuh -- the row-tiled expert GEMMs on CTA pairs, for groups with many
// rows (prefill-sized batches).
//
// Each 2-CTA cluster computes 256-row tiles with the pair form of the 5th-
// generation tensor core (tcgen05 .cta_group::2, M = 256, N = 256): rank r of
// the pair loads rows r*128 .. r*128+127 of the activation tile and one half
// of the weight tile -- gate rows on rank 0 and up rows on rank 1 for the
// gate/up GEMM, weight rows n0 .. n0+127 and n0+128 .. n0+255 for the down
// GEMM -- and keeps its own 128 accumulator rows in its TMEM.  Per SM and K
// block that is 32 KB of operands for the same MMA work that costs 48 KB in the
// single-CTA kernel (tc_gemm.cuh): the single-CTA kernel is bound by those
// operand bytes at prefill shapes, not by the tensor core.
//
// Synchronisation, per K block (stage s):
//   * rank 0's producer arms rank 0's full[s] with the bytes of both CTAs;
//     both producers load their own tiles with the pair form of the TMA load,
//     whose transaction bytes complete on rank 0's full[s];
//   * rank 0's MMA thread waits on full[s], issues the pair MMAs, and commits
//     with a multicast arrive on empty[s] of both CTAs (each producer refills
//     stage s only after that, so no CTA's bytes can run a phase ahead);
//   * tile done: multicast commit on tfull[acc] of both CTAs; every epilogue
//     warp of both CTAs arrives on rank 0's tempty[acc] (locally or remotely);
//   * barriers that the other CTA or the pair's commit arrive on are waited
//     on with cluster-scope acquire; the last cluster barrier comes after rank
//     0 has seen every MMA complete, so neither CTA exits under a pair MMA.
// A per-stage relay through a thread of rank 1 (wait on its own full[s], then
// a cluster-release arrive on rank 0) was measured first: 2.1x slower than one
// CTA per tile with the loads on, as fast as expected with them off -- the
// per-stage release serialised the load pipeline.
// No TMA load uses cluster multicast: each CTA loads only its own tiles.
//
// Warps: 0 TMA producer; 1 TMEM allocation (both ranks) and MMA issuer
// (rank 0); 2..9 epilogue (the row-tiled epilogue of tc_gemm.cuh on this
// CTA's 128 rows).
#pragma once
#include "tc_gemm.cuh"

namespace moe {

constexpr int kPairBM = 256;  // rows per pair tile

template <int BN, bool DUAL, int STAGES>
struct PairCfg {
  static constexpr int N = DUAL ? 2 * BN : BN;  // MMA N: gate | up, or one weight block
  static constexpr int A_BYTES = 128 * kBK * 2;
  static constexpr int BH_BYTES = (N / 2) * kBK * 2;  // this CTA's half of the weight tile
  static constexpr int STAGE_BYTES = A_BYTES + BH_BYTES;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int ACC_COLS = N;
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  static constexpr int BAR_BYTES = (2 * STAGES + 5) * 8 + 16;
  static constexpr int SCHED_INTS = 2 * (512 + 2);
  static constexpr int EPI_OFF = (RING_BYTES + BAR_BYTES + SCHED_INTS * 4 + 127) / 128 * 128;
  static constexpr int SMEM_BYTES = 1024 + EPI_OFF + EPI_WARPS * 2048;
  static_assert(N == 256, "the pair MMA here is M = 256, N = 256");
  static_assert(TMEM_COLS == 512, "TMEM columns");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// tmA*: activation rows (box 64 x 128); tmB*, tmC*: weight maps with 128-row
// boxes (gate, up; the down GEMM uses tmB only).  Launched as 2-CTA clusters.
template <int BN, bool DUAL, int STAGES, int EPI>
__global__ void __launch_bounds__(PairCfg<BN, DUAL, STAGES>::THREADS, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
                const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
                const __grid_constant__ CUtensorMap tmC_r, const __grid_constant__ CUtensorMap tmC_s, TcGemmArgs p) {
  using Cfg = PairCfg<BN, DUAL, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::RING_BYTES);  // used on rank 0
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;      // rank 0: both CTAs' epilogues are done with the accumulator
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem + Cfg::RING_BYTES + Cfg::BAR_BYTES);
  int32_t* s_offs = s_pre + 514;
  uint8_t* epi_stage = smem + Cfg::EPI_OFF;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const unsigned tcode = kStatusTimeoutBase | (kKernGemmTc << 8) | 0x80u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, 2 * Cfg::EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA_r);
    prefetch_tmap(&tmA_s);
    prefetch_tmap(&tmB_r);
    prefetch_tmap(&tmB_s);
    if (DUAL) {
      prefetch_tmap(&tmC_r);
      prefetch_tmap(&tmC_s);
    }
  }
  cluster_sync_all();  // the peer CTA is running and both CTAs' barriers are initialised
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);  // with the peer's warp 1
    tmem_relinquish_pair();
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
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_pre[p.E + 1];

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both ranks, own tiles only)
      const uint64_t pol_keep = policy_evict_last(), pol_stream = policy_evict_first();
      const uint32_t full0 = mapa_rank(full, 0);
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const TileInfo t = decode_tile<BN, kPairBM>(p, s_pre, s_offs, tile);
        const bool sh = t.g == p.E;
        const LoadPolicy lp = load_policy(t, pol_keep, pol_stream);
        const uint64_t pol_w = lp.w, pol_a = lp.a;
        const int arow = (int)t.row0 + (int)rank * 128;
        // gate/up: rank 0 loads the gate rows, rank 1 the up rows; down: the two row halves
        const CUtensorMap* wmap = DUAL ? (rank ? (sh ? &tmC_s : &tmC_r) : (sh ? &tmB_s : &tmB_r))
                                       : (sh ? &tmB_s : &tmB_r);
        const int wrow = DUAL ? t.n0 : t.n0 + (int)rank * 128;
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait_cluster(empty + stage, phase ^ 1, abort_flag, p.status, tcode | 1)) {
            ok = false;
            break;
          }
          const uint32_t land = full0 + stage * 8;  // rank 0's full[stage]
          uint8_t* sa = smem + stage * Cfg::STAGE_BYTES;
          if (rank == 0) mbar_arrive_expect_tx(full + stage, 2 * Cfg::STAGE_BYTES);
          tma_load_2d_pair(sa, sh ? &tmA_s : &tmA_r, land, kb * kBK, arow, pol_a);
          if (sh) tma_load_2d_pair(sa + Cfg::A_BYTES, wmap, land, kb * kBK, wrow, pol_w);
          else tma_load_3d_pair(sa + Cfg::A_BYTES, wmap, land, kb * kBK, wrow, t.g, pol_w);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // copies in flight must land before the CTA exits: rank 0 waits for the
      // stages it armed (which also count rank 1's bytes); rank 1's copies land
      // in its own shared memory and both CTAs stay until the last cluster barrier
      if (*abort_flag && rank == 0)
        for (int s = 0; s < STAGES; ++s)
          if (issued >> s & 1u) drain_wait(full + s, last_par >> s & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------ MMA issuer (rank 0)
      constexpr uint32_t idesc = idesc_bf16(kPairBM, Cfg::N);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const TileInfo t = decode_tile<BN, kPairBM>(p, s_pre, s_offs, tile);
        if (!mbar_wait_cluster(tempty + acc, acc_phase ^ 1, abort_flag, p.status, tcode | 2)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * Cfg::ACC_COLS;
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait_cluster(full + stage, phase, abort_flag, p.status, tcode | 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t accum = (kb != t.kb0 || kk != 0);
            umma_f16_pair(d0, sdesc_sw128(sa + kk * 32), sdesc_sw128(sb + kk * 32), idesc, accum);
          }
          umma_commit_pair(empty + stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair(tfull + acc);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // every MMA issued must finish before TMEM is released
      umma_commit_pair(drain);
      drain_wait(drain, 0);
    }
    __syncwarp();
  } else if (warp < 2 + Cfg::EPI_WARPS) {
    // ------------------------------------------------ epilogue (both ranks, own 128 rows)
    constexpr int EG = Cfg::EPI_WARPS / 4;
    constexpr int CPW = (BN / 32) / EG;
    const int eg = (warp - 2) / 4;
    const int q = warp & 3;
    const int row = (int)rank * 128 + q * 32 + lane;  // row of the 256-row tile
    const uint32_t tempty0 = mapa_rank(tempty, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total; tile += npairs) {
      const TileInfo t = decode_tile<BN, kPairBM>(p, s_pre, s_offs, tile);
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(tfull + acc, acc_phase, abort_flag, p.status, tcode | 4)))
        break;  // the warp stops as one: its TMEM loads are warp-collective
      tc_fence_after();
      const uint32_t tb = tmem_base + acc * Cfg::ACC_COLS + ((uint32_t)(q * 32) << 16);
      epilogue_rows<BN, EPI>(p, t, tb, row, eg * CPW, (eg + 1) * CPW, epi_stage + (warp - 2) * 2048, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cta_scope(tempty0 + acc * 8);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no remote arrival or pair MMA is still in flight for either CTA
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace moe
