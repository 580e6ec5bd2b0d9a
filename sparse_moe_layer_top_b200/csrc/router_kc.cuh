// router_kc.cuh -- the router GEMM with the top-k selection in its epilogue
// for up to 256 experts, its K dimension split over a cluster of 4 CTAs.
//
// The cluster computes the logits of one 128-token row tile for all E <= 256
// experts (tcgen05, M = 128 tokens, N = E rounded up to 16): CTA r of the
// cluster runs the K blocks [r nkb / 4, (r + 1) nkb / 4), so each CTA loads a
// quarter of the token tile and a quarter of W_r once -- the expert-tiled
// router loaded the whole token tile once per 64-expert column tile.  Then the
// four fp32 partial accumulators are exchanged through distributed shared
// memory: CTA c owns experts 64 c .. 64 c + 63; every CTA stages its partial
// columns of each other owner's experts as a 32 KB block in its own shared
// memory and one bulk copy per owner (cp.async.bulk shared::cta ->
// shared::cluster, no multicast) moves it into that owner's receive block,
// completing on the owner's mbarrier (the ring, idle after the main loop,
// holds both); storing the partials into the peers' shared memory thread by
// thread was slower (8 us for the exchange at the 35B shape, against 5).  c sums
// the four K quarters in a fixed order, writes the sums back to TMEM and runs
// the row-tiled router's top-k epilogue (topk_epilogue, tc_gemm.cuh) as
// column tile c: the last of a row tile's owners to finish merges the lists
// and writes ids, weights and the chunk histogram.
//
// Every thread of every CTA passes the cluster barrier at the main loop's end,
// also after a wait gave up, so no CTA waits on a peer that left; all
// mbarrier waits are bounded, and a CTA leaves only once its own bulk copies
// and those into it have completed.
//
// Warps: 0 TMA producer; 1 TMEM owner and MMA issuer; 2..9 exchange and
// top-k epilogue (two warps per TMEM lane quarter, splitting the columns).
#pragma once
#include "tc_gemm.cuh"

namespace moe {

constexpr int kRouterKcCtas = 4;       // cluster size: K quarters, and owners of 64 experts each
constexpr int kRouterKcStages = 4;
constexpr int kRouterKcStageBytes = kBM * kBK * 2 + 256 * kBK * 2;  // token tile + up to 256 expert rows
constexpr int kRouterKcBlock = kBM * 64 * 4;  // one CTA's partial logits of one owner's 64 experts (fp32)
constexpr int kRouterKcRecvBytes = kRouterKcCtas * kRouterKcBlock;           // an owner's four K quarters
constexpr int kRouterKcSendBytes = (kRouterKcCtas - 1) * kRouterKcBlock;     // the blocks for the other owners
constexpr int kRouterKcHandBytes = 4 * 4096;  // top-k hand-over lists: 4 lane quarters x (16 slots x 32 x 8 B)

struct RouterKcCfg {
  static constexpr int RING_BYTES = kRouterKcStages * kRouterKcStageBytes;
  static constexpr int BUF_BYTES =
      RING_BYTES > kRouterKcRecvBytes + kRouterKcSendBytes ? RING_BYTES : kRouterKcRecvBytes + kRouterKcSendBytes;
  static constexpr int BAR_BYTES = (2 * kRouterKcStages + 2 + 8) * 8 + 16;
  static constexpr int SMEM_BYTES = 1024 + BUF_BYTES + BAR_BYTES;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int TMEM_COLS = 256;
  static_assert(kRouterKcHandBytes <= kRouterKcSendBytes, "the hand-over lists reuse the send blocks");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// A 128 x 64 fp32 block, row r's 16-byte chunk j at chunk j ^ (r & 7): the
// row-per-thread writes and reads of 8 consecutive rows hit distinct banks.
__device__ __forceinline__ int kc_chunk(int r, int j) { return r * 16 + (j ^ (r & 7)); }

// tmX: the token matrix (box 64 x 128); tmW: W_r (box 64 x npad rows, npad =
// E rounded up to 16).  p: N_s = E, K_s = d, rows_cap = T, and the TopK fields
// of TcGemmArgs.  Grid: 4 CTAs per 128-token row tile, launched as 4-CTA
// clusters.
template <int KT>
__global__ void __launch_bounds__(RouterKcCfg::THREADS, 1)
    k_router_kc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, TcGemmArgs p,
                int npad) {
  using Cfg = RouterKcCfg;
  constexpr int S = kRouterKcStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::BUF_BYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* recv_full = tfull + 1;  // the three other K quarters of this CTA's experts have landed
  uint64_t* hfull = recv_full + 1;  // [4] top-k hand-over, one pair per lane quarter
  uint64_t* hempty = hfull + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(hempty + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // after the main loop: recv [source rank] and send [owner slot] blocks, then
  // the hand-over lists over the send blocks
  float4* recv = reinterpret_cast<float4*>(smem);
  float4* send = reinterpret_cast<float4*>(smem + kRouterKcRecvBytes);
  uint8_t* hand = smem + kRouterKcRecvBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int rt = (int)(blockIdx.x / kRouterKcCtas);  // row tile
  const unsigned tcode = kStatusTimeoutBase | (kKernGemmTc << 8);
  const int nkb = (p.K_s + kBK - 1) / kBK;
  const int kb_lo = (int)((int64_t)rank * nkb / kRouterKcCtas);
  const int kb_hi = (int)((int64_t)(rank + 1) * nkb / kRouterKcCtas);
  const int owners = (p.N_s + 63) / 64;  // CTAs that own experts (column tiles of 64)
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(tfull, 1);
    mbar_init(recv_full, 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(hfull + q, 32);
      mbar_init(hempty + q, 32);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_begin();  // x and W_r may come from earlier kernels in the stream
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool acc_ok = true;  // (epilogue warps) the accumulator is complete

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer: this CTA's K quarter
      const uint64_t pol_x = policy_evict_first(), pol_w = policy_evict_last();
      const uint32_t tx = (uint32_t)(kBM * kBK * 2 + npad * kBK * 2);
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(empty + stage, phase ^ 1, abort_flag, p.status, tcode | 1)) break;
        uint8_t* sa = smem + stage * kRouterKcStageBytes;
        mbar_arrive_expect_tx(full + stage, tx);
        tma_load_2d(sa, &tmX, full + stage, kb * kBK, rt * kBM, pol_x);
        tma_load_2d(sa + kBM * kBK * 2, &tmW, full + stage, kb * kBK, 0, pol_w);
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
      // every copy lands before the ring becomes the exchange buffers
      if (*abort_flag)
        for (int s = 0; s < S; ++s)
          if (issued >> s & 1u) drain_wait(full + s, last_par >> s & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16(kBM, npad);
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(full + stage, phase, abort_flag, p.status, tcode | 3)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + stage * kRouterKcStageBytes);
        const uint32_t sb = sa + kBM * kBK * 2;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_f16(tmem_base, sdesc_sw128(sa + kk * 32), sdesc_sw128(sb + kk * 32), idesc, (kb != kb_lo || kk != 0));
        umma_commit(empty + stage);
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
      // the accumulator is complete once every MMA issued has finished (none:
      // at once); wait for it here too, so the ring is idle at the barrier
      umma_commit(tfull);
      drain_wait(tfull, 0);
    }
    __syncwarp();
  } else {
    acc_ok = __all_sync(0xffffffffu, mbar_wait(tfull, 0, abort_flag, p.status, tcode | 4));
  }

  // (A) every CTA of the cluster is done with its ring: it becomes the
  // exchange buffers
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const int q = warp & 3, eg = (warp - 2) / 4, row = q * 32 + lane;
  const uint32_t lane_off = (uint32_t)(q * 32) << 16;
  const bool owner = (int)rank < owners;
  if (warp >= 2) {
    // this CTA's partial logits of owner c's experts (owners eg, eg + 2):
    // into its own receive block when c is this CTA, else into the send
    // block for c; zeros without K blocks
    const bool have = acc_ok && kb_hi > kb_lo && !*abort_flag;
    for (int c = eg; c < owners; c += 2) {
      uint32_t a[32], b[32];
      if (have) {
        tmem_ld32(tmem_base + lane_off + c * 64, a);
        tmem_ld32(tmem_base + lane_off + c * 64 + 32, b);
        tmem_wait_regs(a);
        tmem_wait_regs(b);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) a[j] = b[j] = 0u;
      }
      const int slot = c < (int)rank ? c : c - 1;
      float4* blk = c == (int)rank ? recv + (int)rank * (kRouterKcBlock / 16) : send + slot * (kRouterKcBlock / 16);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        blk[kc_chunk(row, j)] = make_float4(__uint_as_float(a[4 * j]), __uint_as_float(a[4 * j + 1]),
                                            __uint_as_float(a[4 * j + 2]), __uint_as_float(a[4 * j + 3]));
#pragma unroll
      for (int j = 0; j < 8; ++j)
        blk[kc_chunk(row, 8 + j)] = make_float4(__uint_as_float(b[4 * j]), __uint_as_float(b[4 * j + 1]),
                                                __uint_as_float(b[4 * j + 2]), __uint_as_float(b[4 * j + 3]));
    }
    fence_proxy_async_smem();  // the send blocks are read by the bulk copies (async proxy)
    named_bar_sync(1, 32 * Cfg::EPI_WARPS);
    if (warp == 2 && lane == 0) {
      // each send block to its owner's receive block of this rank, completing
      // on the owner's recv_full; this CTA's own three quarters arrive likewise
      for (int c = 0; c < owners; ++c) {
        if (c == (int)rank) continue;
        const int slot = c < (int)rank ? c : c - 1;
        bulk_copy_to_cta(mapa_rank(recv + (int)rank * (kRouterKcBlock / 16), (uint32_t)c), send + slot * (kRouterKcBlock / 16),
                         (uint32_t)kRouterKcBlock, mapa_rank(recv_full, (uint32_t)c));
      }
      bulk_commit();
      if (owner) mbar_arrive_expect_tx(recv_full, (uint32_t)((kRouterKcCtas - 1) * kRouterKcBlock));
      bulk_wait_read_all();  // the send blocks may now be reused (hand-over lists)
    }
    named_bar_sync(1, 32 * Cfg::EPI_WARPS);
  }
  if (warp >= 2 && owner) {
    const bool got = __all_sync(0xffffffffu, mbar_wait(recv_full, 0, abort_flag, p.status, tcode | 5));
    if (got && acc_ok && !*abort_flag) {
      // the four K quarters of this CTA's experts, summed in rank order; warp
      // eg takes columns 32 eg .. 32 eg + 31, writes them to TMEM and selects
      uint32_t v[32];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 s = recv[kc_chunk(row, eg * 8 + j)];
#pragma unroll
        for (int r = 1; r < kRouterKcCtas; ++r) {
          const float4 o = recv[r * (kRouterKcBlock / 16) + kc_chunk(row, eg * 8 + j)];
          s.x += o.x;
          s.y += o.y;
          s.z += o.z;
          s.w += o.w;
        }
        v[4 * j] = __float_as_uint(s.x);
        v[4 * j + 1] = __float_as_uint(s.y);
        v[4 * j + 2] = __float_as_uint(s.z);
        v[4 * j + 3] = __float_as_uint(s.w);
      }
      tmem_st32(tmem_base + lane_off + eg * 32, v);
      tmem_wait_st();
      TileInfo t{};
      t.g = 0;
      t.rows = (int)p.rows_cap;
      t.m0 = rt * kBM;
      t.row0 = t.m0;
      t.n0 = (int)rank * 64;
      t.N = p.N_s;
      t.kb0 = 0;
      t.kb1 = nkb;
      const int64_t grow = t.row0 + row;
      float* xv = reinterpret_cast<float*>(hand + q * 4096);
      int* xe = reinterpret_cast<int*>(hand + q * 4096 + 2048);
      topk_epilogue<64, 2, KT>(p, t, tmem_base + lane_off, eg, row, grow, grow < p.rows_cap, xv, xe, hfull + q,
                               hempty + q, 0u, abort_flag, tcode | 9, lane);
    }
  }
  if (warp == 2 && lane == 0) {
    bulk_wait_all();                     // no copy of this CTA is in flight when it exits,
    if (owner) drain_wait(recv_full, 0);  // nor one into it (bounded, also after a wait gave up)
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
