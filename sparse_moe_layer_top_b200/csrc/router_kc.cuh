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
// the four K quarters in a fixed order and selects the best KT (expert, logit)
// pairs of each token among its experts; the owners' lists go to the row
// tile's first CTA by bulk copies, which merges them (equal logits by expert)
// and writes ids, softmax weights renormalised over the kept experts and the
// chunk histogram.
//
// Every thread of every CTA passes the cluster barriers (after the main loop,
// after the owners' sums, before leaving -- once every CTA's bulk copies have
// completed), also after a wait gave up, so no CTA waits on a peer that left
// and no copy lands in a CTA that left; all mbarrier waits are bounded.
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
  static constexpr int BAR_BYTES = (2 * kRouterKcStages + 2 + 4 + 2) * 8 + 16;
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

// Sorting networks on (logit, expert) pairs held in registers, best first:
// a pair is better with the larger logit, or the lower expert on equal logits
// (the router's order).  Fixed, branch-free compare-exchanges: the inserts of
// a sorted-list push are a dependent chain, which measured about 0.4 us per
// pushed candidate per warp when merging lists.
__device__ __forceinline__ bool kc_better(float av, int ae, float bv, int be) {
  return av > bv || (av == bv && ae < be);
}
// after the call, slot a holds the better of the two
__device__ __forceinline__ void kc_cmpx(float& av, int& ae, float& bv, int& be) {
  const bool sw = kc_better(bv, be, av, ae);
  const float tv = sw ? bv : av;
  const int te = sw ? be : ae;
  bv = sw ? av : bv;
  be = sw ? ae : be;
  av = tv;
  ae = te;
}
// bitonic sort of N (a power of two) pairs, best first
template <int N>
__device__ __forceinline__ void kc_sort(float (&v)[N], int (&e)[N]) {
#pragma unroll
  for (int size = 2; size <= N; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          if ((i & size) == 0 || size == N) kc_cmpx(v[i], e[i], v[j], e[j]);
          else kc_cmpx(v[j], e[j], v[i], e[i]);
        }
      }
}
// a (sorted, best first) <- the best N of a and b (sorted, best first): the
// better of a[i] and b[N-1-i] are the best N, in a bitonic order that one
// bitonic merge sorts
template <int N>
__device__ __forceinline__ void kc_merge(float (&av)[N], int (&ae)[N], const float (&bv)[N], const int (&be)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i)
    if (kc_better(bv[N - 1 - i], be[N - 1 - i], av[i], ae[i])) {
      av[i] = bv[N - 1 - i];
      ae[i] = be[N - 1 - i];
    }
#pragma unroll
  for (int stride = N >> 1; stride > 0; stride >>= 1)
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const int j = i ^ stride;
      if (j > i) kc_cmpx(av[i], ae[i], av[j], ae[j]);
    }
}

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
  uint64_t* hfull = recv_full + 1;  // [4] top-k hand-over, one per lane quarter
  uint64_t* lst_ready = hfull + 4;  // this owner's token lists are staged (one arrival per list warp)
  uint64_t* lists_full = lst_ready + 1;  // (rank 0) the other owners' token lists have landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lists_full + 1);
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
    for (int q = 0; q < 4; ++q) mbar_init(hfull + q, 32);
    mbar_init(lst_ready, 4);
    mbar_init(lists_full, 1);
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
      // both stay in L2: W_r serves every row tile, and the gate/up GEMM that
      // follows gathers its rows from x (evict-first here made it about 3 %
      // slower at the 35B shape)
      const uint64_t pol_x = policy_evict_last(), pol_w = policy_evict_last();
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
  // ---- owners: the four K quarters of this CTA's 64 experts, summed in rank
  // order; warp eg holds columns 32 eg .. 32 eg + 31 of its 32 tokens
  uint32_t v[32];
  bool sel = false;  // (warp-uniform) this warp selects
  if (warp >= 2 && owner) {
    const bool got = __all_sync(0xffffffffu, mbar_wait_poll(recv_full, 0, abort_flag, p.status, tcode | 5));
    sel = got && acc_ok && !*abort_flag;
    if (sel) {
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
    }
  }
  // (C) every owner has read its receive blocks: rank 0's become the list buffer
  cluster_sync_all();
  const int list_bytes = KT * kBM * 8;  // an owner's lists: KT logits, then KT experts, per token
  float* lst_v = reinterpret_cast<float*>(send) + 4096;  // staging, past the hand-over (send blocks are read)
  int* lst_e = reinterpret_cast<int*>(lst_v + KT * kBM);
  if (sel) {
    // best KT of this warp's 32 experts (bias added; experts past E at -inf):
    // groups of KT sorted, then merged
    const int e0 = (int)rank * 64 + eg * 32;
    float tv[KT], bv[KT];
    int te[KT], be[KT];
#pragma unroll
    for (int gbase = 0; gbase < 32; gbase += KT) {
      float* gv = gbase == 0 ? tv : bv;
      int* ge = gbase == 0 ? te : be;
#pragma unroll
      for (int i = 0; i < KT; ++i) {
        const int e = e0 + gbase + i;
        ge[i] = e < p.N_s ? e : 0x7fffffff;
        gv[i] = e < p.N_s ? __uint_as_float(v[gbase + i]) + (p.bias ? __ldg(p.bias + e) : 0.f) : -INFINITY;
      }
      if (gbase == 0) {
        kc_sort<KT>(tv, te);
      } else {
        kc_sort<KT>(bv, be);
        kc_merge<KT>(tv, te, bv, be);
      }
    }
    // the second warp of a lane quarter hands its list to the first (its
    // experts are all higher, which keeps the order of equal logits)
    float* xv = reinterpret_cast<float*>(hand + q * 4096);
    int* xe = reinterpret_cast<int*>(hand + q * 4096 + 2048);
    if (eg) {
#pragma unroll
      for (int i = 0; i < KT; ++i) {
        xv[i * 32 + lane] = tv[i];
        xe[i * 32 + lane] = te[i];
      }
      mbar_arrive(hfull + q);
    } else if (__all_sync(0xffffffffu, mbar_wait_poll(hfull + q, 0, abort_flag, p.status, tcode | 9))) {
#pragma unroll
      for (int i = 0; i < KT; ++i) {
        bv[i] = xv[i * 32 + lane];
        be[i] = xe[i * 32 + lane];
      }
      kc_merge<KT>(tv, te, bv, be);
      if (rank != 0) {
        // the owner's list of this token to rank 0's list buffer
#pragma unroll
        for (int i = 0; i < KT; ++i) {
          lst_v[i * kBM + row] = tv[i];
          lst_e[i * kBM + row] = te[i];
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(lst_ready);
        if (warp == 2 && lane == 0 &&
            mbar_wait_poll(lst_ready, 0, abort_flag, p.status, tcode | 10))
          bulk_copy_to_cta(mapa_rank(reinterpret_cast<float*>(recv) + (int)rank * (KT * kBM * 2), 0u), lst_v,
                           (uint32_t)list_bytes, mapa_rank(lists_full, 0u));
      } else {
        // rank 0: merge the other owners' lists (higher experts) and write
        if (warp == 2 && lane == 0 && owners > 1)
          mbar_arrive_expect_tx(lists_full, (uint32_t)((owners - 1) * list_bytes));
        const bool have = owners == 1 ||
                          __all_sync(0xffffffffu, mbar_wait_poll(lists_full, 0, abort_flag, p.status, tcode | 11));
        if (have) {
          const float* rv = reinterpret_cast<const float*>(recv);
          for (int o = 1; o < owners; ++o) {
            const float* ov = rv + o * (KT * kBM * 2);
            const int* oe = reinterpret_cast<const int*>(ov + KT * kBM);
#pragma unroll
            for (int i = 0; i < KT; ++i) {
              bv[i] = ov[i * kBM + row];
              be[i] = oe[i * kBM + row];
            }
            kc_merge<KT>(tv, te, bv, be);
          }
          const int64_t grow = (int64_t)rt * kBM + row;
          if (grow < p.rows_cap) {
            const float m = tv[0];
            float den = 0.f;
#pragma unroll
            for (int i = 0; i < KT; ++i)
              if (i < p.topk) den += __expf(tv[i] - m);
            int32_t* hist = p.counts ? p.counts + (grow / kBM) * p.N_s : nullptr;
#pragma unroll
            for (int i = 0; i < KT; ++i)
              if (i < p.topk) {
                p.ids[grow * p.topk + i] = te[i];
                p.tw[grow * p.topk + i] = __expf(tv[i] - m) / den;
                if (hist) atomicAdd(hist + te[i], 1);
              }
          }
        }
      }
    }
  }
  // (D) every CTA's bulk copies have completed: none is in flight into a CTA
  // that leaves
  if (warp == 2 && lane == 0) bulk_wait_all();
  cluster_sync_all();

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace moe
