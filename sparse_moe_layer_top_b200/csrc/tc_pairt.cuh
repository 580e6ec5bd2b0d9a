// tc_pairt.cuh -- the expert GEMMs on CTA pairs with the tokens as the MMA's
// N operand: any group size, padded to 16 rows instead of a full tile.
//
// A 2-CTA cluster runs tcgen05 .cta_group::2 MMAs of M = 256 weight rows by
// N = the tile's token rows rounded up to 16 (at most 256).  Each CTA holds
// 128 weight rows (its half of M) and half of the token rows (N / 2, the
// pair form's split of B), so per SM and K block it loads 16 KB of weights
// and at most 16 KB of tokens for up to 128 x 256 x 64 MACs -- the operand
// bytes per MMA flop of the row-tiled pair kernel (tc_pair.cuh), whose tiles
// pad every group to 256 rows.  At the prefill shape with Zipf-skewed routing
// most groups are far smaller than 256 rows and the large groups' last tiles
// are ragged; here a tile of 20 tokens costs an N = 32 MMA.
//
// Weight rows per CTA (rank r of the pair, tile at output feature n0):
//   gate/up: gate rows n0 + 64 r .. + 63 in rows 0..63 of the A tile and the
//            up rows of the same features in rows 64..127 (two 64-row TMA
//            boxes), so gate and up of a feature sit in TMEM lanes l and
//            l + 64 of the same CTA; the tile covers 128 features;
//   down:    weight rows n0 + 128 r .. + 127; the tile covers 256 features.
// The accumulator of a CTA holds one weight row per TMEM lane and one token
// per column; the epilogue writes it transposed (each warp store is one
// token's 32 consecutive features).  SwiGLU pairs lane quarters 0 and 2 (and
// 1 and 3): each warp of a pair hands the other half of its 32-token chunk to
// its partner through shared memory and computes H for the half it keeps.
//
// Synchronisation is that of tc_pair.cuh: rank 0 arms its full[s] with both
// CTAs' bytes, both CTAs' TMA loads (pair form, no multicast) complete on it,
// rank 0 issues the MMAs and commits to both CTAs' empty[s] and tfull[acc],
// every epilogue warp of both CTAs arrives on rank 0's tempty[acc].  Tiles are
// dealt round-robin to the pairs in the schedule's panel order.
//
// Warps: 0 TMA producer; 1 TMEM allocation (both ranks) and MMA issuer
// (rank 0); 2..9 epilogue.
#pragma once
#include "tc_pair.cuh"

namespace moe {

constexpr int kPairTRows = 256;  // token rows per tile (the largest MMA N)
constexpr int kTokBox = 32;      // rows of one small token TMA box
constexpr int kTokBoxWide = 128; // rows of the token box of a CTA holding more than 96 rows

template <bool DUAL, int STAGES>
struct PairTCfg {
  static constexpr int BN = DUAL ? 128 : 256;   // output features per tile
  static constexpr int A_BYTES = 128 * kBK * 2;  // this CTA's weight rows
  static constexpr int B_BYTES = 128 * kBK * 2;  // this CTA's token rows (at most 128)
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr int EPI_WARPS = 8;
  // two TMA producer warps (0 and the last one), taking alternate K blocks
  static constexpr int PRODUCER2_WARP = 2 + EPI_WARPS;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS + 32;
  static constexpr int ACC_COLS = kPairTRows;
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  static constexpr int BAR_BYTES = (2 * STAGES + 5) * 8 + 16;
  static constexpr int SCHED_INTS = 2 * (512 + 2);
  static constexpr int EPI_OFF = (RING_BYTES + BAR_BYTES + SCHED_INTS * 4 + 127) / 128 * 128;
  static constexpr int EPI_SCRATCH = 16 * 36 * 4;  // per epilogue warp (kEpiScratchBytes)
  static constexpr int SMEM_BYTES = 1024 + EPI_OFF + EPI_WARPS * EPI_SCRATCH;
  static_assert(TMEM_COLS == 512, "TMEM columns");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Token rows of a tile: `here` real ones, the MMA's N (here rounded up to
// 16), and the rows each CTA holds (N / 2), loaded in kTokBox-row boxes, or
// in one kTokBoxWide-row box when there are more than 96 (fewer TMA issues).
struct PairTShape {
  int here, n, nh, boxes, box_rows;
};
__device__ __forceinline__ PairTShape pairt_shape(const TileInfo& t) {
  PairTShape s;
  s.here = min(kPairTRows, t.rows - t.m0);
  s.n = (s.here + 15) & ~15;
  s.nh = s.n >> 1;
  const bool wide = s.nh > 3 * kTokBox;
  s.box_rows = wide ? kTokBoxWide : kTokBox;
  s.boxes = wide ? 1 : (s.nh + kTokBox - 1) / kTokBox;
  return s;
}

// st.global.v4 with an L2 cache-policy hint.
__device__ __forceinline__ void st_global_v4_hint(void* p, uint4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w), "l"(pol)
               : "memory");
}

// Per-warp epilogue scratch: the SwiGLU hand-over (16 tokens x 32 lanes fp32)
// or the down projection's staging (16 tokens x 32 features fp32, rows padded
// to 36 words so that the 16-byte reads of a quarter warp hit distinct banks).
constexpr int kStageRowWords = 36;
constexpr int kEpiScratchBytes = 16 * kStageRowWords * 4;

// SwiGLU epilogue of one warp (lane quarter q, token-chunk group eg) of rank
// `rank`: chunks of 32 tokens, eg taking every other one.  Quarters 0/1 hold
// gate rows, 2/3 the up rows of the same features; `mine` / `theirs` are this
// warp's and its partner's scratch, `bar` their named barrier.  Each warp
// keeps 16 tokens of a chunk (gate warp the first, up warp the last), stages
// their bf16 H values as 16 rows of 64 bytes and stores them 16 bytes a lane.
__device__ __forceinline__ void pairt_epilogue_swiglu(const TcGemmArgs& p, const TileInfo& t, const PairTShape& s,
                                                      uint32_t tb, uint32_t rank, int q, int eg, float* mine,
                                                      const float* theirs, int bar, int lane, uint64_t pol) {
  const bool gate = q < 2;
  const int f0 = t.n0 + (int)rank * 64 + (q & 1) * 32;  // the warp's first output feature
  uint8_t* stg = reinterpret_cast<uint8_t*>(mine);
#pragma unroll 1
  for (int c = eg; c * 32 < s.here; c += 2) {
    uint32_t a[32];
    tmem_ld32(tb + c * 32, a);
    tmem_wait_regs(a);
    // the gate warp keeps tokens 0..15 of the chunk, the up warp 16..31
    const int keep = gate ? 0 : 16;
#pragma unroll
    for (int i = 0; i < 16; ++i) mine[i * 32 + lane] = __uint_as_float(gate ? a[16 + i] : a[i]);
    named_bar_sync(bar, 64);
    float h[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float other = theirs[i * 32 + lane];
      const float own = __uint_as_float(gate ? a[i] : a[16 + i]);
      h[i] = gate ? silu_f32(own) * other : silu_f32(other) * own;
    }
    named_bar_sync(bar, 64);  // the partner has read `mine`: it becomes the staging rows
#pragma unroll
    for (int i = 0; i < 16; ++i)
      *reinterpret_cast<__nv_bfloat16*>(stg + i * 64 + lane * 2) = __float2bfloat16_rn(h[i]);
    __syncwarp();
    const int j0 = c * 32 + keep;
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int idx = it * 32 + lane, rr = idx >> 2, cc = idx & 3;
      const int j = j0 + rr, f = f0 + cc * 8;
      const int64_t grow = t.row0 + j;
      const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 64 + cc * 16);
      if (j < s.here && grow < p.rows_cap && f < t.N) st_global_v4_hint(p.H + grow * p.ldh + f, v, pol);
    }
    __syncwarp();  // staging read before the next chunk's hand-over overwrites it
  }
}

// Down-projection epilogue (SlotStore: weighted, into the token's slot row;
// Store: into the dispatched row) of one warp: lane = output feature, 32-token
// chunks, eg taking every other one.  The chunks' destination rows and
// weights (lane j: token j of the chunk) are read before the accumulator is
// ready (`dst`, `wt`, filled by pairt_rows_prefetch); each half chunk goes
// through the staging rows and out as one token's 8 features per lane.
constexpr int kMaxChunksPerWarp = kPairTRows / 64;
template <int EPI>
__device__ __forceinline__ void pairt_rows_prefetch(const TcGemmArgs& p, const TileInfo& t, const PairTShape& s,
                                                    int eg, int lane, int (&dst)[kMaxChunksPerWarp],
                                                    float (&wt)[kMaxChunksPerWarp]) {
#pragma unroll
  for (int i = 0; i < kMaxChunksPerWarp; ++i) {
    const int j = (eg + 2 * i) * 32 + lane;
    const int64_t gl = t.row0 + j;
    dst[i] = -1;
    wt[i] = 1.f;
    if (j < s.here && gl < p.rows_cap) {
      if (EPI == kTcSlotStore) {
        const int64_t dr = __ldg(p.row_dst + gl);
        wt[i] = __ldg(p.row_w + gl);
        dst[i] = dr >= 0 && in_range(dr, p.ys_rows, p.status, kSiteSlotRow) ? (int)dr : -1;
      } else {
        dst[i] = (int)gl;
      }
    }
  }
}
template <int EPI>
__device__ __forceinline__ void pairt_epilogue_rows(const TcGemmArgs& p, const TileInfo& t, const PairTShape& s,
                                                    uint32_t tb, uint32_t rank, int q, int eg, int lane,
                                                    const int (&dst)[kMaxChunksPerWarp],
                                                    const float (&wt)[kMaxChunksPerWarp], float* stg, uint64_t pol) {
  const int f0 = t.n0 + (int)rank * 128 + q * 32;
#pragma unroll
  for (int i = 0; i < kMaxChunksPerWarp; ++i) {
    const int c = eg + 2 * i;
    if (c * 32 >= s.here) break;  // uniform over the warp
    uint32_t a[32];
    tmem_ld32(tb + c * 32, a);
    tmem_wait_regs(a);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int j = 0; j < 16; ++j) stg[j * kStageRowWords + lane] = __uint_as_float(a[h * 16 + j]);
      __syncwarp();
#pragma unroll
      for (int it = 0; it < 2; ++it) {
        const int idx = it * 32 + lane, rr = idx >> 2, cc = idx & 3;
        const int dr = __shfl_sync(0xffffffffu, dst[i], h * 16 + rr);
        const float w = __shfl_sync(0xffffffffu, wt[i], h * 16 + rr);
        const float4 x0 = *reinterpret_cast<const float4*>(stg + rr * kStageRowWords + cc * 8);
        const float4 x1 = *reinterpret_cast<const float4*>(stg + rr * kStageRowWords + cc * 8 + 4);
        const int f = f0 + cc * 8;
        if (dr >= 0 && f < t.N) {
          const uint4 v = make_uint4(pack_bf16x2(w * x0.x, w * x0.y), pack_bf16x2(w * x0.z, w * x0.w),
                                     pack_bf16x2(w * x1.x, w * x1.y), pack_bf16x2(w * x1.z, w * x1.w));
          bf16* op = EPI == kTcSlotStore ? p.ys + (int64_t)dr * p.ldy + f : p.out + (int64_t)dr * p.ldo + f;
          st_global_v4_hint(op, v, pol);
        }
      }
      __syncwarp();
    }
  }
}

// tmT_r / tmT_s: token rows (dispatched rows of x for gate/up, of H for down;
// box 64 x kTokBox), routed and shared expert K; tmW_r / tmW_s: the same with
// kTokBoxWide-row boxes; tmB_*: gate (64-row boxes) or down (128-row boxes)
// weights, tmC_*: up weights (64-row boxes).  Launched as 2-CTA clusters.
template <bool DUAL, int STAGES, int EPI>
__global__ void __launch_bounds__(PairTCfg<DUAL, STAGES>::THREADS, 1)
    k_gemm_pairt(const __grid_constant__ CUtensorMap tmT_r, const __grid_constant__ CUtensorMap tmT_s,
                 const __grid_constant__ CUtensorMap tmW_r, const __grid_constant__ CUtensorMap tmW_s,
                 const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
                 const __grid_constant__ CUtensorMap tmC_r, const __grid_constant__ CUtensorMap tmC_s,
                 TcGemmArgs p) {
  using Cfg = PairTCfg<DUAL, STAGES>;
  constexpr int BN = Cfg::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::RING_BYTES);  // used on rank 0
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;  // rank 0: both CTAs' epilogues are done with the accumulator
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem + Cfg::RING_BYTES + Cfg::BAR_BYTES);
  int32_t* s_offs = s_pre + 514;
  float* xbuf = reinterpret_cast<float*>(smem + Cfg::EPI_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const unsigned tcode = kStatusTimeoutBase | (kKernGemmTc << 8) | 0x40u;
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
    prefetch_tmap(&tmT_r);
    prefetch_tmap(&tmT_s);
    prefetch_tmap(&tmW_r);
    prefetch_tmap(&tmW_s);
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
  // the tile schedule comes from earlier kernels in the stream (see k_gemm_pair)
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

  if (warp == 0 || warp == Cfg::PRODUCER2_WARP) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producers (both ranks, own tiles only)
      // producer `which` takes the K blocks whose running index over the
      // pair's tiles is `which` modulo 2 (ring stages of one parity): a single
      // issuing thread completes a TMA box only every few hundred ns
      const unsigned which = warp == 0 ? 0u : 1u;
      const uint64_t pol_keep = policy_evict_last(), pol_stream = policy_evict_first();
      const uint32_t full0 = mapa_rank(full, 0);
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      unsigned g = 0;  // running K-block index
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const TileInfo t = decode_tile<BN, kPairTRows>(p, s_pre, s_offs, tile);
        const PairTShape s = pairt_shape(t);
        const bool sh = t.g == p.E;
        const LoadPolicy lp = load_policy(t, pol_keep, pol_stream);
        const CUtensorMap* tok = s.boxes == 1 && s.box_rows == kTokBoxWide ? (sh ? &tmW_s : &tmW_r)
                                                                             : (sh ? &tmT_s : &tmT_r);
        const CUtensorMap* wb = sh ? &tmB_s : &tmB_r;
        const CUtensorMap* wc = sh ? &tmC_s : &tmC_r;
        const int trow = (int)t.row0 + (int)rank * s.nh;  // this CTA's first token row
        const int wrow = t.n0 + (int)rank * (DUAL ? 64 : 128);
        const uint32_t tx = 2u * (uint32_t)(Cfg::A_BYTES + s.boxes * s.box_rows * kBK * 2);
        for (int kb = t.kb0; kb < t.kb1; ++kb, ++g) {
          if ((g & 1u) != which) continue;
          stage = (int)(g % STAGES);
          phase = (g / STAGES) & 1u;
          if (!mbar_wait_cluster(empty + stage, phase ^ 1, abort_flag, p.status, tcode | 1)) {
            ok = false;
            break;
          }
          const uint32_t land = full0 + stage * 8;  // rank 0's full[stage]
          uint8_t* sa = smem + stage * Cfg::STAGE_BYTES;
          uint8_t* sb = sa + Cfg::A_BYTES;
          if (rank == 0) mbar_arrive_expect_tx(full + stage, tx);
          if (DUAL) {
            if (sh) {
              tma_load_2d_pair(sa, wb, land, kb * kBK, wrow, lp.w);
              tma_load_2d_pair(sa + Cfg::A_BYTES / 2, wc, land, kb * kBK, wrow, lp.w);
            } else {
              tma_load_3d_pair(sa, wb, land, kb * kBK, wrow, t.g, lp.w);
              tma_load_3d_pair(sa + Cfg::A_BYTES / 2, wc, land, kb * kBK, wrow, t.g, lp.w);
            }
          } else {
            if (sh) tma_load_2d_pair(sa, wb, land, kb * kBK, wrow, lp.w);
            else tma_load_3d_pair(sa, wb, land, kb * kBK, wrow, t.g, lp.w);
          }
          for (int b = 0; b < s.boxes; ++b)
            tma_load_2d_pair(sb + b * s.box_rows * kBK * 2, tok, land, kb * kBK, trow + b * s.box_rows, lp.a);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
        }
      }
      // copies in flight must land before the CTA exits (see k_gemm_pair)
      if (*abort_flag && rank == 0)
        for (int s = 0; s < STAGES; ++s)
          if (issued >> s & 1u) drain_wait(full + s, last_par >> s & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------ MMA issuer (rank 0)
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const TileInfo t = decode_tile<BN, kPairTRows>(p, s_pre, s_offs, tile);
        const PairTShape s = pairt_shape(t);
        const uint32_t idesc = idesc_bf16(256, s.n);
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
    // ------------------------------------------------ epilogue (both ranks, own 128 weight rows)
    const int eg = (warp - 2) / 4;
    const int q = warp & 3;
    const int partner = q >= 2 ? warp + 2 : warp - 2;     // same eg, lane quarter q ^ 2
    const int bar = 1 + (q & 1) + 2 * eg;                  // one named barrier per warp pair
    static_assert(Cfg::EPI_SCRATCH == kEpiScratchBytes, "epilogue scratch");
    float* mine = xbuf + (warp - 2) * (kEpiScratchBytes / 4);
    const float* theirs = xbuf + (partner - 2) * (kEpiScratchBytes / 4);
    const uint32_t tempty0 = mapa_rank(tempty, 0);
    const uint64_t pol = p.out_keep ? policy_evict_last() : policy_evict_first();
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total; tile += npairs) {
      const TileInfo t = decode_tile<BN, kPairTRows>(p, s_pre, s_offs, tile);
      const PairTShape s = pairt_shape(t);
      int dst[kMaxChunksPerWarp];
      float wt[kMaxChunksPerWarp];
      if (EPI != kTcSwiGLU) pairt_rows_prefetch<EPI>(p, t, s, eg, lane, dst, wt);
      // both warps of a SwiGLU pair see the same outcome: a phase, once
      // complete, stays visible until both have arrived on tempty
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(tfull + acc, acc_phase, abort_flag, p.status, tcode | 4)))
        break;  // the warp stops as one: its TMEM loads are warp-collective
      tc_fence_after();
      const uint32_t tb = tmem_base + acc * Cfg::ACC_COLS + ((uint32_t)(q * 32) << 16);
      if (EPI == kTcSwiGLU)
        pairt_epilogue_swiglu(p, t, s, tb, rank, q, eg, mine, theirs, bar, lane, pol);
      else
        pairt_epilogue_rows<EPI>(p, t, s, tb, rank, q, eg, lane, dst, wt, mine, pol);
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
