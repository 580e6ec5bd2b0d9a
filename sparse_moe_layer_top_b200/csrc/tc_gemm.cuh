// tc_gemm.cuh -- tensor-core (tcgen05) GEMM kernel for sm_100a, shared by the
// router and the two expert projections.
//
// Grouped GEMM (row-tiled form).  For every group g (expert g, or g == E the
// shared expert) with rows r0 .. r0+rows-1 of the activation matrix A:
//     D[r, n] = sum_c A[r, c] * B_g[n, c],  n < N_g,  c < K_g,
// with B_g K-major (the weights' own out x in layout).  One persistent CTA per
// SM walks a tile list (group, 128-row block, BN-column block, K split); the
// list comes from a device-built prefix sum over groups, or -- in the
// single-group mode the router uses -- from the kernel's arguments.  Tiles of
// one column block of a group are adjacent, so the CTAs that share a weight
// tile run together and the second read of it comes from L2.
//
// Warp roles (6 warps):
//   warp 0      TMA producer: A tile 128 x 64 and B tile(s) BN x 64 per stage,
//               128-byte swizzled, into a STAGES-deep shared-memory ring;
//   warp 1      TMEM owner and MMA issuer: tcgen05.mma M=128, N=BN, K=16,
//               fp32 accumulators in TMEM, double-buffered across tiles;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator rows (warp w reads TMEM
//               lanes 32*(w%4) ..), then one of
//                 SwiGLU    H[r, n] = SiLU(gate) * up -> bf16      (DUAL: two B)
//                 SlotStore Y[dst(r), n] = w(r) * D -> bf16: the routing weight
//                           applied and the row put back in (token, slot) order
//                 Store     out[r, n] = D -> bf16
//                 Logits    part[split][r, n] = D (+ nothing) -> fp32
// Rows of a tile past the end of its group are computed and discarded; rows
// never mix in a GEMM, so those rows cannot disturb the kept ones.
//
// E4M3 weights (FP8 = true, 10 warps): the TMA brings the raw 1-byte weight
// tile (64 bytes per row, unswizzled) into the upper half of the stage's bf16
// B buffer; warps 6..9 read it, multiply by the tile's 128 x 128 block scale,
// write bf16 in the 128-byte-swizzled layout the MMA expects, fence the async
// proxy and release the stage to the MMA warp.  The MMA itself stays bf16.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kBM = 128;
constexpr int kBK = 64;  // 64 bf16 = one 128-byte swizzle row

enum { kTcSwiGLU = 0, kTcSlotStore = 1, kTcStore = 2, kTcLogits = 3 };

struct TcGemmArgs {
  const int32_t* offs;    // [E+2] group row starts (grouped mode)
  const int32_t* prefix;  // [E+2] tile prefix of this schedule (grouped mode)
  int E;
  int N_r, N_s, K_r, K_s;
  int64_t rows_cap;       // rows of the activation/output buffers; no row at or past it is written
  // single-group mode (single_rows >= 0): one group of single_rows rows that
  // uses the "shared" maps, split along K into ksplit parts
  int single_rows, single_tiles, ksplit, kb_per_split;
  bf16* H;                // SwiGLU output [rows, ldh]
  int64_t ldh;
  bf16* ys;               // SlotStore output [T*(k+1), ldy]
  int64_t ldy;
  const int32_t* row_dst; // SlotStore: destination row of each dispatched row
  const float* row_w;     // SlotStore: routing weight of each dispatched row
  bf16* out;              // Store output [rows, ldo]
  int64_t ldo;
  float* part;            // Logits output [ksplit][rows, ldp]
  int64_t ldp, part_stride;
  // E4M3 weights: fp32 scales per 128 x 128 block, [E][N/128][K/128] routed,
  // [N/128][K/128] shared; B = gate (or the single operand), C = up
  const float *sc_b_r, *sc_b_s, *sc_c_r, *sc_c_s;
  unsigned* status;
};

struct TileInfo {
  int g, rows, m0, n0, kb0, kb1, N, split;
  int64_t row0;
};

// s_pre / s_offs: the schedule's tile prefix and group offsets, cached in
// shared memory at kernel start (grouped mode).
template <int BN>
__device__ __forceinline__ TileInfo decode_tile(const TcGemmArgs& p, const int32_t* s_pre, const int32_t* s_offs,
                                                int tile) {
  TileInfo t;
  if (p.single_rows >= 0) {
    t.g = p.E;
    t.rows = p.single_rows;
    const int mtc = (t.rows + kBM - 1) / kBM, ntc = (p.N_s + BN - 1) / BN;
    t.split = tile / (mtc * ntc);
    const int local = tile - t.split * mtc * ntc;
    t.m0 = (local % mtc) * kBM;
    t.n0 = (local / mtc) * BN;
    t.row0 = t.m0;
    t.N = p.N_s;
    const int kbt = (p.K_s + kBK - 1) / kBK;
    t.kb0 = t.split * p.kb_per_split;
    t.kb1 = min(kbt, t.kb0 + p.kb_per_split);
    return t;
  }
  {
    int lo = 0, hi = p.E + 1;  // s_pre[lo] <= tile < s_pre[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_pre[mid] <= tile) lo = mid; else hi = mid;
    }
    t.g = lo;
  }
  const int r0 = s_offs[t.g];
  t.rows = s_offs[t.g + 1] - r0;
  const int mtc = (t.rows + kBM - 1) / kBM;
  const int local = tile - s_pre[t.g];
  const int mb = local % mtc, nb = local / mtc;
  t.m0 = mb * kBM;
  t.row0 = (int64_t)r0 + t.m0;
  t.n0 = nb * BN;
  const bool sh = t.g == p.E;
  t.N = sh ? p.N_s : p.N_r;
  t.kb0 = 0;
  t.kb1 = ((sh ? p.K_s : p.K_r) + kBK - 1) / kBK;
  t.split = 0;
  return t;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Wait (bounded, ignoring the abort flag) for a TMA copy already issued.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) break;
}

template <int BN, bool DUAL, int STAGES>
struct TcGemmCfg {
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES * (DUAL ? 2 : 1);
  static constexpr int ACC_COLS = DUAL ? 2 * BN : BN;
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  static constexpr int BAR_BYTES = (3 * STAGES + 5) * 8 + 16;
  static constexpr int SCHED_INTS = 2 * (512 + 2);  // tile prefix + group offsets, E <= 512
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + SCHED_INTS * 4;
  static_assert(TMEM_COLS == 64 || TMEM_COLS == 128 || TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM columns");
  static_assert(BN % 16 == 0 && BN >= 16 && (DUAL ? 2 * BN : BN) <= 256, "UMMA N for M=128");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Named barrier 1 among the 128 converter threads.
__device__ __forceinline__ void conv_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Barrier 1 with an AND over the converters' flags: all of them see the same answer.
__device__ __forceinline__ bool conv_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}
// Generic-proxy shared-memory writes made visible to the async proxy (tensor core).
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Four E4M3 codes (one 32-bit word, element 0 in the low byte) times a scale -> four bf16.
__device__ __forceinline__ uint2 e4m3x4_scaled_bf16(uint32_t w, float sc) {
  const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xffffu), __NV_E4M3);
  const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w >> 16), __NV_E4M3);
  const float2 a = __half22float2(__half2(lo));
  const float2 b = __half22float2(__half2(hi));
  uint2 r;
  r.x = pack_bf16x2(a.x * sc, a.y * sc);
  r.y = pack_bf16x2(b.x * sc, b.y * sc);
  return r;
}

template <int BN, bool DUAL, int STAGES, int EPI, bool FP8 = false>
__global__ void __launch_bounds__(FP8 ? 320 : 192, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
              const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
              const __grid_constant__ CUtensorMap tmC_r, const __grid_constant__ CUtensorMap tmC_s, TcGemmArgs p) {
  using Cfg = TcGemmCfg<BN, DUAL, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* full8 = drain + 1;  // FP8: TMA landed (A + raw weights); `full` then means converted
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full8 + STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem + STAGES * Cfg::STAGE_BYTES + Cfg::BAR_BYTES);
  int32_t* s_offs = s_pre + 514;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned tcode = kStatusTimeoutBase | (kKernGemmTc << 8);
  if (p.single_rows < 0)
    for (int i = threadIdx.x; i < p.E + 2; i += blockDim.x) {
      s_pre[i] = __ldg(p.prefix + i);
      s_offs[i] = __ldg(p.offs + i);
    }

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, FP8 ? 128 : 1);
      mbar_init(empty + s, 1);
      mbar_init(full8 + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, 4);
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
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = p.single_rows >= 0 ? p.single_tiles : s_pre[p.E + 1];

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const TileInfo t = decode_tile<BN>(p, s_pre, s_offs, tile);
        const bool sh = t.g == p.E;
        bool ok = true;
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1, abort_flag, p.status, tcode | 1)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * Cfg::STAGE_BYTES;
          uint8_t* sb = sa + Cfg::A_BYTES;
          uint64_t* land = (FP8 ? full8 : full) + stage;
          // FP8: raw 1-byte rows packed in the upper half of the bf16 B buffer
          constexpr int NB = DUAL ? 2 * BN : BN;
          uint8_t* sbw = FP8 ? sb + NB * 64 : sb;
          uint8_t* scw = FP8 ? sbw + BN * 64 : sb + Cfg::B_BYTES;
          mbar_arrive_expect_tx(land, FP8 ? Cfg::A_BYTES + NB * 64 : Cfg::STAGE_BYTES);
          tma_load_2d(sa, sh ? &tmA_s : &tmA_r, land, kb * kBK, (int)t.row0, pol_a);
          if (sh) tma_load_2d(sbw, &tmB_s, land, kb * kBK, t.n0, pol_w);
          else tma_load_3d(sbw, &tmB_r, land, kb * kBK, t.n0, t.g, pol_w);
          if (DUAL) {
            if (sh) tma_load_2d(scw, &tmC_s, land, kb * kBK, t.n0, pol_w);
            else tma_load_3d(scw, &tmC_r, land, kb * kBK, t.n0, t.g, pol_w);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag)  // copies in flight must land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if (issued >> s & 1u) drain_wait((FP8 ? full8 : full) + s, last_par >> s & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      // DUAL: the gate and up tiles sit back to back in shared memory, so one
      // MMA of N = 2*BN fills both accumulators (gate at d0, up at d0 + BN) and
      // reads the A tile once instead of twice.
      constexpr uint32_t idesc = idesc_bf16(kBM, DUAL ? 2 * BN : BN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileInfo t = decode_tile<BN>(p, s_pre, s_offs, tile);
        if (!mbar_wait(tempty + acc, acc_phase ^ 1, abort_flag, p.status, tcode | 2)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * Cfg::ACC_COLS;
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(full + stage, phase, abort_flag, p.status, tcode | 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(sa + kk * 32);
            const uint32_t accum = (kb != t.kb0 || kk != 0);
            umma_f16(d0, ad, sdesc_sw128(sb + kk * 32), idesc, accum);
          }
          umma_commit(empty + stage);
          if (++stage == STAGES) {
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
      // every MMA issued must finish before TMEM is released
      umma_commit(drain);
      drain_wait(drain, 0);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileInfo t = decode_tile<BN>(p, s_pre, s_offs, tile);
      if (!mbar_wait(tfull + acc, acc_phase, abort_flag, p.status, tcode | 4)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + acc * Cfg::ACC_COLS + ((uint32_t)(q * 32) << 16);
      const int64_t grow = t.row0 + row;
      const bool valid = t.m0 + row < t.rows && grow < p.rows_cap;
      if (EPI == kTcSwiGLU) {
        bf16* dst = p.H + grow * p.ldh;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(tb + c * 32, g);
          tmem_ld32(tb + BN + c * 32, u);
          tmem_wait_regs(g);
          tmem_wait_regs(u);
          if (valid) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int n = t.n0 + c * 32 + v * 8;
              if (n < t.N) {
                uint4 o;
                uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float g0 = __uint_as_float(g[v * 8 + 2 * e]), g1 = __uint_as_float(g[v * 8 + 2 * e + 1]);
                  const float u0 = __uint_as_float(u[v * 8 + 2 * e]), u1 = __uint_as_float(u[v * 8 + 2 * e + 1]);
                  ow[e] = pack_bf16x2(silu_f32(g0) * u0, silu_f32(g1) * u1);
                }
                *reinterpret_cast<uint4*>(dst + n) = o;
              }
            }
          }
        }
      } else if (EPI == kTcSlotStore) {
        int64_t dr = 0;
        float w = 0.f;
        if (valid) {
          dr = __ldg(p.row_dst + grow);
          w = __ldg(p.row_w + grow);
        }
        bf16* dst = p.ys + dr * p.ldy;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t a[32];
          tmem_ld32(tb + c * 32, a);
          tmem_wait_regs(a);
          if (valid && dr >= 0) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int n = t.n0 + c * 32 + v * 8;
              if (n < t.N) {
                uint4 o;
                uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  ow[e] = pack_bf16x2(w * __uint_as_float(a[v * 8 + 2 * e]), w * __uint_as_float(a[v * 8 + 2 * e + 1]));
                *reinterpret_cast<uint4*>(dst + n) = o;
              }
            }
          }
        }
      } else if (EPI == kTcLogits) {
        float* dst = p.part + (int64_t)t.split * p.part_stride + grow * p.ldp;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t a[32];
          tmem_ld32(tb + c * 32, a);
          tmem_wait_regs(a);
          if (valid) {
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const int n = t.n0 + c * 32 + v * 4;
              if (n < t.N)
                *reinterpret_cast<float4*>(dst + n) =
                    make_float4(__uint_as_float(a[4 * v]), __uint_as_float(a[4 * v + 1]),
                                __uint_as_float(a[4 * v + 2]), __uint_as_float(a[4 * v + 3]));
            }
          }
        }
      } else {
        bf16* dst = p.out + grow * p.ldo;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t a[32];
          tmem_ld32(tb + c * 32, a);
          tmem_wait_regs(a);
          if (valid) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int n = t.n0 + c * 32 + v * 8;
              if (n < t.N) {
                uint4 o;
                uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  ow[e] = pack_bf16x2(__uint_as_float(a[v * 8 + 2 * e]), __uint_as_float(a[v * 8 + 2 * e + 1]));
                *reinterpret_cast<uint4*>(dst + n) = o;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + acc);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  } else if (FP8) {
    // ------------------------------------------------ E4M3 -> bf16 converters (warps 6..9)
    constexpr int NB = DUAL ? 2 * BN : BN;  // bf16 rows of a B stage: gate rows, then up rows
    static_assert(!FP8 || NB == 256, "converter mapping: two rows per thread");
    const int ct = threadIdx.x - 192;
    int stage = 0;
    uint32_t phase = 0;
    bool stop = false;
    for (int tile = blockIdx.x; tile < total && !stop; tile += gridDim.x) {
      const TileInfo t = decode_tile<BN>(p, s_pre, s_offs, tile);
      const bool sh = t.g == p.E;
      const int kb128 = ((sh ? p.K_s : p.K_r) + 127) / 128, nb128 = (t.N + 127) / 128;
      const int64_t eoff = (int64_t)t.g * nb128 * kb128;
      const float* s1 = sh ? p.sc_b_s : p.sc_b_r + eoff;
      const float* s2 = DUAL ? (sh ? p.sc_c_s : p.sc_c_r + eoff) : s1;
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        const bool ok = mbar_wait(full8 + stage, phase, abort_flag, p.status, tcode | 5);
        if (!conv_all(ok)) {
          stop = true;
          break;
        }
        uint8_t* sb = smem + stage * Cfg::STAGE_BYTES + Cfg::A_BYTES;
        const uint8_t* raw = sb + NB * 64;
        uint4 q[2][4];
        float sc[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = ct + 128 * h;
          const uint4* src = reinterpret_cast<const uint4*>(raw + r * 64);
#pragma unroll
          for (int v = 0; v < 4; ++v) q[h][v] = src[v];
          const bool up = DUAL && r >= BN;
          const int n = t.n0 + (up ? r - BN : r);
          sc[h] = n < t.N ? __ldg((up ? s2 : s1) + (n / 128) * kb128 + (kb * kBK) / 128) : 0.f;
        }
        conv_sync();  // every raw byte read before any bf16 byte overwrites it
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = ct + 128 * h;
          uint8_t* dst = sb + r * 128;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint2 a = e4m3x4_scaled_bf16(q[h][v].x, sc[h]);
            const uint2 b = e4m3x4_scaled_bf16(q[h][v].y, sc[h]);
            const uint2 c = e4m3x4_scaled_bf16(q[h][v].z, sc[h]);
            const uint2 d = e4m3x4_scaled_bf16(q[h][v].w, sc[h]);
            *reinterpret_cast<uint4*>(dst + (((2 * v) ^ (r & 7)) << 4)) = make_uint4(a.x, a.y, b.x, b.y);
            *reinterpret_cast<uint4*>(dst + (((2 * v + 1) ^ (r & 7)) << 4)) = make_uint4(c.x, c.y, d.x, d.y);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(full + stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
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
