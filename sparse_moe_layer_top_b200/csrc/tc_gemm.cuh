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
// Warp roles (10 warps):
//   warp 0      TMA producer: A tile 128 x 64 and B tile(s) BN x 64 per stage,
//               128-byte swizzled, into a STAGES-deep shared-memory ring;
//   warp 1      TMEM owner and MMA issuer: tcgen05.mma M=128, N=BN, K=16,
//               fp32 accumulators in TMEM, double-buffered across tiles;
//   warps 2..9  epilogue, two warps per TMEM lane quarter (warp w reads lanes
//               32*(w%4) ..; the pair splits the columns): tcgen05.ld of the
//               accumulator rows, then one of
//                 SwiGLU    H[r, n] = SiLU(gate) * up -> bf16      (DUAL: two B)
//                 SlotStore Y[dst(r), n] = w(r) * D -> bf16: the routing weight
//                           applied and the row put back in (token, slot) order
//                 Store     out[r, n] = D -> bf16
//                 Logits    part[split][r, n] = D (+ nothing) -> fp32
//               (the router that selects its top k in the epilogue is the
//               K-split kernel of router_kc.cuh)
//   warps 10..13 (GATHER only) fetch the A rows straight from the token
//               matrix by row index (cp.async, 128-byte swizzle written by
//               hand): the gate/up GEMM of the fused forward needs no
//               dispatched copy of its activation rows.
// Rows of a tile past the end of its group are computed and discarded; rows
// never mix in a GEMM, so those rows cannot disturb the kept ones.
//
// E4M3 weights (FP8 = true, 15 warps): warp 0 streams raw 1-byte weight
// tiles (64 bytes per row, unswizzled) into a ring of their own, deeper than
// the stage ring so that more weight bytes are in flight, and prefetches the
// matching A tile into L2; warp 14 loads the A tiles into the stage ring;
// warps 6..13 -- one thread per weight row -- multiply the raw tile by its
// 128 x 128 block scale, write bf16 in the 128-byte-swizzled layout the MMA
// expects, fence the async proxy and release the stage to the MMA warp.  The
// MMA itself stays bf16.
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
  int out_keep;           // epilogue stores (H, slot rows, out): 1 L2 evict-last, 0 evict-first
  int panel;              // grouped mode: column blocks per panel of the tile order (decode_tile)
  int swap_small;         // grouped bf16 SwiGLU / SlotStore / Store: tiles of at most kSwapRows rows swap roles
  // single-group mode (single_rows >= 0): one group of single_rows rows that
  // uses the "shared" maps, split along K into ksplit parts
  int single_rows, single_tiles, ksplit, kb_per_split;
  bf16* H;                // SwiGLU output [rows, ldh]
  int64_t ldh;
  bf16* ys;               // SlotStore output [T*(k+1), ldy]
  int64_t ldy;
  int64_t ys_rows;        // SlotStore: rows of ys (checked in the bounds-checking build)
  const int32_t* row_dst; // SlotStore: destination row of each dispatched row
  const float* row_w;     // SlotStore: routing weight of each dispatched row
  bf16* out;              // Store output [rows, ldo]
  int64_t ldo;
  float* part;            // Logits output [ksplit][rows, ldp]
  int64_t ldp, part_stride;
  // the router's top-k selection (router_kc.cuh): topk_ids / topk_w [rows,
  // topk] and the 128-row chunk histograms counts[rows / 128][N_s] (may be
  // NULL; zeroed before the launch); bias [N_s] fp32 (may be NULL) is added to
  // the logits
  int topk;
  int32_t* ids;
  float* tw;
  const float* bias;
  int32_t* counts;
  // Tile order (bf16 kernels): NULL = CTA c takes tiles c, c + grid, ...;
  // else a counter (zeroed by whoever wrote `prefix`) from which a CTA claims
  // each tile after its first, so CTAs that draw cheap tiles draw more.
  int* sched;
  // GATHER: A row r is x[row_tok[r]] (row stride ldx elements), gathered by
  // the kernel instead of loaded from the dispatched-row matrix
  const bf16* gx;
  const int32_t* row_tok;
  int64_t ldx;
  int64_t gx_rows;        // rows of the token matrix (checked in the bounds-checking build)
  // E4M3 weights: fp32 scales per 128 x 128 block, [E][N/128][K/128] routed,
  // [N/128][K/128] shared; B = gate (or the single operand), C = up
  const float *sc_b_r, *sc_b_s, *sc_c_r, *sc_c_s;
  unsigned* status;
};

struct TileInfo {
  int g, rows, m0, n0, kb0, kb1, N, split;
  int64_t row0;
  bool rowmajor;  // the group's weight blocks serve several row blocks (see decode_tile)
  int swap_n;     // 0, or the MMA N of a tile run with swapped roles (see decode_tile)
};

// A tile with at most kSwapRows rows of its group (the groups of a few rows a
// skewed batch gives most experts, and the last rows of larger groups) runs
// with the MMA's roles swapped on the same shared-memory stage: the weight
// rows are the M = 128 operand and the tile's activation rows the N operand,
// N = its rows rounded up to 16, so the tensor core does not compute 128 rows
// for a handful.  The accumulator then holds one weight row (output feature)
// per TMEM lane and one token per column, and the epilogue writes it
// transposed.  Which tiles swap depends only on the row counts, so results
// stay reproducible.
constexpr int kSwapRows = 64;

// L2 hints of a tile's loads.  In column-block-major order (and in a group of
// one row tile) a weight block serves the row tiles running beside it and is
// done (evict-first), while the activation tiles come back for the next column
// block (evict-last).  In panels of several column blocks the other way round:
// an activation tile serves the panel's column blocks back to back, the
// panel's weight blocks come back for every row block.
struct LoadPolicy {
  uint64_t w, a;
};
__device__ __forceinline__ LoadPolicy load_policy(const TileInfo& t, uint64_t keep, uint64_t stream) {
  return t.rowmajor ? LoadPolicy{keep, stream} : LoadPolicy{stream, keep};
}

// s_pre / s_offs: the schedule's tile prefix and group offsets, cached in
// shared memory at kernel start (grouped mode).
template <int BN, int BM = kBM>
__device__ __forceinline__ TileInfo decode_tile(const TcGemmArgs& p, const int32_t* s_pre, const int32_t* s_offs,
                                                int tile) {
  TileInfo t;
  if (p.single_rows >= 0) {
    t.g = p.E;
    t.rows = p.single_rows;
    const int mtc = (t.rows + BM - 1) / BM, ntc = (p.N_s + BN - 1) / BN;
    t.split = tile / (mtc * ntc);
    const int local = tile - t.split * mtc * ntc;
    t.m0 = (local % mtc) * BM;
    t.n0 = (local / mtc) * BN;
    t.row0 = t.m0;
    t.N = p.N_s;
    const int kbt = (p.K_s + kBK - 1) / kBK;
    t.kb0 = t.split * p.kb_per_split;
    t.kb1 = min(kbt, t.kb0 + p.kb_per_split);
    t.rowmajor = false;
    t.swap_n = 0;
    return t;
  }
  const int32_t* pre = s_pre;
  {
    int lo = 0, hi = p.E + 1;  // pre[lo] <= tile < pre[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= tile) lo = mid; else hi = mid;
    }
    t.g = lo;
  }
  const int r0 = s_offs[t.g];
  t.rows = s_offs[t.g + 1] - r0;
  const bool sh = t.g == p.E;
  t.N = sh ? p.N_s : p.N_r;
  const int mtc = (t.rows + BM - 1) / BM, ntc = (t.N + BN - 1) / BN;
  const int local = tile - pre[t.g];
  // Order of a group's tiles: panels of p.panel column blocks, each swept row
  // block by row block (the panel's column blocks adjacent).  The panel's
  // weight blocks (about 32 MB) stay in L2 while the activation tiles stream
  // past, each read from HBM once per panel and shared by the CTAs that run
  // its column blocks together.  Pure column-block-major order re-reads a large
  // group's activation rows for every column block, pure row-block-major its
  // whole weight slice for every row block, and for data that all SMs read
  // B200's L2 holds about half its 126 MB (one copy per die): at the prefill
  // shape a Zipf-hot expert has 134 MB of rows and 64 MB of gate/up weights.
  const int P = min(max(p.panel, 1), ntc);
  const int pan = local / (mtc * P);
  const int p0 = pan * P, cw = min(P, ntc - p0);
  const int i = local - pan * mtc * P;
  const int mb = i / cw, nb = p0 + i % cw;
  t.rowmajor = P > 1 && mtc > 1;  // weight blocks reused across row blocks
  t.m0 = mb * BM;
  t.row0 = (int64_t)r0 + t.m0;
  t.n0 = nb * BN;
  const int here = min(BM, t.rows - t.m0);
  t.swap_n = p.swap_small && here <= kSwapRows ? (here + 15) & ~15 : 0;
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
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitLimitCycles) break;
}

template <int BN, bool DUAL, int STAGES, bool FP8 = false, bool GATHER = false>
struct TcGemmCfg {
  static_assert(!(FP8 && GATHER), "the gathered A path is bf16 only");
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int NB = DUAL ? 2 * BN : BN;          // B rows per stage (gate rows, then up rows)
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES * (DUAL ? 2 : 1);
  // FP8: a separate, deeper ring of raw E4M3 weight tiles (64 bytes per row)
  static constexpr int RAW_BYTES = FP8 ? NB * kBK : 0;
  static constexpr int RAW_STAGES = FP8 ? 6 : 0;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES + RAW_STAGES * RAW_BYTES;
  // FP8: + one converter thread per B row, + one warp issuing the A tiles
  // epilogue warps: 4 (one per TMEM lane quarter) with E4M3 weights, else 8
  // (two per quarter, splitting the accumulator columns) so stores drain faster
  static constexpr int EPI_WARPS = FP8 ? 4 : 8;
  static constexpr int GATHER_WARPS = GATHER ? 4 : 0;  // A rows gathered from x with cp.async
  static constexpr int THREADS = FP8 ? 192 + NB + 32 : 64 + 32 * (EPI_WARPS + GATHER_WARPS);
  static constexpr int ACC_COLS = DUAL ? 2 * BN : BN;
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  // + 4 + 4 barriers and 4 ints of the tile queue
  static constexpr int BAR_BYTES = (3 * STAGES + 2 * RAW_STAGES + 5 + 8) * 8 + 16 + 16;
  static constexpr int SCHED_INTS = 2 * (512 + 2);  // tile prefix + group offsets, E <= 512
  // epilogue staging: 32 rows x 64 bytes per epilogue warp
  static constexpr int EPI_OFF = (RING_BYTES + BAR_BYTES + SCHED_INTS * 4 + 127) / 128 * 128;
  static constexpr int SMEM_BYTES = 1024 + EPI_OFF + EPI_WARPS * 2048;
  static_assert(TMEM_COLS == 64 || TMEM_COLS == 128 || TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM columns");
  static_assert(BN % 16 == 0 && BN >= 16 && (DUAL ? 2 * BN : BN) <= 256, "UMMA N for M=128");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

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

// Epilogue store of a 32-row x 32-column bf16 block held one row per lane
// (w[16] = the row's 32 values as bf16 pairs) to rows rowp (per lane; NULL =
// skip the row) at byte offset colb, of which the first ncols columns exist:
// the block passes through the warp's 2 KB staging buffer (64 bytes per row,
// 16-byte chunks XOR-swizzled so neither the row-wise writes nor the
// column-wise reads conflict) and leaves as 8 rows x 64 contiguous bytes per
// store instruction instead of 32 rows x 16 bytes.  The stores carry an L2
// hint: evict-last when what the epilogue writes (H, the weighted slot rows)
// is small enough for the next kernel to find it in L2 (measured: down GEMM
// 138 -> 135 us at the 35B shape), evict-first when it is far larger than L2
// and would only push out the operands still in use (TcGemmArgs::out_keep).
__device__ __forceinline__ void st_global_evict_last(void* p, uint4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void store_rows_staged(uint8_t* stg, const uint32_t (&w)[16], char* rowp, int64_t colb,
                                                  int ncols, int lane, uint64_t pol) {
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(stg + lane * 64 + ((j ^ sw) << 4)) =
        make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  __syncwarp();
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int idx = it * 32 + lane;
    const int rr = idx >> 2, cc = idx & 3;
    char* rp = reinterpret_cast<char*>(__shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(rowp), rr));
    const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 64 + ((cc ^ ((rr >> 1) & 3)) << 4));
    if (rp && cc * 8 < ncols) st_global_evict_last(rp + colb + cc * 16, v, pol);
  }
  __syncwarp();
}

// The two 128-row halves of a converter stage (gate and up rows, or the two
// 128-row blocks of a 256-row weight tile) each read one row of 128 x 128
// block scales along K.  cur[] holds the scales of the current 128-wide K
// block, nxt[] the next one, loaded one block ahead.
struct ScaleStreams {
  const float* row[2];  // NULL: the half lies past the end of the weight matrix
  int kb128;
  float cur[2], nxt[2];
  __device__ __forceinline__ void start(int kb0) {
    const int j = kb0 / 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      cur[h] = row[h] ? __ldg(row[h] + j) : 0.f;
      nxt[h] = (row[h] && j + 1 < kb128) ? __ldg(row[h] + j + 1) : 0.f;
    }
  }
  // call before converting K-block kb (kb0 <= kb; K-blocks are 64 wide)
  __device__ __forceinline__ void at(int kb, int kb0) {
    if (kb > kb0 && (kb & 1) == 0) {
      const int j = kb / 2;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        cur[h] = nxt[h];
        nxt[h] = (row[h] && j + 1 < kb128) ? __ldg(row[h] + j + 1) : 0.f;
      }
    }
  }
};

// One converter thread's share of a stage: NB raw E4M3 rows of 64 bytes at
// `raw` become NB bf16 rows of 128 bytes at `dst`, 128-byte swizzled.  NB
// threads take four passes; in each, four threads share a row (one 16-byte
// chunk each), so a quarter warp reads 128 consecutive bytes.  Rows 0..127
// use scale stream 0, rows 128..255 stream 1.
template <int NB>
__device__ __forceinline__ void convert_e4m3_rows(const uint8_t* raw, uint8_t* dst, int ct, const float (&cur)[2]) {
  constexpr int RPP = NB / 4;  // rows per pass
  const int sub = ct & 3, rbase = ct >> 2;
  uint4 q[4];
#pragma unroll
  for (int ps = 0; ps < 4; ++ps) q[ps] = *reinterpret_cast<const uint4*>(raw + (rbase + RPP * ps) * kBK + sub * 16);
#pragma unroll
  for (int ps = 0; ps < 4; ++ps) {
    const int r = rbase + RPP * ps;
    const float sc = cur[r >= 128 ? 1 : 0];
    const uint2 a = e4m3x4_scaled_bf16(q[ps].x, sc);
    const uint2 b = e4m3x4_scaled_bf16(q[ps].y, sc);
    const uint2 c = e4m3x4_scaled_bf16(q[ps].z, sc);
    const uint2 d = e4m3x4_scaled_bf16(q[ps].w, sc);
    uint8_t* o = dst + r * 128;
    *reinterpret_cast<uint4*>(o + (((2 * sub) ^ (r & 7)) << 4)) = make_uint4(a.x, a.y, b.x, b.y);
    *reinterpret_cast<uint4*>(o + (((2 * sub + 1) ^ (r & 7)) << 4)) = make_uint4(c.x, c.y, d.x, d.y);
  }
}

// Scale rows of a converter stage for weight rows n0 .. n0+NB-1 of group g.
// dual: rows 0..127 gate (sb), 128..255 up (sc); else 1 or 2 row blocks of sb.
__device__ __forceinline__ void scale_rows(ScaleStreams& ss, bool dual, bool sh, int g, int n0, int N, int K,
                                           const float* sb_r, const float* sb_s, const float* sc_r,
                                           const float* sc_s, int nrows) {
  ss.kb128 = (K + 127) / 128;
  const int nb128 = (N + 127) / 128;
  const int64_t eoff = (int64_t)g * nb128 * ss.kb128;
  const float* base_b = sh ? sb_s : sb_r + eoff;
  if (dual) {
    const bool in = n0 < N;
    const float* base_c = sh ? sc_s : sc_r + eoff;
    ss.row[0] = in ? base_b + (int64_t)(n0 / 128) * ss.kb128 : nullptr;
    ss.row[1] = in ? base_c + (int64_t)(n0 / 128) * ss.kb128 : nullptr;
  } else {
    ss.row[0] = n0 < N ? base_b + (int64_t)(n0 / 128) * ss.kb128 : nullptr;
    ss.row[1] = (nrows > 128 && n0 + 128 < N) ? base_b + (int64_t)(n0 / 128 + 1) * ss.kb128 : nullptr;
  }
}

// Epilogue of one row-tiled tile for the SwiGLU / SlotStore / Store modes, as
// run by one warp: its 32 rows are the TMEM lanes addressed by `tb` (lane
// offset included) and row `row` of the tile is this thread's; it converts the
// 32-column chunks [c0, c1) and stores them through its 2 KB staging buffer.
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_rows(const TcGemmArgs& p, const TileInfo& t, uint32_t tb, int row, int c0,
                                              int c1, uint8_t* stg, int lane) {
  const int64_t grow = t.row0 + row;
  const bool valid = t.m0 + row < t.rows && grow < p.rows_cap;
  // outputs the next kernel will find in L2 are stored evict-last, larger ones evict-first
  const uint64_t pol = p.out_keep ? policy_evict_last() : policy_evict_first();
  // destination row of this lane (NULL: nothing to write) and its scale
  char* rowp = nullptr;
  float w = 1.f;
  if (valid) {
    if (EPI == kTcSwiGLU) {
      rowp = reinterpret_cast<char*>(p.H + grow * p.ldh);
    } else if (EPI == kTcSlotStore) {
      const int64_t dr = __ldg(p.row_dst + grow);
      w = __ldg(p.row_w + grow);
      if (dr >= 0 && in_range(dr, p.ys_rows, p.status, kSiteSlotRow))
        rowp = reinterpret_cast<char*>(p.ys + dr * p.ldy);
    } else {
      rowp = reinterpret_cast<char*>(p.out + grow * p.ldo);
    }
  }
#pragma unroll 1
  for (int c = c0; c < c1; ++c) {
    uint32_t a[32], u[32];
    tmem_ld32(tb + c * 32, a);
    if (EPI == kTcSwiGLU) tmem_ld32(tb + BN + c * 32, u);
    tmem_wait_regs(a);
    if (EPI == kTcSwiGLU) tmem_wait_regs(u);
    uint32_t o[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float x0 = __uint_as_float(a[2 * e]), x1 = __uint_as_float(a[2 * e + 1]);
      if (EPI == kTcSwiGLU)
        o[e] = pack_bf16x2(silu_f32(x0) * __uint_as_float(u[2 * e]), silu_f32(x1) * __uint_as_float(u[2 * e + 1]));
      else
        o[e] = pack_bf16x2(w * x0, w * x1);
    }
    const int n = t.n0 + c * 32;
    store_rows_staged(stg, o, rowp, (int64_t)n * 2, t.N - n, lane, pol);
  }
}

// Epilogue of a tile run with swapped roles (TileInfo::swap_n), as run by one
// epilogue warp of lane quarter q and column group eg (EG = 2): TMEM lane =
// weight row, column = the tile's token j.  SwiGLU: gate rows at columns
// [0, N), up rows at [BN, BN + N); warp eg takes tokens 32 eg ..; the lane's
// output feature is n0 + 32 q + lane.  SlotStore / Store: the two 128-row
// halves of the 256-row weight tile at columns [0, N) and [128, 128 + N);
// warp eg takes half eg, every token.  Each token's row is written 32
// features (64 bytes) per warp.
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_swapped(const TcGemmArgs& p, const TileInfo& t, uint32_t tb, int q, int eg,
                                                 int lane) {
  const int here = min(kBM, t.rows - t.m0);
  const uint64_t pol = p.out_keep ? policy_evict_last() : policy_evict_first();
  if (EPI == kTcSwiGLU) {
    const int j0 = eg * 32;
    if (j0 >= here) return;  // uniform over the warp
    uint32_t a[32], u[32];
    tmem_ld32(tb + j0, a);
    tmem_ld32(tb + BN + j0, u);
    tmem_wait_regs(a);
    tmem_wait_regs(u);
    const int n = t.n0 + q * 32 + lane;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int64_t grow = t.row0 + j0 + j;
      if (j0 + j < here && grow < p.rows_cap && n < t.N) {
        const float h = silu_f32(__uint_as_float(a[j])) * __uint_as_float(u[j]);
        asm volatile("st.global.L2::cache_hint.b16 [%0], %1, %2;" ::"l"(p.H + grow * p.ldh + n),
                     "h"(__bfloat16_as_ushort(__float2bfloat16_rn(h))), "l"(pol)
                     : "memory");
      }
    }
  } else {
    const int n = t.n0 + eg * 128 + q * 32 + lane;
#pragma unroll 1
    for (int j0 = 0; j0 < here; j0 += 32) {
      uint32_t a[32];
      tmem_ld32(tb + eg * 128 + j0, a);
      tmem_wait_regs(a);
      // lane j's token: its destination row and routing weight, then broadcast
      const int64_t gl = t.row0 + j0 + lane;
      const bool lin = j0 + lane < here && gl < p.rows_cap;
      int64_t dst = -1;
      float w = 1.f;
      if (lin) {
        if (EPI == kTcSlotStore) {
          dst = __ldg(p.row_dst + gl);
          w = __ldg(p.row_w + gl);
          if (dst >= 0 && !in_range(dst, p.ys_rows, p.status, kSiteSlotRow)) dst = -1;
        } else {
          dst = gl;
        }
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int64_t dr = __shfl_sync(0xffffffffu, dst, j);
        const float wj = __shfl_sync(0xffffffffu, w, j);
        if (dr >= 0 && n < t.N) {
          bf16* op = EPI == kTcSlotStore ? p.ys + dr * p.ldy + n : p.out + dr * p.ldo + n;
          asm volatile("st.global.L2::cache_hint.b16 [%0], %1, %2;" ::"l"(op),
                       "h"(__bfloat16_as_ushort(__float2bfloat16_rn(wj * __uint_as_float(a[j])))), "l"(pol)
                       : "memory");
        }
      }
    }
  }
}

// A CTA's tile sequence (bf16 kernels), handed from the producer thread to the
// other roles through a 4-slot ring in shared memory: the producer puts each
// tile (a value >= total ends the sequence); every consumer role takes them in
// order, one arrival per warp on `empty`.  Waits are bounded; on abort, take()
// returns -1.
struct TileQueue {
  int* id;
  uint64_t* full;
  uint64_t* empty;
  int slot;
  uint32_t phase;
  __device__ __forceinline__ TileQueue(int* i, uint64_t* f, uint64_t* e)
      : id(i), full(f), empty(e), slot(0), phase(0) {}
  __device__ __forceinline__ void advance() {
    if (++slot == 4) {
      slot = 0;
      phase ^= 1;
    }
  }
  // producer thread
  __device__ __forceinline__ bool put(int tile, volatile int* abort_flag, unsigned* status, unsigned where) {
    if (!mbar_wait(empty + slot, phase ^ 1, abort_flag, status, where)) return false;
    id[slot] = tile;
    mbar_arrive(full + slot);
    advance();
    return true;
  }
  // a whole warp (every lane gets the tile), or one thread (warp_wide false)
  __device__ __forceinline__ int take(bool warp_wide, int lane, volatile int* abort_flag, unsigned* status,
                                      unsigned where) {
    bool ok = mbar_wait(full + slot, phase, abort_flag, status, where);
    if (warp_wide) ok = __all_sync(0xffffffffu, ok);
    if (!ok) return -1;
    const int t = id[slot];
    if (warp_wide) __syncwarp();
    if (!warp_wide || lane == 0) mbar_arrive(empty + slot);
    advance();
    return t;
  }
};

template <int BN, bool DUAL, int STAGES, int EPI, bool FP8 = false, bool GATHER = false>
__global__ void __launch_bounds__(TcGemmCfg<BN, DUAL, STAGES, FP8, GATHER>::THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
              const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
              const __grid_constant__ CUtensorMap tmC_r, const __grid_constant__ CUtensorMap tmC_s, TcGemmArgs p) {
  using Cfg = TcGemmCfg<BN, DUAL, STAGES, FP8, GATHER>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* raw_ring = smem + STAGES * Cfg::STAGE_BYTES;       // FP8 only
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::RING_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* a_full = empty + STAGES;     // FP8: the stage's A tile has landed
  uint64_t* tfull = a_full + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* raw_full = drain + 1;        // FP8: raw weight tile landed
  uint64_t* raw_empty = raw_full + Cfg::RAW_STAGES;  // FP8: raw tile converted
  uint64_t* tq_full = raw_empty + Cfg::RAW_STAGES;  // tile queue (bf16 kernels)
  uint64_t* tq_empty = tq_full + 4;
  int* tq_id = reinterpret_cast<int*>(tq_empty + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tq_id + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_pre = reinterpret_cast<int32_t*>(smem + Cfg::RING_BYTES + Cfg::BAR_BYTES);
  int32_t* s_offs = s_pre + 514;
  uint8_t* epi_stage = smem + Cfg::EPI_OFF;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned tcode = kStatusTimeoutBase | (kKernGemmTc << 8);
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // FP8: one arrival per converter warp; GATHER: the B loads plus one per gather warp
      mbar_init(full + s, FP8 ? Cfg::NB / 32 : 1 + Cfg::GATHER_WARPS);
      mbar_init(empty + s, 1);
      mbar_init(a_full + s, 1);
    }
    for (int s = 0; s < Cfg::RAW_STAGES; ++s) {
      mbar_init(raw_full + s, 1);
      mbar_init(raw_empty + s, Cfg::NB / 32);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, Cfg::EPI_WARPS);
    }
    mbar_init(drain, 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(tq_full + q, 1);
      mbar_init(tq_empty + q, 1 + Cfg::EPI_WARPS + Cfg::GATHER_WARPS);  // MMA thread + each consumer warp
    }
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
  // the tile schedule comes from earlier kernels in the stream: read it once
  // they are done (barrier set-up, tensor-map prefetch and TMEM allocation above
  // overlap the previous kernel's tail under programmatic launch)
  pdl_begin();
  if (p.single_rows < 0)
    for (int i = threadIdx.x; i < p.E + 2; i += blockDim.x) {
      s_pre[i] = __ldg(p.prefix + i);
      s_offs[i] = __ldg(p.offs + i);
    }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = p.single_rows >= 0 ? p.single_tiles : s_pre[p.E + 1];

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      // bf16: A and B tiles into the stage ring.  FP8: raw weight tiles into
      // the raw ring, running ahead of the stage ring, plus an L2 prefetch of
      // the A tile that the A warp will load for the same K-block.
      const uint64_t pol_keep = policy_evict_last(), pol_stream = policy_evict_first();
      constexpr int RING = FP8 ? Cfg::RAW_STAGES : STAGES;
      uint64_t* land0 = FP8 ? raw_full : full;
      uint64_t* free0 = FP8 ? raw_empty : empty;
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      TileQueue tq(tq_id, tq_full, tq_empty);
      for (int tile = blockIdx.x;;) {
        if (!FP8 && !tq.put(min(tile, total), abort_flag, p.status, tcode | 11)) break;
        if (tile >= total) break;
        const TileInfo t = decode_tile<BN>(p, s_pre, s_offs, tile);
        const bool sh = t.g == p.E;
        const LoadPolicy lp = load_policy(t, pol_keep, pol_stream);
        const uint64_t pol_w = lp.w, pol_a = lp.a;
        bool ok = true;
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(free0 + stage, phase ^ 1, abort_flag, p.status, tcode | 1)) {
            ok = false;
            break;
          }
          uint64_t* land = land0 + stage;
          if (FP8) {
            uint8_t* sbw = raw_ring + stage * Cfg::RAW_BYTES;
            uint8_t* scw = sbw + BN * kBK;
            mbar_arrive_expect_tx(land, Cfg::RAW_BYTES);
            if (sh) tma_load_2d(sbw, &tmB_s, land, kb * kBK, t.n0, pol_w);
            else tma_load_3d(sbw, &tmB_r, land, kb * kBK, t.n0, t.g, pol_w);
            if (DUAL) {
              if (sh) tma_load_2d(scw, &tmC_s, land, kb * kBK, t.n0, pol_w);
              else tma_load_3d(scw, &tmC_r, land, kb * kBK, t.n0, t.g, pol_w);
            }
            tma_prefetch_2d(sh ? &tmA_s : &tmA_r, kb * kBK, (int)t.row0);
          } else {
            uint8_t* sa = smem + stage * Cfg::STAGE_BYTES;
            uint8_t* sb = sa + Cfg::A_BYTES;
            mbar_arrive_expect_tx(land, GATHER ? Cfg::STAGE_BYTES - Cfg::A_BYTES : Cfg::STAGE_BYTES);
            if (!GATHER) tma_load_2d(sa, sh ? &tmA_s : &tmA_r, land, kb * kBK, (int)t.row0, pol_a);
            if (sh) tma_load_2d(sb, &tmB_s, land, kb * kBK, t.n0, pol_w);
            else tma_load_3d(sb, &tmB_r, land, kb * kBK, t.n0, t.g, pol_w);
            if (DUAL) {
              uint8_t* sc = sb + Cfg::B_BYTES;
              if (sh) tma_load_2d(sc, &tmC_s, land, kb * kBK, t.n0, pol_w);
              else tma_load_3d(sc, &tmC_r, land, kb * kBK, t.n0, t.g, pol_w);
            }
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == RING) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tile = (!FP8 && p.sched) ? (int)gridDim.x + atomicAdd(p.sched, 1) : tile + (int)gridDim.x;
      }
      if (*abort_flag)  // copies in flight must land before the CTA exits
        for (int s = 0; s < RING; ++s)
          if (issued >> s & 1u) drain_wait(land0 + s, last_par >> s & 1u);
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
      TileQueue tq(tq_id, tq_full, tq_empty);
      for (int tile = FP8 ? (int)blockIdx.x : tq.take(false, lane, abort_flag, p.status, tcode | 12);
           tile >= 0 && tile < total && ok;
           tile = FP8 ? tile + (int)gridDim.x : tq.take(false, lane, abort_flag, p.status, tcode | 12)) {
        const TileInfo t = decode_tile<BN>(p, s_pre, s_offs, tile);
        if (!mbar_wait(tempty + acc, acc_phase ^ 1, abort_flag, p.status, tcode | 2)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * Cfg::ACC_COLS;
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if ((FP8 && !mbar_wait(a_full + stage, phase, abort_flag, p.status, tcode | 6)) ||
              !mbar_wait(full + stage, phase, abort_flag, p.status, tcode | 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + Cfg::A_BYTES;
          if (t.swap_n) {
            // swapped roles: 128 weight rows x the tile's first swap_n
            // activation rows; gate / up (or the two 128-row halves of the
            // weight tile) into columns [0, N) and [BN or 128, + N)
            const uint32_t idesc_s = idesc_bf16(kBM, t.swap_n);
            constexpr uint32_t half_off = DUAL ? Cfg::B_BYTES : 128 * 128;
            constexpr uint32_t col_off = DUAL ? BN : 128;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t xd = sdesc_sw128(sa + kk * 32);
              const uint32_t accum = (kb != t.kb0 || kk != 0);
              umma_f16(d0, sdesc_sw128(sb + kk * 32), xd, idesc_s, accum);
              if (DUAL || BN > 128) umma_f16(d0 + col_off, sdesc_sw128(sb + half_off + kk * 32), xd, idesc_s, accum);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t ad = sdesc_sw128(sa + kk * 32);
              const uint32_t accum = (kb != t.kb0 || kk != 0);
              umma_f16(d0, ad, sdesc_sw128(sb + kk * 32), idesc, accum);
            }
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
  } else if (warp < 2 + Cfg::EPI_WARPS) {
    // ------------------------------------------------ epilogue (warps 2 .. 2+EPI_WARPS-1)
    // warp w reads TMEM lanes 32*(w%4) ..; with 8 warps the two warps of a lane
    // quarter take the two halves of the tile's columns
    constexpr int EG = Cfg::EPI_WARPS / 4;
    const int eg = (warp - 2) / 4;
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    TileQueue tq(tq_id, tq_full, tq_empty);
    for (int tile = FP8 ? (int)blockIdx.x : tq.take(true, lane, abort_flag, p.status, tcode | 13);
         tile >= 0 && tile < total;
         tile = FP8 ? tile + (int)gridDim.x : tq.take(true, lane, abort_flag, p.status, tcode | 13)) {
      const TileInfo t = decode_tile<BN>(p, s_pre, s_offs, tile);
      if (!__all_sync(0xffffffffu, mbar_wait(tfull + acc, acc_phase, abort_flag, p.status, tcode | 4)))
        break;  // the warp stops as one: its TMEM loads are warp-collective
      tc_fence_after();
      const uint32_t tb = tmem_base + acc * Cfg::ACC_COLS + ((uint32_t)(q * 32) << 16);
      const int64_t grow = t.row0 + row;
      const bool valid = t.m0 + row < t.rows && grow < p.rows_cap;
      if (EPI == kTcSwiGLU || EPI == kTcSlotStore || EPI == kTcStore) {
        constexpr int CPW = (BN / 32) / EG;  // 32-column chunks per warp, contiguous
        if (t.swap_n)
          epilogue_swapped<BN, EPI>(p, t, tb, q, eg, lane);
        else
          epilogue_rows<BN, EPI>(p, t, tb, row, eg * CPW, (eg + 1) * CPW, epi_stage + (warp - 2) * 2048, lane);
      } else if (EPI == kTcLogits) {
        float* dst = p.part + (int64_t)t.split * p.part_stride + grow * p.ldp;
#pragma unroll 1
        for (int c = eg; c < BN / 32; c += EG) {
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
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + acc);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  } else if (GATHER) {
    // ------------------------------------------------ A rows gathered from x (warps 10..13)
    // Row r of a tile is x[row_tok[row0 + r]], zeros past the group or the
    // buffer (and past K): thread gt copies 16-byte chunk gt % 8 of rows
    // gt / 8 + RS i (RS = 4 * gather warps) into the 128-byte-swizzled A tile
    // with cp.async, so 8 lanes read one row's 128 contiguous bytes.  A stage
    // goes to the MMA warp (one arrival per gather warp on `full`, after the
    // warp's copies have landed and the async proxy has been fenced) once the
    // next stage's copies are issued (LAG = 1).  Holding stages longer ties up
    // ring slots that the weight loads need: releasing STAGES - 1 stages late
    // made the gate/up GEMM 30 % slower than 1 or 2 late (measured; 4 gather
    // warps beat 2 by about 1 %).
    constexpr int LAG = 1;
    // row stride and rows per thread
    constexpr int RS = 4 * (Cfg::GATHER_WARPS > 0 ? Cfg::GATHER_WARPS : 1), RPT = kBM / RS;
    const int gt = threadIdx.x - 32 * (2 + Cfg::EPI_WARPS);
    const int ch = gt & 7, rb = gt >> 3;
    const uint32_t sw = (uint32_t)(ch ^ (rb & 7)) << 4;  // rows rb + RS i share their row-in-atom
    const uint64_t pol_x = policy_evict_last();
    int stage = 0, issued = 0, arrived = 0;
    uint32_t phase = 0;
    bool stop = false;
    TileQueue tq(tq_id, tq_full, tq_empty);
    for (int tile = tq.take(true, lane, abort_flag, p.status, tcode | 14); tile >= 0 && tile < total && !stop;
         tile = tq.take(true, lane, abort_flag, p.status, tcode | 14)) {
      const TileInfo t = decode_tile<BN>(p, s_pre, s_offs, tile);
      const bf16* src[RPT];
      uint32_t live = 0;
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int r = rb + RS * i;
        const int64_t grow = t.row0 + r;
        const bool in = t.m0 + r < t.rows && grow < p.rows_cap;
        int64_t tok = in ? (int64_t)__ldg(p.row_tok + grow) : 0;
        const bool tin = !in || in_range(tok, p.gx_rows, p.status, kSiteGatherToken);
        if (!tin) tok = 0;  // (checking build) the row reads zeros instead
        src[i] = p.gx + tok * p.ldx + ch * 8;
        live |= (uint32_t)(in && tin) << i;
      }
      const int K = t.g == p.E ? p.K_s : p.K_r;
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(empty + stage, phase ^ 1, abort_flag, p.status, tcode | 10))) {
          stop = true;  // the warp stops as one
          break;
        }
        const uint32_t sa = smem_u32(smem + stage * Cfg::STAGE_BYTES) + sw;
        const uint32_t kin = kb * kBK + ch * 8 < K ? 0xffffu : 0u;
#pragma unroll
        for (int i = 0; i < RPT; ++i)
          cp_async_16(sa + (rb + RS * i) * 128, src[i] + kb * kBK, (live & kin) >> i & 1u ? 16u : 0u, pol_x);
        cp_async_commit();
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
        if (issued - arrived > LAG) {
          cp_async_wait<LAG>();
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(full + arrived % STAGES);
          ++arrived;
        }
      }
    }
    cp_async_wait<0>();  // every copy lands before the CTA can exit
    if (!stop) {
      fence_proxy_async_smem();
      __syncwarp();
      for (; arrived < issued; ++arrived)
        if (lane == 0) mbar_arrive(full + arrived % STAGES);
    }
  } else if (FP8 && warp < 6 + Cfg::NB / 32) {
    // ------------------------------------------------ E4M3 -> bf16 converters
    static_assert(!FP8 || Cfg::NB == 256, "converter mapping covers 256 rows");
    const int ct = threadIdx.x - 192;
    int stage = 0, rstage = 0;
    uint32_t phase = 0, rphase = 0;
    bool stop = false;
    for (int tile = blockIdx.x; tile < total && !stop; tile += gridDim.x) {
      const TileInfo t = decode_tile<BN>(p, s_pre, s_offs, tile);
      const bool sh = t.g == p.E;
      ScaleStreams ss;
      scale_rows(ss, DUAL, sh, t.g, t.n0, t.N, sh ? p.K_s : p.K_r, p.sc_b_r, p.sc_b_s, p.sc_c_r, p.sc_c_s,
                 Cfg::NB);
      ss.start(t.kb0);
      for (int kb = t.kb0; kb < t.kb1; ++kb) {
        ss.at(kb, t.kb0);
        const bool ok = mbar_wait(raw_full + rstage, rphase, abort_flag, p.status, tcode | 5) &&
                        mbar_wait(empty + stage, phase ^ 1, abort_flag, p.status, tcode | 7);
        if (!__all_sync(0xffffffffu, ok)) {  // the warp goes on, or stops, as one
          stop = true;
          break;
        }
        convert_e4m3_rows<Cfg::NB>(raw_ring + rstage * Cfg::RAW_BYTES,
                                   smem + stage * Cfg::STAGE_BYTES + Cfg::A_BYTES, ct, ss.cur);
        // The raw slot goes back to the TMA only now: its bytes have been
        // consumed, and the proxy fence orders these generic-proxy reads before
        // the async-proxy write that will refill the slot.
        fence_proxy_async_smem();
        __syncwarp();  // the warp's writes and proxy fences, then one arrival per warp
        if (lane == 0) {
          mbar_arrive(full + stage);
          mbar_arrive(raw_empty + rstage);
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
        if (++rstage == Cfg::RAW_STAGES) {
          rstage = 0;
          rphase ^= 1;
        }
      }
    }
  } else if (FP8) {
    // ------------------------------------------------ A tiles into the stage ring (FP8 mode)
    if (lane == 0) {
      const uint64_t pol_a = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileInfo t = decode_tile<BN>(p, s_pre, s_offs, tile);
        const bool sh = t.g == p.E;
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1, abort_flag, p.status, tcode | 8)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(a_full + stage, Cfg::A_BYTES);
          tma_load_2d(smem + stage * Cfg::STAGE_BYTES, sh ? &tmA_s : &tmA_r, a_full + stage, kb * kBK, (int)t.row0,
                      pol_a);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag)
        for (int s = 0; s < STAGES; ++s)
          if (issued >> s & 1u) drain_wait(a_full + s, last_par >> s & 1u);
    }
    __syncwarp();
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
