// simt.cuh -- fp32-FMA kernels: the router with top-k, the grouped expert
// GEMMs and the combine.  These carry fp32 problems (where TF32 tensor cores
// could not meet a 1e-5 relative error) and any shape the tensor-core kernels
// do not take.  All accumulate in fp32.
#pragma once
#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------- grouped GEMM
// C[r, n] = sum_c A[r, c] * B_g[n, c] over the rows r of group g (rows
// offs[g] .. offs[g+1]-1 of A) and n < N_g, for every group g (g == E: the
// shared expert).  64 x 64 tiles, 16-deep K steps, 256 threads x (4 x 4)
// outputs; a persistent grid walks the device-built tile prefix.
enum { kEpiSwiGLU = 0, kEpiSlotStore = 1, kEpiStore = 2 };

template <typename TW>
struct WeightSet {
  const TW* routed;       // [E, N_r, K_r]
  const TW* shared;       // [N_s, K_s]
  const float* sc_routed; // E4M3 only: [E][N_r/128][K_r/128]
  const float* sc_shared; // E4M3 only: [N_s/128][K_s/128]
};

template <typename TA, typename TW>
struct SimtGemmArgs {
  const TA* A;            // [rows, lda]
  int64_t lda;
  const int32_t* offs;    // [E+2]
  const int32_t* prefix;  // [E+2] tile prefix (bm = bn = 64)
  int E;
  int64_t rows_cap;       // rows of the activation/output buffers; no row at or past it is touched
  int N_r, N_s, K_r, K_s;
  WeightSet<TW> b1, b2;   // b2: the up projection of the SwiGLU epilogue
  TA* H;                  // kEpiSwiGLU: [rows, ldh]
  int64_t ldh;
  TA* ys;                 // kEpiSlotStore: [T*(k+1), ldy], row_w-weighted, (token, slot) order
  int64_t ldy;
  int64_t ys_rows;        // rows of ys (checked in the bounds-checking build)
  unsigned* status;
  const int32_t* row_dst;
  const float* row_w;
  TA* out;                // kEpiStore: [rows, ldo]
  int64_t ldo;
};

template <typename TW>
__device__ __forceinline__ float load_w(const TW* w, int64_t idx) { return to_f32(w[idx]); }
template <>
__device__ __forceinline__ float load_w<uint8_t>(const uint8_t* w, int64_t idx) { return e4m3_to_f32(w[idx]); }

template <typename TW>
__device__ __forceinline__ float weight_at(const WeightSet<TW>& ws, int g, int E, int N, int K, int n, int c) {
  const TW* base = g < E ? ws.routed + (int64_t)g * N * K : ws.shared;
  float v = load_w<TW>(base, (int64_t)n * K + c);
  if (sizeof(TW) == 1) {
    int kb = (K + 127) / 128;
    const float* s = g < E ? ws.sc_routed + (int64_t)g * ((N + 127) / 128) * kb : ws.sc_shared;
    v *= __ldg(s + (n / 128) * kb + c / 128);
  }
  return v;
}

template <typename TA, typename TW, int EPI>
__global__ void __launch_bounds__(256) k_gemm_simt(SimtGemmArgs<TA, TW> p) {
  pdl_begin();  // after the previous kernel in the stream (programmatic launch)
  constexpr bool kDual = EPI == kEpiSwiGLU;
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  __shared__ float Cs[kDual ? 16 : 1][64 + 4];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int total = __ldg(p.prefix + p.E + 1);
  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    const int g = find_group(p.prefix, p.E + 1, tile);
    const int rows = __ldg(p.offs + g + 1) - __ldg(p.offs + g);
    const int64_t r0 = __ldg(p.offs + g);
    const int N = g < p.E ? p.N_r : p.N_s, K = g < p.E ? p.K_r : p.K_s;
    const int ntn = (N + 63) / 64;
    const int local = tile - __ldg(p.prefix + g);
    const int mt = local % ((rows + 63) / 64), nt = local / ((rows + 63) / 64);
    float acc[4][4] = {}, acc2[4][4] = {};
    (void)ntn;
    for (int c0 = 0; c0 < K; c0 += 16) {
      {  // each thread stages 4 elements of each operand tile
        int rr = tid >> 2, cc = (tid & 3) * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          int m = mt * 64 + rr, c = c0 + cc + q;
          As[cc + q][rr] = (m < rows && c < K && r0 + m >= 0 && r0 + m < p.rows_cap) ? to_f32(p.A[(r0 + m) * p.lda + c]) : 0.f;
          int n = nt * 64 + rr;
          bool okb = n < N && c < K;
          Bs[cc + q][rr] = okb ? weight_at(p.b1, g, p.E, N, K, n, c) : 0.f;
          if (kDual) Cs[cc + q][rr] = okb ? weight_at(p.b2, g, p.E, N, K, n, c) : 0.f;
        }
      }
      __syncthreads();
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float a[4], b[4], b2[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[i] = As[c][ty * 4 + i];
          b[i] = Bs[c][tx * 4 + i];
          if (kDual) b2[i] = Cs[c][tx * 4 + i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            if (kDual) acc2[i][j] = fmaf(a[i], b2[j], acc2[i][j]);
          }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int m = mt * 64 + ty * 4 + i;
      int64_t r = r0 + m;
      if (m >= rows || r < 0 || r >= p.rows_cap) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int n = nt * 64 + tx * 4 + j;
        if (n >= N) continue;
        if (EPI == kEpiSwiGLU) {
          from_f32(silu_f32(acc[i][j]) * acc2[i][j], p.H + r * p.ldh + n);
        } else if (EPI == kEpiSlotStore) {
          int64_t dr = __ldg(p.row_dst + r);
          if (dr >= 0 && in_range(dr, p.ys_rows, p.status, kSiteSlotRow))
            from_f32(__ldg(p.row_w + r) * acc[i][j], p.ys + dr * p.ldy + n);
        } else {
          from_f32(acc[i][j], p.out + r * p.ldo + n);
        }
      }
    }
  }
}

// ---------------------------------------------------------------- combine
// y[t] = sum_j topk_w[t,j] * y_perm[pos[t,j]] + y_perm[offs[E] + t] (shared),
// one block per token, fp32 sums.
template <typename TA>
__global__ void __launch_bounds__(256) k_combine(const TA* __restrict__ yp, const int32_t* __restrict__ pos,
                                                 const float* __restrict__ tw, const int32_t* __restrict__ offs,
                                                 int E, int k, int d, int64_t T, TA* __restrict__ y,
                                                 int64_t rows, unsigned* status) {
  pdl_begin();  // after the previous kernel in the stream (programmatic launch)
  const int64_t t = blockIdx.x;
  const int64_t rs = offs[E], re = offs[E + 1];
  const bool shared = re > rs && in_range(rs + t, rows, status, kSiteCombineRow);
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < k; ++j) {
      int r = __ldg(pos + t * k + j);
      if (r >= 0 && in_range(r, rows, status, kSiteCombineRow))
        acc = fmaf(__ldg(tw + t * k + j), to_f32(yp[(int64_t)r * d + c]), acc);
    }
    if (shared) acc += to_f32(yp[(rs + t) * d + c]);
    from_f32(acc, y + t * d + c);
  }
}

// y[t] = sum over the token's k+1 slots of ys[t*(k+1) + j] (routed slots with
// a dropped pair are skipped; slot k is the shared expert).  The slots already
// carry their routing weights; the sum runs in fp32 in slot order, so the
// result does not depend on scheduling.  One block per token, 8 elements per
// thread and step.
template <typename TA>
__global__ void __launch_bounds__(256) k_slot_sum(const TA* __restrict__ ys, const int32_t* __restrict__ pos, int k,
                                                  int has_shared, int d, TA* __restrict__ y) {
  pdl_begin();  // after the previous kernel in the stream (programmatic launch)
  const int64_t t = blockIdx.x;
  const TA* src = ys + t * (int64_t)(k + 1) * d;
  unsigned ok = 0;
  for (int j = 0; j < k; ++j) ok |= (__ldg(pos + t * k + j) >= 0 ? 1u : 0u) << j;
  if (has_shared) ok |= 1u << k;
  for (int c = threadIdx.x * 8; c < d; c += blockDim.x * 8) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (sizeof(TA) == 2) {
      // slot rows are read in batches of up to 9 (k = 8: all of them) issued
      // before the batch's first addition; the additions keep slot order
      constexpr int B = 9;
      for (int j0 = 0; j0 <= k; j0 += B) {
        uint4 v[B];
#pragma unroll
        for (int i = 0; i < B; ++i) {
          const int j = j0 + i;
          if (j <= k && (ok >> j & 1u)) v[i] = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)j * d + c));
        }
#pragma unroll
        for (int i = 0; i < B; ++i) {
          const int j = j0 + i;
          if (j <= k && (ok >> j & 1u)) {
            const bf16* h = reinterpret_cast<const bf16*>(&v[i]);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] += to_f32(h[e]);
          }
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      *reinterpret_cast<uint4*>(y + t * d + c) = o;
    } else {
      for (int j = 0; j <= k; ++j) {
        if (!(ok >> j & 1u)) continue;
        const TA* row = src + (int64_t)j * d + c;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += to_f32(row[e]);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) from_f32(acc[e], y + t * d + c + e);
    }
  }
}

}  // namespace moe
