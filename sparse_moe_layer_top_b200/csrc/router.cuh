// router.cuh -- the router: logits over the E experts, softmax, top-k and
// renormalisation (Qwen3.6 explainer, router paragraphs: a small linear
// network scores every expert, a softmax top-k keeps the K best; the kept
// weights are renormalised to sum to one).
//
// bf16 problems: the logits come from the tensor-core GEMM kernel in its
// single-group mode, split along d into `nsplit` fp32 partial sums written to
// separate buffers; k_topk adds the partials in a fixed order (so routing is
// bit-for-bit reproducible), adds the bias and selects.  fp32 problems:
// k_router_simt computes each logit with fp32 FMAs and selects in one kernel.
// Selection: the k largest logits by repeated warp arg-max, equal values going
// to the lower expert index; weights = softmax over the kept logits, which is
// the full softmax renormalised over the kept experts.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kChunkTokens = 128;  // tokens per dispatch chunk (one k_topk / k_count block)

// Warp-wide selection over one token's logits l[] (lane owns experts lane + 32 i;
// NPL = 32-expert columns held, entries past E are -inf).  Each round takes the
// warp arg-max (a strict > scan inside the lane keeps its lowest expert, the
// shuffle tree prefers the lower expert on equal values) and sets the taken
// entry to -inf.  Lanes < k write the ids and weights; `hist` (may be NULL)
// counts the selected experts.
template <int NPL>
__device__ __forceinline__ void warp_select(float (&l)[NPL], int k, int64_t t, int32_t* ids, float* tw, int* hist) {
  const int lane = threadIdx.x & 31;
  float v0 = 0.f, den = 0.f, my_v = 0.f;
  int my_e = 0;
  for (int s = 0; s < k; ++s) {
    float bv = l[0];
    int be = lane;
#pragma unroll
    for (int i = 1; i < NPL; ++i)
      if (l[i] > bv) {
        bv = l[i];
        be = lane + 32 * i;
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (be == lane + 32 * i) l[i] = -INFINITY;
    if (s == 0) v0 = bv;
    den += __expf(bv - v0);
    if (lane == s) {  // lane s keeps selection s (k <= 16 < 32)
      my_v = bv;
      my_e = be;
    }
  }
  if (lane < k) {
    ids[t * k + lane] = my_e;
    tw[t * k + lane] = __expf(my_v - v0) / den;
    if (hist) atomicAdd(hist + my_e, 1);
  }
}

// fp32 path: one warp per token, logits by fp32 FMA.
template <typename TA, int NPL>
__global__ void __launch_bounds__(256) k_router_simt(const TA* __restrict__ x, const TA* __restrict__ wr,
                                                     const float* __restrict__ bias, int64_t T, int d, int E, int k,
                                                     int32_t* __restrict__ ids, float* __restrict__ tw) {
  pdl_begin();  // after the previous kernel in the stream (programmatic launch)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * 8 + warp;
  if (t >= T) return;
  const TA* xt = x + t * d;
  float l[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    float acc = -INFINITY;
    if (e < E) {
      const TA* w = wr + (int64_t)e * d;
      acc = 0.f;
      for (int j = 0; j < d; ++j) acc = fmaf(to_f32(xt[j]), to_f32(w[j]), acc);
      if (bias) acc += bias[e];
    }
    l[i] = acc;
  }
  warp_select<NPL>(l, k, t, ids, tw, nullptr);
}

// Top-k from split logits, one warp per token.  When `counts` is given
// (zeroed beforehand), the selected experts are also counted into the
// per-chunk histograms counts[(t / kChunkTokens) * E + e] for the dispatch.
template <int NPL>
__global__ void __launch_bounds__(256) k_topk(const float* __restrict__ part, int nsplit, int64_t split_stride,
                                              int64_t ldp, const float* __restrict__ bias, int64_t T, int E, int k,
                                              int32_t* __restrict__ ids, float* __restrict__ tw,
                                              int32_t* __restrict__ counts) {
  pdl_begin();  // after the previous kernel in the stream (programmatic launch)
  const int lane = threadIdx.x & 31;
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  float l[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) l[i] = (lane + 32 * i < E) ? (bias ? __ldg(bias + lane + 32 * i) : 0.f) : -INFINITY;
  const float* row = part + t * ldp;
#pragma unroll 4
  for (int s = 0; s < nsplit; ++s) {
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (lane + 32 * i < E) l[i] += __ldg(row + s * split_stride + lane + 32 * i);
  }
  warp_select<NPL>(l, k, t, ids, tw, counts ? counts + (t / kChunkTokens) * E : nullptr);
}

// Values per lane for E experts: the smallest of 4, 8, 16 with 32 * NPL >= E.
inline int select_npl(int E) { return E <= 128 ? 4 : E <= 256 ? 8 : 16; }

}  // namespace moe
