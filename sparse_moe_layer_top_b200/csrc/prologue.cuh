// prologue.cuh -- the block's neighbours on its input (both optional):
//
//   zero-centred RMSNorm   x_n = x / sqrt(mean_j x_j^2 + eps) * (1 + gamma)
//       (Qwen3-Next story page: a "zero-centred" RMSNorm whose parameters start
//        at zero, so the applied scale is 1 + gamma; Architecture page, config
//        key rms_norm_eps = 1e-6), stored in the activation type: the router
//        and the experts then read x_n as the block's input;
//   shared-expert gate     g = sigmoid(x_n . w_sg), the weight of the shared
//       expert's row (not on the pages; an option, off by default).
//
// One warp per token; sums in fp32; the gate uses the stored (rounded) x_n.
#pragma once
#include "common.cuh"

namespace moe {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Eight consecutive values of a row (d % 8 == 0), as fp32.
__device__ __forceinline__ void load8(const bf16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const bf16* h = reinterpret_cast<const bf16*>(&u);
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = __bfloat162float(h[e]);
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}
// Round eight values to the activation type, store them, and return the
// rounded values.
__device__ __forceinline__ void store8(bf16* p, float (&v)[8]) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = u;
  const bf16* h = reinterpret_cast<const bf16*>(&u);
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = __bfloat162float(h[e]);
}
__device__ __forceinline__ void store8(float* p, float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// gamma != NULL: x_out = RMSNorm(x); gate_w != NULL: gate_out[t] = sigmoid(x_n . gate_w)
// (x_n = x without a norm).
template <typename TA>
__global__ void __launch_bounds__(256) k_prologue(const TA* __restrict__ x, const TA* __restrict__ gamma, float eps,
                                                  const TA* __restrict__ gate_w, int64_t T, int d,
                                                  TA* __restrict__ x_out, float* __restrict__ gate_out) {
  pdl_begin();  // after the previous kernel in the stream (programmatic launch)
  const int lane = threadIdx.x & 31;
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  const TA* xr = x + t * d;
  float r = 1.f;
  if (gamma) {
    float ss = 0.f;
    for (int j = lane * 8; j < d; j += 256) {
      float v[8];
      load8(xr + j, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
    }
    ss = warp_sum(ss);
    r = 1.0f / sqrtf(ss / (float)d + eps);
  }
  float z = 0.f;
  for (int j = lane * 8; j < d; j += 256) {
    float v[8];
    load8(xr + j, v);
    if (gamma) {
      float g[8];
      load8(gamma + j, g);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = v[e] * r * (1.0f + g[e]);
      store8(x_out + t * d + j, v);
    }
    if (gate_w) {
      float w[8];
      load8(gate_w + j, w);
#pragma unroll
      for (int e = 0; e < 8; ++e) z = fmaf(v[e], w[e], z);
    }
  }
  if (gate_w) {
    z = warp_sum(z);
    if (lane == 0) gate_out[t] = 1.0f / (1.0f + expf(-z));
  }
}

}  // namespace moe
