// common.cuh -- element types, conversions and small device helpers shared by
// the kernels of libmoe.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace moe {

using bf16 = __nv_bfloat16;
using fp8 = __nv_fp8_storage_t;  // raw E4M3 code

constexpr int kMaxK = 16;  // largest k (experts per token) the kernels support

// Device status codes: high byte = which check, low bits = where.
enum : unsigned {
  kStatusBadExpertId = 0x06000001u,  // a routing id outside [0, E)
  kStatusBadCount = 0x06000002u,     // expert parallelism: a negative or short row count
  kStatusTimeoutBase = 0x07000000u,  // | (kernel id << 8) | wait site
  kStatusBoundsBase = 0x08000000u,   // bounds-checking build: | index site (kSite*)
};
enum : unsigned { kKernRouterTc = 1, kKernGemmTc = 2, kKernGemmSwap = 3 };

// Index sites the bounds-checking build (-DMOE_CHECKS) verifies: the row a
// pair is dispatched to, the rows the dispatch copies into, the token row a
// gathering GEMM reads, the (token, slot) row a down-GEMM epilogue stores, and
// the dispatched row moe_combine reads for a pair (a caller's input there).
enum : unsigned {
  kSiteDispatchRow = 1,
  kSiteCopyRow = 2,
  kSiteGatherToken = 3,
  kSiteSlotRow = 4,
  kSiteCombineRow = 5,
};

// True when 0 <= i < cap.  In the bounds-checking build an index outside that
// range records kStatusBoundsBase | site in the device status word (the first
// fault wins) and the caller skips the access; the normal build assumes the
// index is in range and the check compiles away.
__device__ __forceinline__ bool in_range(int64_t i, int64_t cap, unsigned* status, unsigned site) {
#ifdef MOE_CHECKS
  if (i >= 0 && i < cap) return true;
  if (status) atomicCAS(status, 0u, kStatusBoundsBase | site);
  return false;
#else
  (void)i;
  (void)cap;
  (void)status;
  (void)site;
  return true;
#endif
}

// Programmatic dependent launch.  Each kernel calls pdl_begin() before it
// touches what the previous kernel in the stream wrote (or overwrites what that
// kernel may still read).  A kernel releases its dependents only as its blocks
// exit (the implicit trigger; an explicit early trigger measured slower), so
// the next kernel's launch and set-up overlap this kernel's tail.  A no-op for
// a kernel launched without the programmatic-serialisation attribute.
__device__ __forceinline__ void pdl_begin() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void from_f32(float v, float* dst) { *dst = v; }
__device__ __forceinline__ void from_f32(float v, bf16* dst) { *dst = __float2bfloat16_rn(v); }

// E4M3 code -> float through the hardware conversion.
__device__ __forceinline__ float e4m3_to_f32(uint8_t q) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(q), __NV_E4M3);
  return __half2float(__half(h));
}

__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + __expf(-z)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__host__ __device__ __forceinline__ int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Locate the group whose tile range holds `tile`: prefix[g] <= tile < prefix[g+1].
__device__ __forceinline__ int find_group(const int32_t* prefix, int ngroups, int tile) {
  int lo = 0, hi = ngroups;  // invariant prefix[lo] <= tile < prefix[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (__ldg(prefix + mid) <= tile) lo = mid; else hi = mid;
  }
  return lo;
}

// One GEMM's tile schedule over the E+1 groups (group E = shared expert):
// tiles of group g = m_tiles(rows_g) * ceil(N_g / bn), with
// m_tiles = ceil(rows / bm) for the row-tiled kernels, and 0 or 1 for the
// weight-row (swap) kernels whose N covers every row of a group.
// Tiles of a grouped GEMM: ceil(rows / bm) x ceil(n / bn) per group (one
// row tile per group when swap).  With small_rows > 0 (the split form) the
// groups of at most small_rows rows are counted in a prefix of their own, with
// tiles of bm_small x bn_small (0: bm, bn): the large groups run on CTA pairs
// and the small ones in weight-row form, each kernel walking its own prefix.
struct Schedule {
  int bm, bn, n_routed, n_shared, swap, small_rows, bm_small, bn_small;
};

__host__ __device__ __forceinline__ bool sched_small(const Schedule& s, int rows) {
  return s.small_rows > 0 && rows > 0 && rows <= s.small_rows;
}

__device__ __forceinline__ int sched_tiles(const Schedule& s, int g, int E, int rows) {
  int n = g < E ? s.n_routed : s.n_shared;
  if (rows <= 0 || n <= 0) return 0;
  const bool small = sched_small(s, rows);
  const int bm = small && s.bm_small > 0 ? s.bm_small : s.bm;
  const int bn = small && s.bn_small > 0 ? s.bn_small : s.bn;
  int mt = s.swap ? 1 : (int)cdiv(rows, bm);
  return mt * (int)cdiv(n, bn);
}

}  // namespace moe
