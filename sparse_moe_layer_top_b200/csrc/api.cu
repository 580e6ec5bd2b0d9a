// api.cu -- host side of libmoe.so: argument checks, workspace carving, TMA
// tensor-map encoding and the launch sequence of every entry point of moe.h.
// One translation unit: the kernels are included from the headers beside it.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/moe.h"
#include "common.cuh"
#include "ep.cuh"
#include "permute.cuh"
#include "prologue.cuh"
#include "router.cuh"
#include "simt.cuh"
#include "tc_gemm.cuh"
#include "tc_swap.cuh"
#include "tc_swap8.cuh"
#include "tc_pair.cuh"
#include "tc_pairt.cuh"
#include "router_kc.cuh"

using namespace moe;

// ============================================================== errors
static thread_local char g_err[512] = "no error";
static thread_local int g_launches = 0;
static thread_local int g_launches_pending = 0;
constexpr int kProfileCapacity = 4096;

static moe_status fail(moe_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return s;
}

#define CUDA_TRY(call)                                                                      \
  do {                                                                                      \
    cudaError_t e_ = (call);                                                                \
    if (e_ != cudaSuccess) return fail(MOE_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

// NVTX ranges on the host around every entry point and every stage of the
// fused forward, for nsys and ncu's NVTX filters (header-only NVTX 3: without
// a tool attached a range costs a branch).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// The profiling mode a thread starts in: MOE_PROFILE=1 (every launch) or 2
// (the tensor-core GEMMs) in the environment, else off (moe_profile_enable).
static int env_profile_mode() {
  static const int m = [] {
    const char* e = getenv("MOE_PROFILE");
    const int v = e ? atoi(e) : 0;
    return v == 1 || v == 2 ? v : 0;
  }();
  return m;
}

// Optional per-launch timing: when enabled, every kernel launch of the
// calling thread is bracketed by two CUDA events recorded on its stream.
struct LaunchEvent {
  const char* name;
  cudaEvent_t begin, end;
};
struct Profiler {
  bool on = env_profile_mode() != 0, pending = false;
  int mode = env_profile_mode();
  int used = 0;
  LaunchEvent ev[kProfileCapacity];
  int created = 0;
};
static thread_local Profiler g_prof;

// Mode 2 records only the tensor-core GEMM launches (names "gemm_tc_*").
static bool prof_wants(const char* name) {
  return g_prof.mode == 1 || (g_prof.mode == 2 && strncmp(name, "gemm_tc", 7) == 0);
}
static void prof_begin(const char* name, cudaStream_t st) {
  Profiler& P = g_prof;
  P.pending = false;
  if (!P.on || P.used >= kProfileCapacity || !prof_wants(name)) return;
  if (P.used == P.created) {
    if (cudaEventCreate(&P.ev[P.used].begin) != cudaSuccess) return;
    if (cudaEventCreate(&P.ev[P.used].end) != cudaSuccess) return;
    ++P.created;
  }
  cudaEventRecord(P.ev[P.used].begin, st);
  P.pending = true;
}
static void prof_end(const char* name, cudaStream_t st) {
  Profiler& P = g_prof;
  if (!P.on || !P.pending || P.used >= P.created) return;
  P.pending = false;
  P.ev[P.used].name = name;
  cudaEventRecord(P.ev[P.used].end, st);
  ++P.used;
}

#define PROF_BEGIN(name, st) prof_begin(name, st)
#define LAUNCH_CHECK(name, st)                                                               \
  do {                                                                                       \
    cudaError_t e_ = cudaGetLastError();                                                     \
    if (e_ != cudaSuccess) return fail(MOE_ERR_CUDA, "launch %s: %s", name, cudaGetErrorString(e_)); \
    prof_end(name, st);                                                                      \
    ++g_launches_pending;                                                                    \
  } while (0)

// Kernel launch.  Every launch of a library call after its first carries the
// programmatic-serialisation attribute: the kernel may be scheduled as the
// previous one's blocks exit, runs its set-up, and waits for it
// (griddepcontrol.wait) before touching its results -- every kernel of the
// library does.  The first launch of a call (whose predecessor may be the
// caller's own kernel) and the first after a memset go in plain stream order.
static thread_local bool g_pdl_next = false;
static void pdl_reset() { g_pdl_next = false; }

template <typename... KArgs, typename... Args>
static cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = g_pdl_next ? 1 : 0;
  g_pdl_next = true;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ============================================================== device state
// The device status word: kernels record a rejected input or a wait that gave
// up; moe_device_status() reads and clears it.
static __device__ unsigned g_status;

constexpr int kMaxDevices = 64;
struct DeviceInfo {
  bool ready = false;
  unsigned* status = nullptr;
  int sms = 0;
  int pair_ctas = 0;  // CTAs of the pair GEMMs: 2 x the 2-CTA clusters that fit at once
  int pairt_ctas = 0;  // the same for the token-N pair GEMMs
  bool attr_set = false;
};
static DeviceInfo g_dev[kMaxDevices];
static std::mutex g_dev_mu;
static int g_path = 0;

template <typename K>
static cudaError_t allow_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// GEMM instantiations used by the library.
using Gemm1Cfg = TcGemmCfg<128, true, 4>;
using Gemm1GCfg = TcGemmCfg<128, true, 4, false, true>;  // A rows gathered from the token matrix
using Gemm2Cfg = TcGemmCfg<256, false, 4>;
// the router that selects in its epilogue: 64-expert column tiles, 8 stages
constexpr int kFp8Stages = 2;
using Gemm1F8Cfg = TcGemmCfg<128, true, kFp8Stages, true>;
using Gemm2F8Cfg = TcGemmCfg<256, false, kFp8Stages, true>;
constexpr int kPairStages = 6;
using Pair1Cfg = PairCfg<128, true, kPairStages>;
using Pair2Cfg = PairCfg<256, false, kPairStages>;
constexpr int kPairTStages = 6;
static_assert(kPairTRows == kPairBM, "the token-N pair form shares the pair form's tile schedule");
using PairT1Cfg = PairTCfg<true, kPairTStages>;
using PairT2Cfg = PairTCfg<false, kPairTStages>;

// Launch a pair GEMM as 2-CTA clusters.
template <typename K>
static cudaError_t launch_pair(K kernel, int ctas, int threads, int smem, cudaStream_t st, const CUtensorMap& a0,
                               const CUtensorMap& a1, const CUtensorMap& b0, const CUtensorMap& b1,
                               const CUtensorMap& c0, const CUtensorMap& c1, const TcGemmArgs& args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = g_pdl_next ? 2 : 1;
  g_pdl_next = true;
  return cudaLaunchKernelEx(&cfg, kernel, a0, a1, b0, b1, c0, c1, args);
}

// Launch a token-N pair GEMM as 2-CTA clusters (eight tensor maps).
template <typename K>
static cudaError_t launch_pairt(K kernel, int ctas, int threads, int smem, cudaStream_t st, const CUtensorMap* m,
                                const TcGemmArgs& args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = g_pdl_next ? 2 : 1;
  g_pdl_next = true;
  return cudaLaunchKernelEx(&cfg, kernel, m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], args);
}

// Launch the K-split router as 4-CTA clusters.
template <typename K>
static cudaError_t launch_router_kc(K kernel, int ctas, cudaStream_t st, const CUtensorMap& x, const CUtensorMap& w,
                                    const TcGemmArgs& args, int npad) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3((unsigned)RouterKcCfg::THREADS);
  cfg.dynamicSmemBytes = (size_t)RouterKcCfg::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kRouterKcCtas;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = g_pdl_next ? 2 : 1;
  g_pdl_next = true;
  return cudaLaunchKernelEx(&cfg, kernel, x, w, args, npad);
}

static moe_status device_info(DeviceInfo** out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    void* p = nullptr;
    CUDA_TRY(cudaGetSymbolAddress(&p, g_status));
    d.status = static_cast<unsigned*>(p);
    CUDA_TRY(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    int major = 0, minor = 0;
    CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    CUDA_TRY(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    if (major != 10 || minor != 0)
      return fail(MOE_ERR_UNSUPPORTED, "libmoe is built for sm_100a; device %d is sm_%d%d", dev, major, minor);
    CUDA_TRY(allow_smem(k_gemm_tc<128, true, 4, kTcSwiGLU>, Gemm1Cfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_tc<128, true, 4, kTcSwiGLU, false, true>, Gemm1GCfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_tc<256, false, 4, kTcSlotStore>, Gemm2Cfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_tc<256, false, 4, kTcStore>, Gemm2Cfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_tc<256, false, 4, kTcLogits>, Gemm2Cfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_tc<128, true, kFp8Stages, kTcSwiGLU, true>, Gemm1F8Cfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_tc<256, false, kFp8Stages, kTcSlotStore, true>, Gemm2F8Cfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_tc<256, false, kFp8Stages, kTcStore, true>, Gemm2F8Cfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_swap<true, kTcSwiGLU>, SwapCfg<true>::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_swap<false, kTcSlotStore>, SwapCfg<false>::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_swap<false, kTcStore>, SwapCfg<false>::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_pair<128, true, kPairStages, kTcSwiGLU>, Pair1Cfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_pair<256, false, kPairStages, kTcSlotStore>, Pair2Cfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_pair<256, false, kPairStages, kTcStore>, Pair2Cfg::SMEM_BYTES));
    {
      // 2-CTA clusters of the larger pair kernel that fit on the device at once
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(d.sms & ~1));
      cfg.blockDim = dim3((unsigned)Pair2Cfg::THREADS);
      cfg.dynamicSmemBytes = (size_t)std::max(Pair1Cfg::SMEM_BYTES, Pair2Cfg::SMEM_BYTES);
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int clusters = 0;
      CUDA_TRY(cudaOccupancyMaxActiveClusters(&clusters, k_gemm_pair<256, false, kPairStages, kTcSlotStore>, &cfg));
      d.pair_ctas = 2 * std::max(1, std::min(clusters, d.sms / 2));
    }
    CUDA_TRY(allow_smem(k_router_kc<8>, RouterKcCfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_router_kc<16>, RouterKcCfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_pairt<true, kPairTStages, kTcSwiGLU>, PairT1Cfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_pairt<false, kPairTStages, kTcSlotStore>, PairT2Cfg::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_pairt<false, kPairTStages, kTcStore>, PairT2Cfg::SMEM_BYTES));
    {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(d.sms & ~1));
      cfg.blockDim = dim3((unsigned)PairT1Cfg::THREADS);
      cfg.dynamicSmemBytes = (size_t)std::max(PairT1Cfg::SMEM_BYTES, PairT2Cfg::SMEM_BYTES);
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int clusters = 0;
      CUDA_TRY(cudaOccupancyMaxActiveClusters(&clusters, k_gemm_pairt<true, kPairTStages, kTcSwiGLU>, &cfg));
      d.pairt_ctas = 2 * std::max(1, std::min(clusters, d.sms / 2));
    }
    CUDA_TRY(allow_smem(k_gemm_swap8<true, kTcSwiGLU>, Swap8Cfg<true>::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_swap8<true, kTcSlotStore>, Swap8Cfg<true>::SMEM_BYTES));
    CUDA_TRY(allow_smem(k_gemm_swap8<true, kTcStore>, Swap8Cfg<true>::SMEM_BYTES));
    d.ready = true;
  }
  *out = &d;
  return MOE_OK;
}

// ============================================================== tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static moe_status encode_fn(EncodeTiledFn* out) {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(err));
  *out = fn;
  return MOE_OK;
}

// Box {64 elements, box_rows} (x {1}); bf16 tiles are 128-byte swizzled for the
// MMA, 1-byte E4M3 tiles are loaded plain for the converter warps, or, `wide`,
// as 128-code rows with 128-byte swizzling (the TMEM-operand kernels).
// Out-of-range reads give zeros.
static moe_status map_tile(CUtensorMap* m, const void* base, bool bytes, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, uint32_t box_rows, bool wide = false) {
  EncodeTiledFn enc;
  moe_status s = encode_fn(&enc);
  if (s != MOE_OK) return s;
  cuuint64_t gd[3], gs[2];
  const bool swz = !bytes || wide;
  cuuint32_t box[3] = {(cuuint32_t)(wide ? kBK8 : kBK), box_rows, 1}, es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) gd[i] = dims[i] ? dims[i] : 1;
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = enc(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank,
                   const_cast<void*>(base), gd, gs, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) rank %d dims %llu x %llu", (int)r, rank,
                (unsigned long long)gd[0], (unsigned long long)gd[1]);
  return MOE_OK;
}
static moe_status map2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t stride_elems,
                        uint32_t box_rows, bool bytes = false, bool wide = false) {
  const uint64_t eb = bytes ? 1 : 2;
  uint64_t dims[2] = {inner, outer}, st[1] = {stride_elems * eb};
  return map_tile(m, base, bytes, 2, dims, st, box_rows, wide);
}
static moe_status map3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                        uint32_t box_rows, bool bytes = false, bool wide = false) {
  const uint64_t eb = bytes ? 1 : 2;
  uint64_t dims[3] = {inner, mid, outer}, st[2] = {inner * eb, inner * mid * eb};
  return map_tile(m, base, bytes, 3, dims, st, box_rows, wide);
}

// ============================================================== checks
static size_t esize(int dt) { return dt == MOE_F32 ? 4 : dt == MOE_BF16 ? 2 : 1; }
static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static moe_status check(const moe_problem* p) {
  if (!p) return fail(MOE_ERR_INVALID_ARG, "problem is NULL");
  if (p->T < 0) return fail(MOE_ERR_INVALID_ARG, "T = %lld < 0", (long long)p->T);
  if (p->d <= 0 || p->E <= 0 || p->k <= 0 || p->I <= 0 || p->I_s < 0)
    return fail(MOE_ERR_INVALID_ARG, "sizes must be positive (d=%d E=%d k=%d I=%d I_s=%d)", p->d, p->E, p->k, p->I,
                p->I_s);
  if (p->E > kMaxE) return fail(MOE_ERR_UNSUPPORTED, "E = %d > %d", p->E, kMaxE);
  if (p->k > p->E || p->k > kMaxK) return fail(MOE_ERR_INVALID_ARG, "k = %d must be <= min(E, %d)", p->k, kMaxK);
  if (p->act_dtype != MOE_F32 && p->act_dtype != MOE_BF16)
    return fail(MOE_ERR_INVALID_ARG, "activation type %d is not F32 or BF16", p->act_dtype);
  if (p->w_dtype != MOE_F32 && p->w_dtype != MOE_BF16 && p->w_dtype != MOE_FP8_E4M3_B128)
    return fail(MOE_ERR_INVALID_ARG, "weight type %d unknown", p->w_dtype);
  if (p->act_dtype == MOE_F32 && p->w_dtype != MOE_F32)
    return fail(MOE_ERR_UNSUPPORTED, "F32 activations need F32 weights");
  if (p->act_dtype == MOE_BF16 && p->w_dtype == MOE_F32)
    return fail(MOE_ERR_UNSUPPORTED, "BF16 activations take BF16 or FP8 weights");
  if (p->d % 8 || p->I % 8 || p->I_s % 8)
    return fail(MOE_ERR_ALIGNMENT, "d, I, I_s must be multiples of 8 (16-byte rows)");
  if (p->w_dtype == MOE_FP8_E4M3_B128 && (p->d % 128 || p->I % 128 || p->I_s % 128))
    return fail(MOE_ERR_INVALID_ARG, "FP8 block scales need d, I, I_s multiples of 128");
  if (p->T * (int64_t)(p->k + 1) >= (int64_t)1 << 31) return fail(MOE_ERR_UNSUPPORTED, "T*(k+1) >= 2^31");
  return MOE_OK;
}

static bool misaligned(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) != 0; }

#define NEED(ptr)                                                                              \
  do {                                                                                         \
    if (!(ptr)) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", #ptr);                          \
    if (misaligned(ptr)) return fail(MOE_ERR_ALIGNMENT, "%s is not 16-byte aligned", #ptr);    \
  } while (0)
#define MAYBE(ptr)                                                                             \
  do {                                                                                         \
    if ((ptr) && misaligned(ptr)) return fail(MOE_ERR_ALIGNMENT, "%s is not 16-byte aligned", #ptr); \
  } while (0)

// Tensor-core expert kernels: bf16 activations; bf16 or E4M3 weights.
static bool tc_shapes(const moe_problem& p) {
  return p.act_dtype == MOE_BF16 && (p.w_dtype == MOE_BF16 || p.w_dtype == MOE_FP8_E4M3_B128);
}

static moe_status choose(bool tc_possible, bool* use_tc) {
  if (g_path == 1) {
    *use_tc = false;
  } else if (g_path >= 2) {
    if (!tc_possible) return fail(MOE_ERR_UNSUPPORTED, "tensor-core path required but the types do not allow it");
    *use_tc = true;
  } else {
    *use_tc = tc_possible;
  }
  return MOE_OK;
}

// Expert GEMM form: 0 SIMT, 1 row-tiled tensor core, 2 weight-row (swap)
// tensor core, 3 row-tiled on CTA pairs, 4 split (CTA pairs for the groups of
// kSplitRows rows or more, weight-row tiles for the others, one launch each
// per projection; chosen with moe_set_path(5) only: on the Zipf prefill
// workload it measured 10.9 ms against 10.5-10.6 for the row-tiled form, whose
// interleaved tile order already runs the small groups' weight streaming
// beside the large groups' tensor work).  Automatic choice: the weight-row
// form when an expert sees at most one token chunk on average (T*k <= 64*E),
// where a 128-row activation tile would be mostly empty; the pair form (bf16
// weights) when experts average kPairRowsPerExpert rows or more, where its
// 256-row tiles waste little on group tails (measured: 12-15 % faster at 4096
// rows per expert, even at 1024, slower on prefill-sized Zipf-skewed groups);
// else the row-tiled form.
enum { kFormSimt = 0, kFormRows = 1, kFormSwap = 2, kFormPair = 3, kFormSplit = 4, kFormPairT = 5 };
constexpr int kPairRowsPerExpert = 2048;
constexpr int kSplitRows = 256;
static moe_status choose_form(const moe_problem& p, int* form) {
  bool tc;
  moe_status s = choose(tc_shapes(p), &tc);
  if (s != MOE_OK) return s;
  if (!tc) *form = kFormSimt;
  else if (g_path == 2) *form = kFormRows;
  else if (g_path == 3) *form = kFormSwap;
  else if (g_path == 4) *form = p.w_dtype == MOE_BF16 ? kFormPair : kFormRows;
  else if (g_path == 5) *form = p.w_dtype == MOE_BF16 ? kFormSplit : kFormRows;
  else if (g_path == 6) *form = p.w_dtype == MOE_BF16 ? kFormPairT : kFormRows;
  else if (p.T * (int64_t)p.k <= (int64_t)kNCH * p.E) *form = kFormSwap;
  else if (p.w_dtype == MOE_BF16 && p.T * (int64_t)p.k >= (int64_t)kPairRowsPerExpert * p.E) *form = kFormPair;
  else *form = kFormRows;
  return MOE_OK;
}

// ============================================================== workspace
// Router split along d: enough (row block, expert block, split) tiles to cover
// the GPU, each split at least 4 K-blocks deep.  A fixed target keeps the
// workspace size a pure function of the problem.
constexpr int kRouterBN = 256;
constexpr int kTargetTiles = 148;

// The router with the selection in its epilogue (128-token x 64-expert
// tiles, no K split, no logit partials; the column tiles of a row tile merge
// their candidate lists): for up to 256 experts and enough token tiles to
// spread over the GPU; otherwise the split-K logits and k_topk.
static_assert(kChunkTokens == kBM, "the fused router writes one histogram chunk per row tile");
static bool router_fused(const moe_problem& p) { return p.E <= kRouterBN && cdiv(p.T, kBM) >= 16; }

struct RouterSplit {
  int ksplit, kb_per, tiles;
  int64_t ldp;  // row stride of the logit partials (floats)
};
static RouterSplit router_split(const moe_problem& p) {
  RouterSplit r;
  const int kblocks = (int)cdiv(p.d, kBK);
  const int mn = (int)(cdiv(std::max<int64_t>(p.T, 1), kBM) * cdiv(p.E, kRouterBN));
  int ks = (int)std::min<int64_t>(cdiv(kTargetTiles, mn), std::max(1, kblocks / 4));
  ks = std::max(ks, 1);
  r.kb_per = (int)cdiv(kblocks, ks);
  r.ksplit = (int)cdiv(kblocks, r.kb_per);
  r.tiles = mn * r.ksplit;
  r.ldp = (int64_t)align_up(p.E, 32);
  return r;
}

// Router scratch: the split-K logit partials, or for the fused router the
// per-(row tile, lane quarter) counters followed by the candidate lists.
static size_t router_scratch_bytes(const moe_problem& p) {
  if (p.act_dtype != MOE_BF16) return 0;
  if (router_fused(p)) return 0;
  const RouterSplit rs = router_split(p);
  return (size_t)rs.ksplit * p.T * rs.ldp * 4;
}

struct Layout {
  size_t counts = 0, pre_a = 0, pre_b = 0, part = 0, ids = 0, tw = 0, offs = 0, row_tok = 0, row_w = 0, pos = 0,
         row_dst = 0, xp = 0, xn = 0, gate = 0, h = 0, total = 0;
};

static int64_t rows_total(const moe_problem& p) { return p.T * p.k + (p.I_s > 0 ? p.T : 0); }
static int64_t n_chunks(const moe_problem& p) { return std::max<int64_t>(1, cdiv(p.T, kChunkTokens)); }
static int64_t ldh_of(const moe_problem& p) { return std::max(p.I, p.I_s); }

// Workspace of moe_layer_forward (forward) or of the stage calls.  In the
// forward, the dispatched rows x_perm and the weighted (token, slot) rows of
// the down projection share one buffer: the gate/up GEMM has consumed the
// former before the down GEMM writes the latter.
static Layout layout(const moe_problem& p, bool forward) {
  Layout L;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t r = o;
    o += align_up(std::max<size_t>(bytes, 1), 256);
    return r;
  };
  const int64_t n = p.T * p.k, Rp = rows_total(p);
  const size_t ab = esize(p.act_dtype);
  // chunk histograms, then the fused router's row-tile counters (one memset clears both)
  L.counts = take(n_chunks(p) * p.E * 4);
  // tile prefix [E+2], the GEMM's tile-claim counter, the small groups' prefix [E+2]
  L.pre_a = take((2 * p.E + 5) * 4);
  L.pre_b = take((2 * p.E + 5) * 4);
  if (p.act_dtype == MOE_BF16) L.part = take(router_scratch_bytes(p));
  if (forward) {
    L.ids = take(n * 4);
    L.tw = take(n * 4);
    L.offs = take((p.E + 2) * 4);
    L.row_tok = take(Rp * 4);
    L.row_w = take(Rp * 4);
    L.pos = take(n * 4);
    L.row_dst = take(Rp * 4);
    L.xp = take(std::max(Rp, p.T * (p.k + 1)) * p.d * ab);
    L.xn = take(p.T * p.d * ab);  // the normalised block input (moe_block_forward with a norm)
    L.gate = take(p.T * 4);       // the shared expert's gate per token
  }
  L.h = take(Rp * ldh_of(p) * ab);
  L.total = o;
  return L;
}

// ============================================================== launch pieces
static Schedule sched_simt(int n_r, int n_s) { return Schedule{64, 64, n_r, n_s, 0, 0, 0, 0}; }
static Schedule sched_tc(int bn, int n_r, int n_s) { return Schedule{kBM, bn, n_r, n_s, 0, 0, 0, 0}; }

// Router and top-k.  `counts` (may be NULL) receives the per-chunk histograms
// for the dispatch when the tensor-core path is taken; *counted says so.
static moe_status launch_router(const moe_problem& p, const void* x, const void* wr, const float* bias,
                                int32_t* ids, float* tw, float* part, int32_t* counts, bool* counted,
                                cudaStream_t st, DeviceInfo* dev) {
  *counted = false;
  if (p.T == 0) return MOE_OK;
  bool tc;
  moe_status s = choose(p.act_dtype == MOE_BF16, &tc);
  if (s != MOE_OK) return s;
  if (!tc) {
    dim3 grid((unsigned)cdiv(p.T, 8));
    PROF_BEGIN("router_simt", st);
    const int npl = select_npl(p.E);
    if (p.act_dtype == MOE_F32) {
      auto kf = npl == 4 ? k_router_simt<float, 4> : npl == 8 ? k_router_simt<float, 8> : k_router_simt<float, 16>;
      CUDA_TRY(launch(kf, grid, 256, 0, st, (const float*)x, (const float*)wr, bias, p.T, p.d, p.E, p.k, ids, tw));
    } else {
      auto kb = npl == 4 ? k_router_simt<bf16, 4> : npl == 8 ? k_router_simt<bf16, 8> : k_router_simt<bf16, 16>;
      CUDA_TRY(launch(kb, grid, 256, 0, st, (const bf16*)x, (const bf16*)wr, bias, p.T, p.d, p.E, p.k, ids, tw));
    }
    LAUNCH_CHECK("router_simt", st);
    return MOE_OK;
  }
  const RouterSplit rs = router_split(p);
  CUtensorMap ax, bw;
  if ((s = map2d(&ax, x, p.d, p.T, p.d, kBM)) != MOE_OK) return s;
  if ((s = map2d(&bw, wr, p.d, p.E, p.d, kRouterBN)) != MOE_OK) return s;
  if (router_fused(p)) {
    // every logit of a row tile in one 4-CTA cluster: select in the epilogue
    // (no scratch: the partials and lists move through the cluster's shared
    // memory); the chunk histograms are counted with atomics
    const int64_t row_tiles = cdiv(p.T, kBM);
    const int npad = std::max(16, (int)align_up((size_t)p.E, 16));  // the MMA's N: every expert
    CUtensorMap bwn;
    if ((s = map2d(&bwn, wr, p.d, p.E, p.d, (uint32_t)npad)) != MOE_OK) return s;
    if (counts) {
      CUDA_TRY(cudaMemsetAsync(counts, 0, (size_t)n_chunks(p) * p.E * 4, st));
      pdl_reset();
    }
    TcGemmArgs a{};
    a.E = 0;
    a.N_s = p.E;
    a.K_s = p.d;
    a.rows_cap = p.T;
    a.topk = p.k;
    a.ids = ids;
    a.tw = tw;
    a.bias = bias;
    a.counts = counts;
    a.status = dev->status;
    PROF_BEGIN("gemm_tc_router", st);
    const int ctas = (int)row_tiles * kRouterKcCtas;
    if (p.k <= 8) CUDA_TRY(launch_router_kc(k_router_kc<8>, ctas, st, ax, bwn, a, npad));
    else CUDA_TRY(launch_router_kc(k_router_kc<16>, ctas, st, ax, bwn, a, npad));
    LAUNCH_CHECK("gemm_tc_router", st);
    *counted = counts != nullptr;
    return MOE_OK;
  }
  TcGemmArgs a{};
  a.E = 0;
  a.N_s = p.E;
  a.K_s = p.d;
  a.rows_cap = p.T;
  a.single_rows = (int)p.T;
  a.single_tiles = rs.tiles;
  a.ksplit = rs.ksplit;
  a.kb_per_split = rs.kb_per;
  a.part = part;
  a.ldp = rs.ldp;
  a.part_stride = p.T * rs.ldp;
  a.status = dev->status;
  if (counts) {  // the chunk histograms k_topk counts into
    CUDA_TRY(cudaMemsetAsync(counts, 0, (size_t)n_chunks(p) * p.E * 4, st));
    pdl_reset();
  }
  PROF_BEGIN("gemm_tc_router", st);
  CUDA_TRY(launch(k_gemm_tc<kRouterBN, false, 4, kTcLogits>, std::min(rs.tiles, dev->sms), Gemm2Cfg::THREADS,
                  Gemm2Cfg::SMEM_BYTES, st, ax, ax, bw, bw, bw, bw, a));
  LAUNCH_CHECK("gemm_tc_router", st);
  PROF_BEGIN("topk", st);
  const int npl = select_npl(p.E);
  auto kt = npl == 4 ? k_topk<4> : npl == 8 ? k_topk<8> : k_topk<16>;
  CUDA_TRY(launch(kt, (unsigned)cdiv(p.T, 8), 256, 0, st, part, rs.ksplit, p.T * rs.ldp, rs.ldp, bias, p.T, p.E, p.k,
                  ids, tw, counts));
  LAUNCH_CHECK("topk", st);
  *counted = counts != nullptr;
  return MOE_OK;
}

// Histogram (unless the router wrote it), then one kernel that scans it and
// scatters: offs, row_tok, row_w, pos, row_dst (may be NULL), the shared rows,
// and optionally the tile prefixes.
// Dispatch: the stable sort of the (token, slot) pairs by expert and, when xp
// is given, the copy of x's rows into their dispatched rows (and the shared
// expert's rows), in one kernel.
static moe_status launch_dispatch(const moe_problem& p, const int32_t* ids, const float* tw, bool counted,
                                  int32_t* offs, int32_t* row_tok, float* row_w, int32_t* pos, int32_t* row_dst,
                                  int32_t* counts, Schedule sa, int32_t* pre_a, Schedule sb, int32_t* pre_b,
                                  const void* x, void* xp, cudaStream_t st, DeviceInfo* dev,
                                  const float* shared_gate = nullptr) {
  const int nch = (int)n_chunks(p);
  if (p.T == 0) {
    CUDA_TRY(cudaMemsetAsync(counts, 0, (size_t)p.E * 4, st));
    pdl_reset();
  } else if (!counted) {
    PROF_BEGIN("count", st);
    CUDA_TRY(launch(k_count, nch, 256, 0, st, ids, p.T, p.k, p.E, counts, dev->status));
    LAUNCH_CHECK("count", st);
  }
  const int vec = (int)(p.d * esize(p.act_dtype) / 16);
  PROF_BEGIN("dispatch", st);
  CUDA_TRY(launch(k_dispatch, nch * kSubBlocks, kScatterWarps * 32, 0, st, ids, tw, p.T, p.k, p.E, counts, nch,
                  p.I_s > 0, offs, sa, pre_a, sb, pre_b, row_tok, row_w, pos, row_dst, shared_gate,
                  (const uint4*)x, vec, (uint4*)xp, dev->status));
  LAUNCH_CHECK("dispatch", st);
  return MOE_OK;
}

struct ExpertWeights {
  const void *wg, *wu, *wd, *sg, *su, *sd;
  const float* scales;
};

// FP8 scale sub-buffers (see moe.h).
static void scale_parts(const moe_problem& p, const float* sc, const float* part[6]) {
  const int64_t gd = p.d / 128, gi = p.I / 128, gs = p.I_s / 128;
  const int64_t off[6] = {0,
                          (int64_t)p.E * gi * gd,
                          2 * (int64_t)p.E * gi * gd,
                          3 * (int64_t)p.E * gi * gd,
                          3 * (int64_t)p.E * gi * gd + gs * gd,
                          3 * (int64_t)p.E * gi * gd + 2 * gs * gd};
  for (int i = 0; i < 6; ++i) part[i] = sc ? sc + off[i] : nullptr;
}

// Output of the down projection: either the weighted rows in (token, slot)
// order (the fused forward) or the unweighted rows in dispatch order (the
// expert stage alone).
// Largest token matrix the gate/up GEMM gathers from.  At the 35B shape (16
// MiB) the matrix stays in L2 while the weights stream past; at the prefill
// shape (128 MiB) it does not, but in the panel tile order each activation
// tile is fetched once per panel either way, and the gather spares the
// dispatch its 1.5 GB copy (measured on one box: step 10.62 against 10.80 and
// 10.87 ms; with the column-major order of the first version it was 7 %
// slower there, and the limit was 32 MiB).
constexpr int64_t kGatherMaxBytes = 256ll << 20;

// Whether the fused forward's gate/up GEMM gathers its rows from the block's
// input: the row-tiled bf16 form, with a token matrix of at most
// kGatherMaxBytes (every row is read k + 1 times).
static bool gathers_rows(const moe_problem& p, int form) {
  return form == kFormRows && p.w_dtype == MOE_BF16 && p.T * p.d * 2 <= kGatherMaxBytes;
}

// The gate/up GEMM's activation rows taken straight from the token matrix
// (row r = x[row_tok[r]]) instead of from the dispatched rows; x NULL: not.
struct GatherSrc {
  const void* x = nullptr;
  const int32_t* row_tok = nullptr;
};

struct DownOut {
  void* ys;               // slot layout [T*(k+1), d], or NULL
  const int32_t* row_dst;
  const float* row_w;
  void* out;              // dispatch layout [R', d], or NULL
};

template <typename TA, typename TW>
static moe_status simt_gemms(const moe_problem& p, const void* xp, const int32_t* offs, const ExpertWeights& w,
                             int32_t* pre_a, int32_t* pre_b, void* H, const DownOut& o, cudaStream_t st,
                             DeviceInfo* dev) {
  const float* sp[6];
  scale_parts(p, w.scales, sp);
  const unsigned grid = (unsigned)dev->sms * 4;
  SimtGemmArgs<TA, TW> a{};
  a.offs = offs;
  a.E = p.E;
  a.rows_cap = rows_total(p);
  // gate/up: A = dispatched rows [R', d], N = I (I_s), K = d
  a.A = (const TA*)xp;
  a.lda = p.d;
  a.prefix = pre_a;
  a.N_r = p.I;
  a.N_s = p.I_s;
  a.K_r = p.d;
  a.K_s = p.d;
  a.b1 = WeightSet<TW>{(const TW*)w.wg, (const TW*)w.sg, sp[0], sp[3]};
  a.b2 = WeightSet<TW>{(const TW*)w.wu, (const TW*)w.su, sp[1], sp[4]};
  a.H = (TA*)H;
  a.ldh = ldh_of(p);
  PROF_BEGIN("gemm_simt_swiglu", st);
  CUDA_TRY(launch(k_gemm_simt<TA, TW, kEpiSwiGLU>, grid, 256, 0, st, a));
  LAUNCH_CHECK("gemm_simt_swiglu", st);
  // down: A = H [R', ldh], N = d, K = I (I_s)
  SimtGemmArgs<TA, TW> b{};
  b.offs = offs;
  b.E = p.E;
  b.rows_cap = rows_total(p);
  b.A = (const TA*)H;
  b.lda = ldh_of(p);
  b.prefix = pre_b;
  b.N_r = p.d;
  b.N_s = p.d;
  b.K_r = p.I;
  b.K_s = p.I_s;
  b.b1 = WeightSet<TW>{(const TW*)w.wd, (const TW*)w.sd, sp[2], sp[5]};
  b.b2 = b.b1;
  if (o.ys) {
    b.ys = (TA*)o.ys;
    b.ys_rows = p.T * (p.k + 1);
    b.status = dev->status;
    b.ldy = p.d;
    b.row_dst = o.row_dst;
    b.row_w = o.row_w;
    PROF_BEGIN("gemm_simt_slot", st);
    CUDA_TRY(launch(k_gemm_simt<TA, TW, kEpiSlotStore>, grid, 256, 0, st, b));
    LAUNCH_CHECK("gemm_simt_slot", st);
  } else {
    b.out = (TA*)o.out;
    b.ldo = p.d;
    PROF_BEGIN("gemm_simt_store", st);
    CUDA_TRY(launch(k_gemm_simt<TA, TW, kEpiStore>, grid, 256, 0, st, b));
    LAUNCH_CHECK("gemm_simt_store", st);
  }
  return MOE_OK;
}

// Tile order of the grouped tensor-core GEMMs: panels of column blocks whose
// weight blocks take about kPanelBytes together (decode_tile); column-block-
// major (a panel of one) when a group's whole weight slice is at most
// kSmallSliceBytes, where a group's rows are few and everything stays in L2
// (the 35B shapes: 4 and 2 MB per expert; measured there, panels of every
// column block made the gate/up GEMM 231 -> 252 us).
constexpr int64_t kPanelBytes = 32ll << 20, kSmallSliceBytes = 16ll << 20;
static int panel_of(int64_t weight_tile_bytes, int64_t column_blocks) {
  if (weight_tile_bytes * column_blocks <= kSmallSliceBytes) return 1;
  return (int)std::max<int64_t>(1, std::min<int64_t>(64, kPanelBytes / std::max<int64_t>(weight_tile_bytes, 1)));
}

// Epilogue outputs of up to this many bytes are stored with an L2
// evict-last hint (the next kernel reads them back); larger ones evict-first.
constexpr int64_t kKeepOutBytes = 160ll << 20;
static int keep_out(int64_t bytes) { return bytes <= kKeepOutBytes ? 1 : 0; }

template <bool FP8>
static moe_status tc_gemms_t(const moe_problem& p, const void* xp, const int32_t* offs, const ExpertWeights& w,
                             int32_t* pre_a, int32_t* pre_b, void* H, const DownOut& o, cudaStream_t st,
                             DeviceInfo* dev, const GatherSrc& g) {
  const int64_t Rp = rows_total(p), ldh = ldh_of(p);
  const bool sh = p.I_s > 0;
  constexpr int S = FP8 ? kFp8Stages : 4;
  using C1 = TcGemmCfg<128, true, S, FP8>;
  using C2 = TcGemmCfg<256, false, S, FP8>;
  const float* sp[6];
  scale_parts(p, w.scales, sp);
  moe_status s;
  CUtensorMap aR, aS, bR, bS, cR, cS;
  // gate/up + SwiGLU
  if ((s = map2d(&aR, xp, p.d, Rp, p.d, kBM)) != MOE_OK) return s;
  if ((s = map3d(&bR, w.wg, p.d, p.I, p.E, 128, FP8)) != MOE_OK) return s;
  if ((s = map3d(&cR, w.wu, p.d, p.I, p.E, 128, FP8)) != MOE_OK) return s;
  bS = bR;
  cS = cR;
  if (sh) {
    if ((s = map2d(&bS, w.sg, p.d, p.I_s, p.d, 128, FP8)) != MOE_OK) return s;
    if ((s = map2d(&cS, w.su, p.d, p.I_s, p.d, 128, FP8)) != MOE_OK) return s;
  }
  TcGemmArgs a{};
  a.offs = offs;
  a.prefix = pre_a;
  a.E = p.E;
  a.rows_cap = Rp;
  a.single_rows = -1;
  a.N_r = p.I;
  a.N_s = p.I_s;
  a.K_r = p.d;
  a.K_s = p.d;
  a.H = (bf16*)H;
  a.ldh = ldh;
  a.out_keep = keep_out(Rp * ldh * 2);
  a.panel = panel_of(2 * 128 * (int64_t)p.d * (FP8 ? 1 : 2), cdiv(p.I, 128));  // gate and up rows, 128 columns
  a.swap_small = FP8 ? 0 : 1;  // tiles of at most 64 rows run with the MMA roles swapped
  a.sc_b_r = sp[0];
  a.sc_b_s = sp[3];
  a.sc_c_r = sp[1];
  a.sc_c_s = sp[4];
  a.status = dev->status;
  if (!FP8) a.sched = pre_a + p.E + 2;  // tiles claimed in order (the prefix writer zeroed it)
  PROF_BEGIN("gemm_tc_swiglu", st);
  if (!FP8 && g.x) {
    a.gx = (const bf16*)g.x;
    a.gx_rows = p.T;
    a.row_tok = g.row_tok;
    a.ldx = p.d;
    CUDA_TRY(launch(k_gemm_tc<128, true, 4, kTcSwiGLU, false, true>, dev->sms, Gemm1GCfg::THREADS,
                    Gemm1GCfg::SMEM_BYTES, st, aR, aR, bR, bS, cR, cS, a));
  } else {
    CUDA_TRY(launch(k_gemm_tc<128, true, S, kTcSwiGLU, FP8>,
                    dev->sms, C1::THREADS, C1::SMEM_BYTES, st, aR, aR, bR, bS, cR, cS, a));
  }
  LAUNCH_CHECK("gemm_tc_swiglu", st);
  // down
  if ((s = map2d(&aR, H, p.I, Rp, ldh, kBM)) != MOE_OK) return s;
  aS = aR;
  if (sh && (s = map2d(&aS, H, p.I_s, Rp, ldh, kBM)) != MOE_OK) return s;
  if ((s = map3d(&bR, w.wd, p.I, p.d, p.E, 256, FP8)) != MOE_OK) return s;
  bS = bR;
  if (sh && (s = map2d(&bS, w.sd, p.I_s, p.d, p.I_s, 256, FP8)) != MOE_OK) return s;
  TcGemmArgs b{};
  b.offs = offs;
  b.prefix = pre_b;
  b.E = p.E;
  b.rows_cap = Rp;
  b.single_rows = -1;
  b.N_r = p.d;
  b.N_s = p.d;
  b.K_r = p.I;
  b.K_s = p.I_s;
  b.sc_b_r = sp[2];
  b.sc_b_s = sp[5];
  b.status = dev->status;
  b.out_keep = keep_out((o.ys ? p.T * (p.k + 1) : Rp) * p.d * 2);
  b.panel = panel_of(256 * (int64_t)std::max(p.I, p.I_s) * (FP8 ? 1 : 2), cdiv(p.d, 256));
  b.swap_small = FP8 ? 0 : 1;
  if (!FP8) b.sched = pre_b + p.E + 2;
  if (o.ys) {
    b.ys = (bf16*)o.ys;
    b.ys_rows = p.T * (p.k + 1);
    b.ldy = p.d;
    b.row_dst = o.row_dst;
    b.row_w = o.row_w;
    PROF_BEGIN("gemm_tc_down", st);
    CUDA_TRY(launch(k_gemm_tc<256, false, S, kTcSlotStore, FP8>,
                    dev->sms, C2::THREADS, C2::SMEM_BYTES, st, aR, aS, bR, bS, bR, bS, b));
    LAUNCH_CHECK("gemm_tc_down", st);
  } else {
    b.out = (bf16*)o.out;
    b.ldo = p.d;
    PROF_BEGIN("gemm_tc_store", st);
    CUDA_TRY(launch(k_gemm_tc<256, false, S, kTcStore, FP8>,
                    dev->sms, C2::THREADS, C2::SMEM_BYTES, st, aR, aS, bR, bS, bR, bS, b));
    LAUNCH_CHECK("gemm_tc_store", st);
  }
  return MOE_OK;
}

static moe_status tc_gemms(const moe_problem& p, const void* xp, const int32_t* offs, const ExpertWeights& w,
                           int32_t* pre_a, int32_t* pre_b, void* H, const DownOut& o, cudaStream_t st,
                           DeviceInfo* dev, const GatherSrc& g) {
  if (p.w_dtype == MOE_FP8_E4M3_B128) return tc_gemms_t<true>(p, xp, offs, w, pre_a, pre_b, H, o, st, dev, g);
  return tc_gemms_t<false>(p, xp, offs, w, pre_a, pre_b, H, o, st, dev, g);
}

// Which projections a launcher enqueues: the split form runs both gate/up
// launches before either down launch, since a down GEMM stores its slot rows
// into the buffer the other gate/up GEMM reads its dispatched rows from.
enum { kPhaseGateUp = 1, kPhaseDown = 2, kPhaseBoth = 3 };

template <bool FP8>
static moe_status swap_gemms_t(const moe_problem& p, const void* xp, const int32_t* offs, const ExpertWeights& w,
                               int32_t* pre_a, int32_t* pre_b, void* H, const DownOut& o, cudaStream_t st,
                               DeviceInfo* dev, int phases = kPhaseBoth) {
  using C1 = SwapCfg<true>;
  const int grid = dev->sms;
  using C2 = SwapCfg<false>;
  const int64_t Rp = rows_total(p), ldh = ldh_of(p);
  const bool sh = p.I_s > 0;
  const float* sp[6];
  scale_parts(p, w.scales, sp);
  moe_status s;
  CUtensorMap xR, xS, bR, bS, cR, cS;
  // gate/up + SwiGLU: weights [E, I, d] are the M operand, token rows the N operand
  if (phases & kPhaseGateUp) {
    if ((s = map2d(&xR, xp, p.d, Rp, p.d, kNCH)) != MOE_OK) return s;
    if ((s = map3d(&bR, w.wg, p.d, p.I, p.E, 128, FP8, FP8)) != MOE_OK) return s;
    if ((s = map3d(&cR, w.wu, p.d, p.I, p.E, 128, FP8, FP8)) != MOE_OK) return s;
    bS = bR;
    cS = cR;
    if (sh) {
      if ((s = map2d(&bS, w.sg, p.d, p.I_s, p.d, 128, FP8, FP8)) != MOE_OK) return s;
      if ((s = map2d(&cS, w.su, p.d, p.I_s, p.d, 128, FP8, FP8)) != MOE_OK) return s;
    }
    TcGemmArgs a{};
    a.offs = offs;
    a.prefix = pre_a;
    a.E = p.E;
    a.rows_cap = Rp;
    a.single_rows = -1;
    a.N_r = p.I;
    a.N_s = p.I_s;
    a.K_r = p.d;
    a.K_s = p.d;
    a.H = (bf16*)H;
    a.ldh = ldh;
    a.sc_b_r = sp[0];
    a.sc_b_s = sp[3];
    a.sc_c_r = sp[1];
    a.sc_c_s = sp[4];
    a.status = dev->status;
    PROF_BEGIN("gemm_tc_swiglu", st);
    if (FP8)
      CUDA_TRY(launch(k_gemm_swap8<true, kTcSwiGLU>,
                      grid, Swap8Cfg<true>::THREADS, Swap8Cfg<true>::SMEM_BYTES, st, xR, xR, bR, bS, cR, cS, a));
    else
      CUDA_TRY(launch(k_gemm_swap<true, kTcSwiGLU>,
                      grid, C1::THREADS, C1::SMEM_BYTES, st, xR, xR, bR, bS, cR, cS, a));
    LAUNCH_CHECK("gemm_tc_swiglu", st);
  }
  if (!(phases & kPhaseDown)) return MOE_OK;
  // down: W_down [E, d, I] is the M operand, H rows the N operand
  if ((s = map2d(&xR, H, p.I, Rp, ldh, kNCH)) != MOE_OK) return s;
  xS = xR;
  if (sh && (s = map2d(&xS, H, p.I_s, Rp, ldh, kNCH)) != MOE_OK) return s;
  if ((s = map3d(&bR, w.wd, p.I, p.d, p.E, 128, FP8, FP8)) != MOE_OK) return s;
  bS = bR;
  if (sh && (s = map2d(&bS, w.sd, p.I_s, p.d, p.I_s, 128, FP8, FP8)) != MOE_OK) return s;
  TcGemmArgs b{};
  b.offs = offs;
  b.prefix = pre_b;
  b.E = p.E;
  b.rows_cap = Rp;
  b.single_rows = -1;
  b.N_r = p.d;
  b.N_s = p.d;
  b.K_r = p.I;
  b.K_s = p.I_s;
  b.sc_b_r = sp[2];
  b.sc_b_s = sp[5];
  b.sc_c_r = sp[2];  // E4M3: the second 128-row half of each 256-row tile, same matrix
  b.sc_c_s = sp[5];
  b.status = dev->status;
  if (o.ys) {
    b.ys = (bf16*)o.ys;
    b.ys_rows = p.T * (p.k + 1);
    b.ldy = p.d;
    b.row_dst = o.row_dst;
    b.row_w = o.row_w;
    PROF_BEGIN("gemm_tc_down", st);
    if (FP8)
      CUDA_TRY(launch(k_gemm_swap8<true, kTcSlotStore>,
                      grid, Swap8Cfg<true>::THREADS, Swap8Cfg<true>::SMEM_BYTES, st, xR, xS, bR, bS, bR, bS, b));
    else
      CUDA_TRY(launch(k_gemm_swap<false, kTcSlotStore>,
                      grid, C2::THREADS, C2::SMEM_BYTES, st, xR, xS, bR, bS, bR, bS, b));
    LAUNCH_CHECK("gemm_tc_down", st);
  } else {
    b.out = (bf16*)o.out;
    b.ldo = p.d;
    PROF_BEGIN("gemm_tc_store", st);
    if (FP8)
      CUDA_TRY(launch(k_gemm_swap8<true, kTcStore>,
                      grid, Swap8Cfg<true>::THREADS, Swap8Cfg<true>::SMEM_BYTES, st, xR, xS, bR, bS, bR, bS, b));
    else
      CUDA_TRY(launch(k_gemm_swap<false, kTcStore>,
                      grid, C2::THREADS, C2::SMEM_BYTES, st, xR, xS, bR, bS, bR, bS, b));
    LAUNCH_CHECK("gemm_tc_store", st);
  }
  return MOE_OK;
}

// Row-tiled expert GEMMs on CTA pairs (bf16 weights): 256-row tiles, each CTA
// loading 128 activation rows and a 128-row half of the weight tile.
static moe_status pair_gemms(const moe_problem& p, const void* xp, const int32_t* offs, const ExpertWeights& w,
                             int32_t* pre_a, int32_t* pre_b, void* H, const DownOut& o, cudaStream_t st,
                             DeviceInfo* dev, int phases = kPhaseBoth) {
  const int grid = dev->pair_ctas;
  const int64_t Rp = rows_total(p), ldh = ldh_of(p);
  const bool sh = p.I_s > 0;
  moe_status s;
  CUtensorMap aR, aS, bR, bS, cR, cS;
  // gate/up + SwiGLU: rank 0 streams gate rows, rank 1 up rows
  if (phases & kPhaseGateUp) {
    if ((s = map2d(&aR, xp, p.d, Rp, p.d, kBM)) != MOE_OK) return s;
    if ((s = map3d(&bR, w.wg, p.d, p.I, p.E, 128)) != MOE_OK) return s;
    if ((s = map3d(&cR, w.wu, p.d, p.I, p.E, 128)) != MOE_OK) return s;
    bS = bR;
    cS = cR;
    if (sh) {
      if ((s = map2d(&bS, w.sg, p.d, p.I_s, p.d, 128)) != MOE_OK) return s;
      if ((s = map2d(&cS, w.su, p.d, p.I_s, p.d, 128)) != MOE_OK) return s;
    }
    TcGemmArgs a{};
    a.offs = offs;
    a.prefix = pre_a;
    a.E = p.E;
    a.rows_cap = Rp;
    a.single_rows = -1;
    a.N_r = p.I;
    a.N_s = p.I_s;
    a.K_r = p.d;
    a.K_s = p.d;
    a.H = (bf16*)H;
    a.ldh = ldh;
    a.out_keep = keep_out(Rp * ldh * 2);
    a.panel = panel_of(2 * 128 * (int64_t)p.d * 2, cdiv(p.I, 128));
    a.status = dev->status;
    PROF_BEGIN("gemm_tc_swiglu", st);
    CUDA_TRY(launch_pair(k_gemm_pair<128, true, kPairStages, kTcSwiGLU>, grid, Pair1Cfg::THREADS,
                         Pair1Cfg::SMEM_BYTES, st, aR, aR, bR, bS, cR, cS, a));
    LAUNCH_CHECK("gemm_tc_swiglu", st);
  }
  if (!(phases & kPhaseDown)) return MOE_OK;
  // down: the two 128-row halves of each 256-row weight block
  if ((s = map2d(&aR, H, p.I, Rp, ldh, kBM)) != MOE_OK) return s;
  aS = aR;
  if (sh && (s = map2d(&aS, H, p.I_s, Rp, ldh, kBM)) != MOE_OK) return s;
  if ((s = map3d(&bR, w.wd, p.I, p.d, p.E, 128)) != MOE_OK) return s;
  bS = bR;
  if (sh && (s = map2d(&bS, w.sd, p.I_s, p.d, p.I_s, 128)) != MOE_OK) return s;
  TcGemmArgs b{};
  b.offs = offs;
  b.prefix = pre_b;
  b.E = p.E;
  b.rows_cap = Rp;
  b.single_rows = -1;
  b.N_r = p.d;
  b.N_s = p.d;
  b.K_r = p.I;
  b.K_s = p.I_s;
  b.status = dev->status;
  b.out_keep = keep_out((o.ys ? p.T * (p.k + 1) : Rp) * p.d * 2);
  b.panel = panel_of(256 * (int64_t)std::max(p.I, p.I_s) * 2, cdiv(p.d, 256));
  if (o.ys) {
    b.ys = (bf16*)o.ys;
    b.ys_rows = p.T * (p.k + 1);
    b.ldy = p.d;
    b.row_dst = o.row_dst;
    b.row_w = o.row_w;
    PROF_BEGIN("gemm_tc_down", st);
    CUDA_TRY(launch_pair(k_gemm_pair<256, false, kPairStages, kTcSlotStore>, grid, Pair2Cfg::THREADS,
                         Pair2Cfg::SMEM_BYTES, st, aR, aS, bR, bS, bR, bS, b));
    LAUNCH_CHECK("gemm_tc_down", st);
  } else {
    b.out = (bf16*)o.out;
    b.ldo = p.d;
    PROF_BEGIN("gemm_tc_store", st);
    CUDA_TRY(launch_pair(k_gemm_pair<256, false, kPairStages, kTcStore>, grid, Pair2Cfg::THREADS,
                         Pair2Cfg::SMEM_BYTES, st, aR, aS, bR, bS, bR, bS, b));
    LAUNCH_CHECK("gemm_tc_store", st);
  }
  return MOE_OK;
}

// Expert GEMMs on CTA pairs with the tokens as the MMA's N (bf16 weights):
// tiles of up to 256 dispatched rows, the MMA's N their count rounded up to
// 16; each CTA loads 128 weight rows and half of the tile's token rows.
static moe_status pairt_gemms(const moe_problem& p, const void* xp, const int32_t* offs, const ExpertWeights& w,
                              int32_t* pre_a, int32_t* pre_b, void* H, const DownOut& o, cudaStream_t st,
                              DeviceInfo* dev) {
  const int grid = dev->pairt_ctas;
  const int64_t Rp = rows_total(p), ldh = ldh_of(p);
  const bool sh = p.I_s > 0;
  moe_status s;
  // maps: tokens (small boxes, routed / shared K), tokens (wide boxes), B, C
  CUtensorMap m[8];
  CUtensorMap &tR = m[0], &tS = m[1], &uR = m[2], &uS = m[3], &bR = m[4], &bS = m[5], &cR = m[6], &cS = m[7];
  // gate/up + SwiGLU: each CTA streams 64 gate and 64 up rows of its features
  if ((s = map2d(&tR, xp, p.d, Rp, p.d, kTokBox)) != MOE_OK) return s;
  if ((s = map2d(&uR, xp, p.d, Rp, p.d, kTokBoxWide)) != MOE_OK) return s;
  tS = tR;
  uS = uR;
  if ((s = map3d(&bR, w.wg, p.d, p.I, p.E, 64)) != MOE_OK) return s;
  if ((s = map3d(&cR, w.wu, p.d, p.I, p.E, 64)) != MOE_OK) return s;
  bS = bR;
  cS = cR;
  if (sh) {
    if ((s = map2d(&bS, w.sg, p.d, p.I_s, p.d, 64)) != MOE_OK) return s;
    if ((s = map2d(&cS, w.su, p.d, p.I_s, p.d, 64)) != MOE_OK) return s;
  }
  TcGemmArgs a{};
  a.offs = offs;
  a.prefix = pre_a;
  a.E = p.E;
  a.rows_cap = Rp;
  a.single_rows = -1;
  a.N_r = p.I;
  a.N_s = p.I_s;
  a.K_r = p.d;
  a.K_s = p.d;
  a.H = (bf16*)H;
  a.ldh = ldh;
  a.out_keep = keep_out(Rp * ldh * 2);
  a.panel = panel_of(2 * 128 * (int64_t)p.d * 2, cdiv(p.I, 128));
  a.status = dev->status;
  PROF_BEGIN("gemm_tc_swiglu", st);
  CUDA_TRY(launch_pairt(k_gemm_pairt<true, kPairTStages, kTcSwiGLU>, grid, PairT1Cfg::THREADS, PairT1Cfg::SMEM_BYTES,
                        st, m, a));
  LAUNCH_CHECK("gemm_tc_swiglu", st);
  // down: each CTA streams 128 rows of a 256-row weight block
  if ((s = map2d(&tR, H, p.I, Rp, ldh, kTokBox)) != MOE_OK) return s;
  if ((s = map2d(&uR, H, p.I, Rp, ldh, kTokBoxWide)) != MOE_OK) return s;
  tS = tR;
  uS = uR;
  if (sh && (s = map2d(&tS, H, p.I_s, Rp, ldh, kTokBox)) != MOE_OK) return s;
  if (sh && (s = map2d(&uS, H, p.I_s, Rp, ldh, kTokBoxWide)) != MOE_OK) return s;
  if ((s = map3d(&bR, w.wd, p.I, p.d, p.E, 128)) != MOE_OK) return s;
  bS = bR;
  if (sh && (s = map2d(&bS, w.sd, p.I_s, p.d, p.I_s, 128)) != MOE_OK) return s;
  cR = bR;
  cS = bS;
  TcGemmArgs b{};
  b.offs = offs;
  b.prefix = pre_b;
  b.E = p.E;
  b.rows_cap = Rp;
  b.single_rows = -1;
  b.N_r = p.d;
  b.N_s = p.d;
  b.K_r = p.I;
  b.K_s = p.I_s;
  b.status = dev->status;
  b.out_keep = keep_out((o.ys ? p.T * (p.k + 1) : Rp) * p.d * 2);
  b.panel = panel_of(256 * (int64_t)std::max(p.I, p.I_s) * 2, cdiv(p.d, 256));
  if (o.ys) {
    b.ys = (bf16*)o.ys;
    b.ys_rows = p.T * (p.k + 1);
    b.ldy = p.d;
    b.row_dst = o.row_dst;
    b.row_w = o.row_w;
    PROF_BEGIN("gemm_tc_down", st);
    CUDA_TRY(launch_pairt(k_gemm_pairt<false, kPairTStages, kTcSlotStore>, grid, PairT2Cfg::THREADS,
                          PairT2Cfg::SMEM_BYTES, st, m, b));
    LAUNCH_CHECK("gemm_tc_down", st);
  } else {
    b.out = (bf16*)o.out;
    b.ldo = p.d;
    PROF_BEGIN("gemm_tc_store", st);
    CUDA_TRY(launch_pairt(k_gemm_pairt<false, kPairTStages, kTcStore>, grid, PairT2Cfg::THREADS,
                          PairT2Cfg::SMEM_BYTES, st, m, b));
    LAUNCH_CHECK("gemm_tc_store", st);
  }
  return MOE_OK;
}

// The split form: the large groups' tiles are counted in pre_a / pre_b, the
// others' in the second prefix of each (pre + E + 3); each kernel walks its
// own list and writes its own rows of H and of the slot rows.  A down GEMM
// stores its slot rows over the dispatched rows that both gate/up GEMMs read,
// so both gate/up GEMMs run before either down GEMM.
static moe_status split_gemms(const moe_problem& p, const void* xp, const int32_t* offs, const ExpertWeights& w,
                              int32_t* pre_a, int32_t* pre_b, void* H, const DownOut& o, cudaStream_t st,
                              DeviceInfo* dev) {
  int32_t* sa = pre_a + p.E + 3;
  int32_t* sb = pre_b + p.E + 3;
  moe_status s;
  if ((s = pair_gemms(p, xp, offs, w, pre_a, pre_b, H, o, st, dev, kPhaseGateUp)) != MOE_OK) return s;
  if ((s = swap_gemms_t<false>(p, xp, offs, w, sa, sb, H, o, st, dev, kPhaseGateUp)) != MOE_OK) return s;
  if ((s = pair_gemms(p, xp, offs, w, pre_a, pre_b, H, o, st, dev, kPhaseDown)) != MOE_OK) return s;
  return swap_gemms_t<false>(p, xp, offs, w, sa, sb, H, o, st, dev, kPhaseDown);
}

static moe_status expert_gemms(const moe_problem& p, int form, const void* xp, const int32_t* offs,
                               const ExpertWeights& w, int32_t* pre_a, int32_t* pre_b, void* H, const DownOut& o,
                               cudaStream_t st, DeviceInfo* dev, const GatherSrc& g = GatherSrc{}) {
  if (form == kFormSwap) {
    if (p.w_dtype == MOE_FP8_E4M3_B128) return swap_gemms_t<true>(p, xp, offs, w, pre_a, pre_b, H, o, st, dev);
    return swap_gemms_t<false>(p, xp, offs, w, pre_a, pre_b, H, o, st, dev);
  }
  if (form == kFormRows) return tc_gemms(p, xp, offs, w, pre_a, pre_b, H, o, st, dev, g);
  if (form == kFormPair) return pair_gemms(p, xp, offs, w, pre_a, pre_b, H, o, st, dev);
  if (form == kFormSplit) return split_gemms(p, xp, offs, w, pre_a, pre_b, H, o, st, dev);
  if (form == kFormPairT) return pairt_gemms(p, xp, offs, w, pre_a, pre_b, H, o, st, dev);
  if (p.act_dtype == MOE_F32) return simt_gemms<float, float>(p, xp, offs, w, pre_a, pre_b, H, o, st, dev);
  if (p.w_dtype == MOE_BF16) return simt_gemms<bf16, bf16>(p, xp, offs, w, pre_a, pre_b, H, o, st, dev);
  return simt_gemms<bf16, uint8_t>(p, xp, offs, w, pre_a, pre_b, H, o, st, dev);
}

static void schedules(const moe_problem& p, int form, Schedule* sa, Schedule* sb) {
  if (form == kFormRows) {
    *sa = sched_tc(128, p.I, p.I_s);
    *sb = sched_tc(256, p.d, p.d);
  } else if (form == kFormPair || form == kFormPairT) {  // 256-row tiles of CTA pairs
    *sa = Schedule{kPairBM, 128, p.I, p.I_s, 0, 0, 0, 0};
    *sb = Schedule{kPairBM, 256, p.d, p.d, 0, 0, 0, 0};
  } else if (form == kFormSwap) {  // (token chunk, 128 weight rows) tiles; E4M3 down: 256 rows
    *sa = Schedule{kNCH, 128, p.I, p.I_s, 0, 0, 0, 0};
    *sb = Schedule{kNCH, p.w_dtype == MOE_FP8_E4M3_B128 ? 256 : 128, p.d, p.d, 0, 0, 0, 0};
  } else if (form == kFormSplit) {  // pair tiles for the large groups, weight-row tiles for the rest
    *sa = Schedule{kPairBM, 128, p.I, p.I_s, 0, kSplitRows - 1, kNCH, 128};
    *sb = Schedule{kPairBM, 256, p.d, p.d, 0, kSplitRows - 1, kNCH, 128};
  } else {
    *sa = sched_simt(p.I, p.I_s);
    *sb = sched_simt(p.d, p.d);
  }
}

static moe_status check_weights(const moe_problem& p, const ExpertWeights& w) {
  NEED(w.wg);
  NEED(w.wu);
  NEED(w.wd);
  if (p.I_s > 0) {
    NEED(w.sg);
    NEED(w.su);
    NEED(w.sd);
  }
  if (p.w_dtype == MOE_FP8_E4M3_B128) NEED(w.scales);
  return MOE_OK;
}

// ============================================================== C ABI
extern "C" {

moe_status moe_check_problem(const moe_problem* p) { return check(p); }

size_t moe_workspace_size(const moe_problem* p) { return check(p) == MOE_OK ? layout(*p, true).total : 0; }
size_t moe_stage_workspace_size(const moe_problem* p) { return check(p) == MOE_OK ? layout(*p, false).total : 0; }

moe_status moe_set_path(int path) {
  if (path < 0 || path > 6) return fail(MOE_ERR_INVALID_ARG, "path %d is not 0, 1, 2, 3, 4, 5 or 6", path);
  g_path = path;
  return MOE_OK;
}

moe_status moe_set_wait_limit(int64_t cycles) {
  DeviceInfo* dev;
  moe_status s = device_info(&dev);
  if (s != MOE_OK) return s;
  const long long v = cycles > 0 ? (long long)cycles : kWaitLimitCycles;
  CUDA_TRY(cudaMemcpyToSymbol(g_wait_limit, &v, sizeof v));
  return MOE_OK;
}

int moe_last_launch_count(void) { return g_launches; }

int moe_bounds_checked(void) {
#ifdef MOE_CHECKS
  return 1;
#else
  return 0;
#endif
}

moe_status moe_profile_enable(int on) {
  if (on < 0 || on > 2) return fail(MOE_ERR_INVALID_ARG, "profile mode %d is not 0, 1 or 2", on);
  g_prof.on = on != 0;
  g_prof.mode = on;
  g_prof.used = 0;
  return MOE_OK;
}

int moe_profile_read(int max, float* ms, const char** names) {
  Profiler& P = g_prof;
  int n = std::min(max, P.used);
  for (int i = 0; i < n; ++i) {
    float t = -1.f;
    if (cudaEventSynchronize(P.ev[i].end) != cudaSuccess ||
        cudaEventElapsedTime(&t, P.ev[i].begin, P.ev[i].end) != cudaSuccess)
      t = -1.f;
    if (ms) ms[i] = t;
    if (names) names[i] = P.ev[i].name;
  }
  P.used = 0;
  return n;
}

const char* moe_last_error_string(void) { return g_err; }

moe_status moe_device_status(int32_t* detail) {
  DeviceInfo* dev;
  moe_status s = device_info(&dev);
  if (s != MOE_OK) return s;
  CUDA_TRY(cudaDeviceSynchronize());
  unsigned v = 0, zero = 0;
  CUDA_TRY(cudaMemcpyFromSymbol(&v, g_status, sizeof v));
  CUDA_TRY(cudaMemcpyToSymbol(g_status, &zero, sizeof zero));
  if (detail) *detail = (int32_t)v;
  if (v == 0) return MOE_OK;
  if ((v >> 24) == 0x07) return fail(MOE_ERR_TIMEOUT, "device wait timed out (code 0x%08x)", v);
  return fail(MOE_ERR_DEVICE_CHECK, "device check failed (code 0x%08x)", v);
}

moe_status moe_router_topk(const moe_problem* p, const void* x, const void* w_router, const float* router_bias,
                           int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("moe_router_topk");
  moe_status s = check(p);
  if (s != MOE_OK) return s;
  if (p->T == 0) {
    g_launches = 0;
    return MOE_OK;
  }
  NEED(x);
  NEED(w_router);
  MAYBE(router_bias);
  NEED(topk_ids);
  NEED(topk_w);
  const Layout L = layout(*p, false);
  if (p->act_dtype == MOE_BF16) {
    NEED(ws);
    if (ws_bytes < L.total)
      return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu needed", ws_bytes, L.total);
  }
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != MOE_OK) return s;
  g_launches_pending = 0;
  pdl_reset();
  bool counted;
  float* part = ws ? (float*)((char*)ws + L.part) : nullptr;
  s = launch_router(*p, x, w_router, router_bias, topk_ids, topk_w, part, nullptr, &counted, (cudaStream_t)stream,
                    dev);
  if (s == MOE_OK) g_launches = g_launches_pending;
  return s;
}

moe_status moe_permute(const moe_problem* p, const void* x, const int32_t* topk_ids, const float* topk_w,
                       void* x_perm, int32_t* row_tok, float* row_w, int32_t* pos, int32_t* offs, void* ws,
                       size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("moe_permute");
  moe_status s = check(p);
  if (s != MOE_OK) return s;
  NEED(offs);
  NEED(ws);
  if (p->T > 0) {
    NEED(x);
    NEED(topk_ids);
    NEED(topk_w);
    NEED(x_perm);
    NEED(row_tok);
    NEED(row_w);
    NEED(pos);
  }
  const Layout L = layout(*p, false);
  if (ws_bytes < L.total)
    return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu needed", ws_bytes, L.total);
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != MOE_OK) return s;
  g_launches_pending = 0;
  pdl_reset();
  cudaStream_t st = (cudaStream_t)stream;
  char* w = (char*)ws;
  s = launch_dispatch(*p, topk_ids, topk_w, false, offs, row_tok, row_w, pos, nullptr, (int32_t*)(w + L.counts),
                      Schedule{}, nullptr, Schedule{}, nullptr, x, x_perm, st, dev);
  if (s == MOE_OK) g_launches = g_launches_pending;
  return s;
}

moe_status moe_expert_ffn(const moe_problem* p, const void* x_perm, const int32_t* offs, const void* w_gate,
                          const void* w_up, const void* w_down, const void* ws_gate, const void* ws_up,
                          const void* ws_down, const float* scales, void* y_perm, void* ws, size_t ws_bytes,
                          void* stream) {
  NvtxRange nvtx_("moe_expert_ffn");
  moe_status s = check(p);
  if (s != MOE_OK) return s;
  if (p->T == 0) {
    g_launches = 0;
    return MOE_OK;
  }
  NEED(x_perm);
  NEED(offs);
  NEED(y_perm);
  NEED(ws);
  ExpertWeights w{w_gate, w_up, w_down, ws_gate, ws_up, ws_down, scales};
  if ((s = check_weights(*p, w)) != MOE_OK) return s;
  const Layout L = layout(*p, false);
  if (ws_bytes < L.total)
    return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu needed", ws_bytes, L.total);
  int form;
  if ((s = choose_form(*p, &form)) != MOE_OK) return s;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != MOE_OK) return s;
  g_launches_pending = 0;
  pdl_reset();
  cudaStream_t st = (cudaStream_t)stream;
  char* wsp = (char*)ws;
  Schedule sa, sb;
  schedules(*p, form, &sa, &sb);
  int32_t* pre_a = (int32_t*)(wsp + L.pre_a);
  int32_t* pre_b = (int32_t*)(wsp + L.pre_b);
  PROF_BEGIN("tile_prefix", st);
  CUDA_TRY(launch(k_tile_prefix, 1, 1024, 0, st, offs, p->E, sa, pre_a, sb, pre_b));
  LAUNCH_CHECK("tile_prefix", st);
  DownOut o{nullptr, nullptr, nullptr, y_perm};
  s = expert_gemms(*p, form, x_perm, offs, w, pre_a, pre_b, wsp + L.h, o, st, dev);
  if (s == MOE_OK) g_launches = g_launches_pending;
  return s;
}

moe_status moe_combine(const moe_problem* p, const void* y_perm, const int32_t* pos, const float* topk_w,
                       const int32_t* offs, void* y, void* stream) {
  NvtxRange nvtx_("moe_combine");
  moe_status s = check(p);
  if (s != MOE_OK) return s;
  if (p->T == 0) {
    g_launches = 0;
    return MOE_OK;
  }
  NEED(y_perm);
  NEED(pos);
  NEED(topk_w);
  NEED(offs);
  NEED(y);
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != MOE_OK) return s;
  g_launches_pending = 0;
  pdl_reset();
  cudaStream_t st = (cudaStream_t)stream;
  PROF_BEGIN("combine", st);
  if (p->act_dtype == MOE_F32)
    CUDA_TRY(launch(k_combine<float>, (unsigned)p->T, 256, 0, st, (const float*)y_perm, pos, topk_w, offs, p->E,
                    p->k, p->d, p->T, (float*)y, rows_total(*p), dev->status));
  else
    CUDA_TRY(launch(k_combine<bf16>, (unsigned)p->T, 256, 0, st, (const bf16*)y_perm, pos, topk_w, offs, p->E,
                    p->k, p->d, p->T, (bf16*)y, rows_total(*p), dev->status));
  LAUNCH_CHECK("combine", st);
  g_launches = g_launches_pending;
  return MOE_OK;
}

// Launch the block's input prologue: x_out = zero-centred RMSNorm(x) when
// gamma is given, gate_out[t] = sigmoid(x_n[t] . gate_w) when gate_w is given.
static moe_status launch_prologue(const moe_problem& p, const void* x, const void* gamma, float eps,
                                  const void* gate_w, void* x_out, float* gate_out, cudaStream_t st) {
  const unsigned grid = (unsigned)cdiv(p.T, 8);
  PROF_BEGIN("prologue", st);
  if (p.act_dtype == MOE_F32)
    CUDA_TRY(launch(k_prologue<float>, grid, 256, 0, st, (const float*)x, (const float*)gamma, eps,
                    (const float*)gate_w, p.T, p.d, (float*)x_out, gate_out));
  else
    CUDA_TRY(launch(k_prologue<bf16>, grid, 256, 0, st, (const bf16*)x, (const bf16*)gamma, eps, (const bf16*)gate_w,
                    p.T, p.d, (bf16*)x_out, gate_out));
  LAUNCH_CHECK("prologue", st);
  return MOE_OK;
}

static moe_status block_forward(const moe_problem* p, const moe_block_options* opt, const void* x,
                                const void* w_router, const float* router_bias, const void* w_gate,
                                const void* w_up, const void* w_down, const void* ws_gate, const void* ws_up,
                                const void* ws_down, const float* scales, void* y, int32_t* topk_ids_out,
                                float* topk_w_out, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_("moe_layer_forward");
  moe_status s = check(p);
  if (s != MOE_OK) return s;
  const void* norm_w = opt ? opt->norm_weight : nullptr;
  const void* gate_w = opt ? opt->shared_gate : nullptr;
  if (norm_w && !(opt->norm_eps >= 0.f && opt->norm_eps < 1e30f))
    return fail(MOE_ERR_INVALID_ARG, "norm_eps must be finite and >= 0");
  if (p->T == 0) {
    g_launches = 0;
    return MOE_OK;
  }
  NEED(x);
  NEED(w_router);
  MAYBE(router_bias);
  NEED(y);
  MAYBE(topk_ids_out);
  MAYBE(topk_w_out);
  MAYBE(norm_w);
  MAYBE(gate_w);
  NEED(ws);
  ExpertWeights w{w_gate, w_up, w_down, ws_gate, ws_up, ws_down, scales};
  if ((s = check_weights(*p, w)) != MOE_OK) return s;
  const Layout L = layout(*p, true);
  if (ws_bytes < L.total)
    return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu needed", ws_bytes, L.total);
  int form;
  if ((s = choose_form(*p, &form)) != MOE_OK) return s;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != MOE_OK) return s;
  g_launches_pending = 0;
  pdl_reset();
  cudaStream_t st = (cudaStream_t)stream;
  char* wsp = (char*)ws;
  int32_t* ids = topk_ids_out ? topk_ids_out : (int32_t*)(wsp + L.ids);
  float* tw = topk_w_out ? topk_w_out : (float*)(wsp + L.tw);
  int32_t* counts = (int32_t*)(wsp + L.counts);
  int32_t* offs = (int32_t*)(wsp + L.offs);
  int32_t* row_tok = (int32_t*)(wsp + L.row_tok);
  float* row_w = (float*)(wsp + L.row_w);
  int32_t* pos = (int32_t*)(wsp + L.pos);
  int32_t* row_dst = (int32_t*)(wsp + L.row_dst);
  int32_t* pre_a = (int32_t*)(wsp + L.pre_a);
  int32_t* pre_b = (int32_t*)(wsp + L.pre_b);
  void* xp = wsp + L.xp;
  // the block's input: x, or its zero-centred RMSNorm; the shared expert's
  // gate (only where there is a shared expert to weight)
  const void* xin = x;
  float* gate = (gate_w && p->I_s > 0) ? (float*)(wsp + L.gate) : nullptr;
  if (norm_w || gate) {
    if ((s = launch_prologue(*p, x, norm_w, norm_w ? opt->norm_eps : 0.f, gate ? gate_w : nullptr, wsp + L.xn, gate,
                             st)) != MOE_OK)
      return s;
    if (norm_w) xin = wsp + L.xn;
  }
  bool counted;
  {
    NvtxRange r_("moe.router");
    s = launch_router(*p, xin, w_router, router_bias, ids, tw, (float*)(wsp + L.part), counts, &counted, st, dev);
  }
  if (s != MOE_OK) return s;
  Schedule sa, sb;
  schedules(*p, form, &sa, &sb);
  // the row-tiled bf16 gate/up GEMM gathers its rows from the block's input
  // (up to kGatherMaxBytes of it): the dispatch then writes no copy of them.
  // Measured: 35B shape (x 16 MB) 0.524 -> 0.484 ms; prefill (x 128 MB, in
  // the panel tile order) 10.80 -> 10.62 ms.
  GatherSrc gs;
  if (gathers_rows(*p, form)) gs = GatherSrc{xin, row_tok};
  {
    NvtxRange r_("moe.dispatch");
    s = launch_dispatch(*p, ids, tw, counted, offs, row_tok, row_w, pos, row_dst, counts, sa, pre_a, sb, pre_b, xin,
                        gs.x ? nullptr : xp, st, dev, gate);
  }
  if (s != MOE_OK) return s;
  DownOut o{xp, row_dst, row_w, nullptr};  // the slot rows reuse the dispatched-row buffer
  {
    NvtxRange r_("moe.expert_gemms");
    s = expert_gemms(*p, form, xp, offs, w, pre_a, pre_b, wsp + L.h, o, st, dev, gs);
  }
  if (s != MOE_OK) return s;
  NvtxRange r_sum_("moe.slot_sum");
  PROF_BEGIN("slot_sum", st);
  if (p->act_dtype == MOE_F32)
    CUDA_TRY(launch(k_slot_sum<float>,
                    (unsigned)p->T, 256, 0, st, (const float*)xp, pos, p->k, p->I_s > 0, p->d, (float*)y));
  else
    CUDA_TRY(launch(k_slot_sum<bf16>,
                    (unsigned)p->T, 256, 0, st, (const bf16*)xp, pos, p->k, p->I_s > 0, p->d, (bf16*)y));
  LAUNCH_CHECK("slot_sum", st);
  g_launches = g_launches_pending;
  return MOE_OK;
}

moe_status moe_layer_forward(const moe_problem* p, const void* x, const void* w_router, const float* router_bias,
                             const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate,
                             const void* ws_up, const void* ws_down, const float* scales, void* y,
                             int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes, void* stream) {
  return block_forward(p, nullptr, x, w_router, router_bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, scales, y,
                       topk_ids_out, topk_w_out, ws, ws_bytes, stream);
}

moe_status moe_block_forward(const moe_problem* p, const moe_block_options* opt, const void* x,
                             const void* w_router, const float* router_bias, const void* w_gate, const void* w_up,
                             const void* w_down, const void* ws_gate, const void* ws_up, const void* ws_down,
                             const float* scales, void* y, int32_t* topk_ids_out, float* topk_w_out, void* ws,
                             size_t ws_bytes, void* stream) {
  return block_forward(p, opt, x, w_router, router_bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, scales, y,
                       topk_ids_out, topk_w_out, ws, ws_bytes, stream);
}

moe_status moe_rmsnorm(const moe_problem* p, const void* x, const void* norm_weight, float eps, void* x_out,
                       void* stream) {
  NvtxRange nvtx_("moe_rmsnorm");
  moe_status s = check(p);
  if (s != MOE_OK) return s;
  if (!(eps >= 0.f && eps < 1e30f)) return fail(MOE_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (p->T == 0) {
    g_launches = 0;
    return MOE_OK;
  }
  NEED(x);
  NEED(norm_weight);
  NEED(x_out);
  g_launches_pending = 0;
  pdl_reset();
  if ((s = launch_prologue(*p, x, norm_weight, eps, nullptr, x_out, nullptr, (cudaStream_t)stream)) != MOE_OK)
    return s;
  g_launches = g_launches_pending;
  return MOE_OK;
}

moe_status moe_forward_plan(const moe_problem* p, int32_t* expert_form, int32_t* router_selects,
                            int32_t* gathered) {
  moe_status s = check(p);
  if (s != MOE_OK) return s;
  int form;
  if ((s = choose_form(*p, &form)) != MOE_OK) return s;
  bool router_tc;
  if ((s = choose(p->act_dtype == MOE_BF16, &router_tc)) != MOE_OK) return s;
  if (expert_form) *expert_form = form;
  if (router_selects) *router_selects = router_tc && router_fused(*p) ? 1 : 0;
  if (gathered) *gathered = gathers_rows(*p, form) ? 1 : 0;
  return MOE_OK;
}

moe_status moe_ep_expand_ids(const int32_t* counts, int32_t G, int32_t E_local, int64_t R, int32_t* ids,
                             void* stream) {
  NvtxRange nvtx_("moe_ep_expand_ids");
  if (G < 1 || E_local < 1 || (int64_t)G * E_local > kEpMaxBlocks)
    return fail(MOE_ERR_INVALID_ARG, "G = %d, E_local = %d: need G, E_local >= 1 and G * E_local <= %d", G, E_local,
                kEpMaxBlocks);
  if (R < 0 || R > INT32_MAX) return fail(MOE_ERR_INVALID_ARG, "R = %lld out of range", (long long)R);
  if (R == 0) {
    g_launches = 0;
    return MOE_OK;
  }
  NEED(counts);
  NEED(ids);
  DeviceInfo* dev;
  moe_status s;
  if ((s = device_info(&dev)) != MOE_OK) return s;
  g_launches_pending = 0;
  pdl_reset();
  cudaStream_t st = (cudaStream_t)stream;
  const unsigned grid = (unsigned)std::min<int64_t>(cdiv(R, 256), 4 * (int64_t)dev->sms);
  PROF_BEGIN("ep_expand_ids", st);
  CUDA_TRY(launch(k_ep_expand_ids, grid, 256, 0, st, counts, G * E_local, (int)E_local, R, ids, dev->status));
  LAUNCH_CHECK("ep_expand_ids", st);
  g_launches = g_launches_pending;
  return MOE_OK;
}

}  // extern "C"

// ============================================================== router without a workspace
// For callers that cannot allocate device memory themselves (see
// moe_router_topk_static in moe.h): the logit partials go to a fixed array
// that every device holding this library keeps for the life of the process.
static __device__ __align__(256) unsigned char g_router_scratch[MOE_ROUTER_STATIC_SCRATCH_BYTES];
static void* g_router_scratch_ptr[kMaxDevices];
static std::mutex g_router_scratch_mu;

// Device address of this device's copy of the array (host code may not use
// the symbol itself: on the host it names a stand-in, not device memory).
static moe_status router_scratch(void** out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_router_scratch_mu);
  if (!g_router_scratch_ptr[dev]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_router_scratch);
    if (e != cudaSuccess || !ptr)
      return fail(MOE_ERR_CUDA, "cudaGetSymbolAddress(router scratch): %s", cudaGetErrorString(e));
    g_router_scratch_ptr[dev] = ptr;
  }
  *out = g_router_scratch_ptr[dev];
  return MOE_OK;
}

extern "C" moe_status moe_router_topk_static(const moe_problem* p, const void* x, const void* w_router,
                                             const float* router_bias, int32_t* topk_ids, float* topk_w,
                                             void* stream) {
  NvtxRange nvtx_("moe_router_topk_static");
  moe_status s = check(p);
  if (s != MOE_OK) return s;
  if (p->T == 0) {
    g_launches = 0;
    return MOE_OK;
  }
  NEED(x);
  NEED(w_router);
  MAYBE(router_bias);
  NEED(topk_ids);
  NEED(topk_w);
  const size_t need = router_scratch_bytes(*p);
  if (need > (size_t)MOE_ROUTER_STATIC_SCRATCH_BYTES)
    return fail(MOE_ERR_UNSUPPORTED,
                "router needs %zu bytes of scratch; the built-in array holds %zu (use moe_router_topk with a workspace)",
                need, (size_t)MOE_ROUTER_STATIC_SCRATCH_BYTES);
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != MOE_OK) return s;
  void* scratch = nullptr;
  if ((s = router_scratch(&scratch)) != MOE_OK) return s;
  g_launches_pending = 0;
  pdl_reset();
  bool counted;
  s = launch_router(*p, x, w_router, router_bias, topk_ids, topk_w, (float*)scratch, nullptr, &counted,
                    (cudaStream_t)stream, dev);
  if (s == MOE_OK) g_launches = g_launches_pending;
  return s;
}
