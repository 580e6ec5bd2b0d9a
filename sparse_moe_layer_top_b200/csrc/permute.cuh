// permute.cuh -- dispatch of (token, slot) pairs to expert-contiguous rows.
//
// The token "is sent to" its k experts (Qwen3.6 explainer, router paragraph).
// Here that is a stable counting sort by expert over chunks of kChunkTokens
// tokens (chunk c = the pairs of tokens c*kChunkTokens ...):
//   counts      per-chunk histogram over the E experts (written by k_topk, or
//               by k_count when the routing comes from elsewhere);
//   k_dispatch  kSubBlocks blocks per chunk: column sums of the histograms
//               give the group offsets offs[E+2] and each block's first row
//               per expert (block 0 also writes the tile prefix sums of the
//               GEMM schedules); within a block, warps take consecutive token
//               ranges and rank equal experts by warp match masks, so row
//               order = (token, slot) order; the shared-expert rows are
//               written too, and each warp then copies its tokens' x rows into
//               their dispatched rows (16-byte vectors).
// Group E (the shared expert) is every token in order at rows offs[E] + t.
#pragma once
#include "common.cuh"
#include "router.cuh"

namespace moe {

constexpr int kScatterWarps = 8;   // warps of k_dispatch (256 threads)
constexpr int kMaxE = 512;

__global__ void __launch_bounds__(256) k_count(const int32_t* __restrict__ ids, int64_t T, int k, int E,
                                               int32_t* __restrict__ counts, unsigned* status) {
  pdl_begin();  // after the previous kernel in the stream (programmatic launch)
  __shared__ int32_t h[kMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int64_t n = T * k;
  const int64_t c0 = (int64_t)blockIdx.x * kChunkTokens * k;
  const int64_t c1 = min(n, c0 + (int64_t)kChunkTokens * k);
  for (int64_t i = c0 + threadIdx.x; i < c1; i += blockDim.x) {
    int e = __ldg(ids + i);
    if ((unsigned)e < (unsigned)E) atomicAdd(&h[e], 1);
    else atomicCAS(status, 0u, (unsigned)kStatusBadExpertId);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(int64_t)blockIdx.x * E + e] = h[e];
}

// Inclusive block-wide scan of one int per thread (blockDim.x == 1024).
__device__ __forceinline__ int block_incl_scan(int v, int* sm_warp) {
  int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) sm_warp[w] = v;
  __syncthreads();
  if (w == 0) {
    int s = sm_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int t = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += t;
    }
    sm_warp[lane] = s;
  }
  __syncthreads();
  if (w > 0) v += sm_warp[w - 1];
  __syncthreads();
  return v;
}

// Tile prefix of one schedule from the group sizes (E+1 groups, one thread each).
// prefix[E + 2] is the GEMM's tile-claim counter, zeroed here (see TcGemmArgs::sched).
// A schedule that splits off its small groups (Schedule::small_rows) has
// prefix[0 .. E+1] over the other groups and prefix[E+3 .. 2E+4] over the
// small ones (each counting only its own groups' tiles).
__device__ __forceinline__ void write_tile_prefix(const Schedule& s, int E, int rows_g, int32_t* prefix,
                                                  int* sm_warp) {
  const int g = threadIdx.x;
  const int tiles = (g <= E) ? sched_tiles(s, g, E, rows_g) : 0;
  const bool small = g <= E && sched_small(s, rows_g);
  for (int part = 0; part < (s.small_rows > 0 ? 2 : 1); ++part) {
    int32_t* q = part ? prefix + E + 3 : prefix;
    const int mine = small == (part == 1) ? tiles : 0;
    const int incl = block_incl_scan(mine, sm_warp);
    if (g <= E) q[g] = incl - mine;
    if (g == E) q[E + 1] = incl;
  }
  if (g == E) prefix[E + 2] = 0;
}

// Tile prefixes from caller-supplied group offsets (the expert stage alone).
__global__ void __launch_bounds__(1024) k_tile_prefix(const int32_t* __restrict__ offs, int E, Schedule sa,
                                                      int32_t* __restrict__ prefix_a, Schedule sb,
                                                      int32_t* __restrict__ prefix_b) {
  pdl_begin();  // after the previous kernel in the stream (programmatic launch)
  __shared__ int sm_warp[32];
  int g = threadIdx.x;
  int rows = g <= E ? offs[g + 1] - offs[g] : 0;
  if (prefix_a) write_tile_prefix(sa, E, rows, prefix_a, sm_warp);
  if (prefix_b) write_tile_prefix(sb, E, rows, prefix_b, sm_warp);
}

// Inclusive scan over a block of 256 threads, each holding two consecutive
// values (v0, v1) of a 512-entry sequence; returns the inclusive sums.
__device__ __forceinline__ int2 block256_scan2(int v0, int v1, int* sm_warp) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int v = v0 + v1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) sm_warp[w] = v;
  __syncthreads();
  int before = 0;
  for (int i = 0; i < w; ++i) before += sm_warp[i];
  __syncthreads();
  const int incl1 = before + v;  // through v1
  return make_int2(incl1 - v1, incl1);
}

// Scan, scatter and copy in one kernel.  Block b takes kBlockTokens tokens
// of chunk c = b / kSubBlocks: it sums the chunk histograms of every expert over
// all chunks and over the chunks before c, scans the totals into the group
// offsets, adds the pairs of its chunk's earlier tokens, and then places its
// own pairs in (token, slot) order.  Block 0 also writes offs and the tile
// prefixes of the two GEMM schedules.  With xp given, each warp then copies its
// tokens' rows of x to their k dispatched rows and their shared-expert row (a
// row is read once and written k + 1 times).  256 threads, E <= 512.
constexpr int kSubBlocks = 4;                              // blocks per histogram chunk
constexpr int kBlockTokens = kChunkTokens / kSubBlocks;    // 32 tokens per block
constexpr int kWarpTokens = kBlockTokens / kScatterWarps;  // 4 tokens per warp
__global__ void __launch_bounds__(kScatterWarps * 32) k_dispatch(
    const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int64_t T, int k, int E,
    const int32_t* __restrict__ counts, int nchunks, int has_shared, int32_t* __restrict__ offs, Schedule sa,
    int32_t* __restrict__ prefix_a, Schedule sb, int32_t* __restrict__ prefix_b, int32_t* __restrict__ row_tok,
    float* __restrict__ row_w, int32_t* __restrict__ pos, int32_t* __restrict__ row_dst,
    const float* __restrict__ shared_gate, const uint4* __restrict__ x, int vec_per_row, uint4* __restrict__ xp,
    unsigned* status) {
  pdl_begin();  // after the previous kernel in the stream (programmatic launch)
  __shared__ int32_t wb[kScatterWarps][kMaxE];
  __shared__ int32_t s_base[kMaxE];
  __shared__ int32_t s_dst[kScatterWarps][kWarpTokens * kMaxK];  // dispatched row of each of a warp's pairs
  __shared__ int sm_warp[32];
  __shared__ int s_R, s_tot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x / kSubBlocks, sub = blockIdx.x % kSubBlocks;
  const int64_t t_blk = (int64_t)c * kChunkTokens + (int64_t)sub * kBlockTokens;  // first token of the block
  // 1. per expert: total over all chunks, and over the chunks before this one
  int tot[2] = {0, 0}, pre[2] = {0, 0};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int e = 2 * threadIdx.x + h;
    if (e < E) {
#pragma unroll 8
      for (int cc = 0; cc < nchunks; ++cc) {
        const int v = __ldg(counts + (int64_t)cc * E + e);
        tot[h] += v;
        pre[h] += cc < c ? v : 0;
      }
    }
  }
  // 2. group offsets
  const int2 inc = block256_scan2(tot[0], tot[1], sm_warp);
  const int start0 = inc.x - tot[0], start1 = inc.y - tot[1];
  if (threadIdx.x == blockDim.x - 1) s_R = inc.y;  // routed rows = sum of all totals
  if (2 * threadIdx.x < E) s_base[2 * threadIdx.x] = start0 + pre[0];
  if (2 * threadIdx.x + 1 < E) s_base[2 * threadIdx.x + 1] = start1 + pre[1];
  __syncthreads();
  const int R = s_R;
  if (blockIdx.x == 0) {
    if (2 * threadIdx.x < E) offs[2 * threadIdx.x] = start0;
    if (2 * threadIdx.x + 1 < E) offs[2 * threadIdx.x + 1] = start1;
    if (threadIdx.x == 0) {
      offs[E] = R;
      offs[E + 1] = R + (has_shared ? (int)T : 0);
    }
    // tile prefixes over the E+1 groups (group E: the shared expert); with
    // E == 512 the shared group is one past the 512 the block scans
    // (a schedule that splits off its small groups gets a second prefix over
    // them at pf + E + 3, as write_tile_prefix lays it out)
    for (int which = 0; which < 2; ++which) {
      const Schedule& sc = which ? sb : sa;
      int32_t* pf = which ? prefix_b : prefix_a;
      if (!pf) continue;
      for (int part = 0; part < (sc.small_rows > 0 ? 2 : 1); ++part) {
        int32_t* q = part ? pf + E + 3 : pf;
        int tl[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int g = 2 * threadIdx.x + h;
          const int rows = g < E ? tot[h] : (has_shared ? (int)T : 0);
          const int n = g <= E ? sched_tiles(sc, g, E, rows) : 0;
          tl[h] = sched_small(sc, rows) == (part == 1) ? n : 0;
        }
        const int2 ti = block256_scan2(tl[0], tl[1], sm_warp);
        if (2 * threadIdx.x <= E) q[2 * threadIdx.x] = ti.x - tl[0];
        if (2 * threadIdx.x + 1 <= E) q[2 * threadIdx.x + 1] = ti.y - tl[1];
        if (threadIdx.x == blockDim.x - 1) s_tot = ti.y;
        __syncthreads();
        if (threadIdx.x == 0) {
          if (E < kMaxE) {
            q[E + 1] = s_tot;
          } else {
            const int sh_rows = has_shared ? (int)T : 0;
            q[E] = s_tot;
            q[E + 1] = s_tot + (sched_small(sc, sh_rows) == (part == 1) ? sched_tiles(sc, E, E, sh_rows) : 0);
          }
          if (part == 0) pf[E + 2] = 0;  // the GEMM's tile-claim counter
        }
        __syncthreads();
      }
    }
  }
  // 3. pairs of the chunk's tokens before this block: they precede ours in every group
  const int64_t n = T * k;
  for (int64_t i = (int64_t)c * kChunkTokens * k + threadIdx.x; i < min(n, t_blk * k); i += blockDim.x) {
    const int e = __ldg(ids + i);
    if ((unsigned)e < (unsigned)E) atomicAdd(&s_base[e], 1);
  }
  __syncthreads();
  // 4. the block's pairs: per-warp histograms, their scan, then ranks by match masks
  const int64_t s0 = (t_blk + (int64_t)warp * kWarpTokens) * k;
  const int64_t s1 = min(n, s0 + (int64_t)kWarpTokens * k);
  for (int e = lane; e < E; e += 32) wb[warp][e] = 0;
  __syncwarp();
  for (int64_t i = s0 + lane; i < s1; i += 32) {
    const int e = __ldg(ids + i);
    if ((unsigned)e < (unsigned)E) atomicAdd(&wb[warp][e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = s_base[e];
    for (int w = 0; w < kScatterWarps; ++w) {
      const int v = wb[w][e];
      wb[w][e] = run;
      run += v;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int64_t b = s0; b < s1; b += 32) {
    const int64_t i = b + lane;
    const bool act = i < s1;
    const int e = act ? __ldg(ids + i) : -1;
    bool ok = act && (unsigned)e < (unsigned)E;
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
    int r = 0;
    if (ok) r = wb[warp][e] + __popc(peers & lt);
    __syncwarp();
    if (ok && (peers & lt) == 0) wb[warp][e] += __popc(peers);
    __syncwarp();
    if (ok && !in_range(r, R, status, kSiteDispatchRow)) ok = false;  // (checking build) the pair is dropped
    if (ok) {
      const int64_t t = i / k;
      row_tok[r] = (int32_t)t;
      row_w[r] = __ldg(topk_w + i);
      pos[i] = r;
      if (row_dst) row_dst[r] = (int32_t)(t * (k + 1) + (i - t * k));
    } else if (act) {
      pos[i] = -1;
    }
    if (act) s_dst[warp][i - s0] = ok ? r : -1;
  }
  if (has_shared) {
    for (int64_t t = t_blk + threadIdx.x; t < min(T, t_blk + kBlockTokens); t += blockDim.x) {
      row_tok[R + t] = (int32_t)t;
      row_w[R + t] = shared_gate ? __ldg(shared_gate + t) : 1.0f;  // the shared expert's weight
      if (row_dst) row_dst[R + t] = (int32_t)(t * (k + 1) + k);
    }
  }
  if (!xp) return;
  // 5. each warp copies its tokens' rows: read once, written to the token's
  //    dispatched rows and its shared-expert row, four 16-byte vectors per lane
  //    in flight
  __syncwarp();
  for (int tt = 0; tt < kWarpTokens; ++tt) {
    const int64_t t = t_blk + (int64_t)warp * kWarpTokens + tt;
    if (t >= T) break;
    const uint4* src = x + t * vec_per_row;
    for (int v0 = 0; v0 < vec_per_row; v0 += 128) {
      uint4 a[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < vec_per_row) a[u] = __ldg(src + v);
      }
      for (int j = 0; j <= k; ++j) {
        int64_t r;
        if (j < k) {
          r = s_dst[warp][tt * k + j];
          if (r < 0) continue;
        } else {
          if (!has_shared) break;
          r = R + t;
        }
        if (!in_range(r, R + (has_shared ? T : 0), status, kSiteCopyRow)) continue;
        uint4* dst = xp + r * vec_per_row;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = v0 + u * 32 + lane;
          if (v < vec_per_row) dst[v] = a[u];
        }
      }
    }
  }
}

}  // namespace moe
