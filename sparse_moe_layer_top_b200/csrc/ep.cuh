// ep.cuh -- expert parallelism, receive side.
//
// The block split over G ranks, rank g holding the contiguous experts
// [g * E_l, (g + 1) * E_l): a rank's dispatch (a stable sort by expert) leaves
// the rows bound for each rank contiguous and grouped by expert, so the rows
// a rank receives are the blocks (source s, local expert e) in that order.
// k_ep_expand_ids gives every received row its local expert, which a k = 1
// dispatch then regroups by expert across sources.
//
// counts[s * E_l + e] = rows of source s for local expert e (n = G * E_l
// blocks).  Each CTA builds the inclusive prefix of the counts in shared
// memory; row r takes the first block b with prefix[b] > r and e = b % E_l.
// A negative count (read as 0), or a row past the counts' total (written -1,
// which the following dispatch drops as an out-of-range id), sets the device
// status.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kEpMaxBlocks = 4096;  // largest G * E_l

__global__ void __launch_bounds__(256) k_ep_expand_ids(const int32_t* __restrict__ counts, int n, int E_l,
                                                        int64_t R, int32_t* __restrict__ ids, unsigned* status) {
  pdl_begin();  // after the previous kernel in the stream (programmatic launch)
  __shared__ int64_t pre[kEpMaxBlocks];
  __shared__ int64_t part[256];
  const int tid = threadIdx.x;
  const int per = (n + 255) / 256;  // <= 16 blocks per thread
  const int b0 = min(n, tid * per), b1 = min(n, b0 + per);
  int64_t s = 0;
  bool bad = false;
  for (int b = b0; b < b1; ++b) {
    const int c = __ldg(counts + b);
    bad |= c < 0;
    s += max(c, 0);
    pre[b] = s;
  }
  part[tid] = s;
  __syncthreads();
  if (tid == 0) {  // exclusive scan of the 256 partial sums
    int64_t a = 0;
    for (int i = 0; i < 256; ++i) {
      const int64_t v = part[i];
      part[i] = a;
      a += v;
    }
  }
  __syncthreads();
  for (int b = b0; b < b1; ++b) pre[b] += part[tid];
  __syncthreads();
  if (bad && blockIdx.x == 0) atomicCAS(status, 0u, (unsigned)kStatusBadCount);
  const int64_t total = pre[n - 1];
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + tid; r < R; r += (int64_t)gridDim.x * blockDim.x) {
    if (r >= total) {
      ids[r] = -1;
      atomicCAS(status, 0u, (unsigned)kStatusBadCount);
      continue;
    }
    int lo = 0, hi = n - 1;  // the first block whose inclusive prefix exceeds r
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] > r) hi = mid; else lo = mid + 1;
    }
    ids[r] = lo % E_l;
  }
}

}  // namespace moe
