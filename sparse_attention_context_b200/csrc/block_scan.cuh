// block_scan.cuh -- ordered flag ranking across a 1024-thread CTA: ballot +
// popc inside each warp, one shared-memory scan of the 32 warp totals.
#pragma once
#include <cstdint>

namespace isa {

// Exclusive prefix count of `flag` over the CTA in thread order; `total`
// receives the CTA-wide count.  `ws` is >= 33 ints of shared memory.  Every
// thread of the CTA (blockDim.x == 1024) must call it.
__device__ __forceinline__ int block_rank_1024(bool flag, int* ws, int& total) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) ws[w] = __popc(bal);
  __syncthreads();
  if (w == 0) {
    int v = ws[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += n;
    }
    ws[lane] = v;  // inclusive
  }
  __syncthreads();
  const int off = w ? ws[w - 1] : 0;
  total = ws[31];
  __syncthreads();  // ws may be reused right after
  return off + in_warp;
}

// Exclusive prefix sum of `v` over the CTA in thread order; `total`
// receives the CTA-wide sum.  Same calling rules as block_rank_1024.
__device__ __forceinline__ int block_exclusive_sum_1024(int v, int* ws, int& total) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) ws[w] = incl;
  __syncthreads();
  if (w == 0) {
    int t = ws[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += n;
    }
    ws[lane] = t;  // inclusive over warps
  }
  __syncthreads();
  const int off = w ? ws[w - 1] : 0;
  total = ws[31];
  __syncthreads();  // ws may be reused right after
  return off + incl - v;
}

}  // namespace isa
