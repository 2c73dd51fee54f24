// route.cu -- ISA dynamic query grouping (stage 2, second half).
//
// "Lightning Unified Video Editing via In-Context Sparse Attention",
// abstract: high-error queries go to full attention, the rest to 0-th order
// Taylor attention, with query sharpness as the error proxy.  Reading: per
// (b, h) the n_route queries of largest sharpness (ties: lower index first)
// are routed; both buckets are written in ascending token order.
//
// One 1024-thread CTA per (b, h):
//  0. the head's N sharpness values are copied once into shared memory when
//     they fit (N <= kRouteSmemKeys), else every pass reads them from L2;
//  1. exact radix select (4 passes of 8 bits, MSB first) of the n_route-th
//     largest sharpness bit pattern T (sharpness is positive, so its bit
//     pattern orders like its value); the histogram has one copy per lane,
//     rows padded so that equal bins of a warp fall in distinct banks
//     (sharpness values cluster in a few exponent bins);
//  2. ordered compaction: thread t visits i = 1024 j + t; per (j, warp) the
//     counts of equal-to-T and of routed keys are scanned CTA-wide in (j,
//     warp) order, so every key gets its rank among equal keys and then its
//     output slot from a warp ballot; both buckets are written coalesced.
#include "block_scan.cuh"
#include "isa_internal.h"

namespace isa {

// Dynamic shared memory: the resident keys (N words, when they fit) and two
// count arrays of ceil(N/1024)*32 ints; the static part (histograms, scan
// scratch) is about 34 KB of the 227 KB a CTA may hold.
constexpr int kRouteSmemBudget = 227 * 1024 - 36 * 1024;
inline int route_count_words(int N) { return 2 * ((N + 1023) / 1024) * 32; }

template <bool RESIDENT>
__global__ void __launch_bounds__(1024) route_kernel(const float* __restrict__ sharp, int32_t* __restrict__ routed,
                                                     int32_t* __restrict__ taylor, int N, int n_route,
                                                     int* __restrict__ status) {
  extern __shared__ unsigned dyn_sm[];
  __shared__ int hist[32][257];  // per lane, padded
  __shared__ int tot[256];
  __shared__ unsigned sh_sel;
  __shared__ int sh_rem;
  __shared__ int scan_ws[33];
  const int bh = blockIdx.x, tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const unsigned* u = reinterpret_cast<const unsigned*>(sharp + static_cast<size_t>(bh) * N);
  int32_t* rout = routed + static_cast<size_t>(bh) * n_route;
  int32_t* tout = taylor + static_cast<size_t>(bh) * (N - n_route);
  const int iters = (N + 1023) / 1024;
  unsigned* keys_sm = dyn_sm;
  int* ceq = reinterpret_cast<int*>(dyn_sm + (RESIDENT ? N : 0));  // per (j, warp): equal keys, then offsets
  int* csel = ceq + iters * 32;                                     // per (j, warp): routed keys, then offsets
  if constexpr (RESIDENT) {
    for (int i = tid; i < N; i += 1024) keys_sm[i] = __ldg(u + i);
    __syncthreads();
  }
  auto key = [&](int i) -> unsigned {
    if constexpr (RESIDENT) return keys_sm[i];
    else return __ldg(u + i);
  };

  unsigned T = 0u;
  int need_eq = 0;
  const bool partial = n_route > 0 && n_route < N;
  if (partial) {
    unsigned prefix = 0u, pmask = 0u;
    int remaining = n_route;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int i = tid; i < 32 * 257; i += 1024) (&hist[0][0])[i] = 0;
      __syncthreads();
      for (int i = tid; i < N; i += 1024) {
        const unsigned x = key(i);
        if ((x & pmask) == prefix) atomicAdd(&hist[lane][(x >> shift) & 255u], 1);
      }
      __syncthreads();
      if (tid < 256) {
        int s = 0;
#pragma unroll 8
        for (int l = 0; l < 32; ++l) s += hist[l][tid];
        tot[tid] = s;
      }
      __syncthreads();
      if (w == 0) {
        // lane l owns bins 255-8l .. 248-8l (descending); find the bin where
        // the count from the top first reaches `remaining`
        int s = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) s += tot[255 - 8 * lane - k];
        int incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += n;
        }
        const int before = incl - s;
        if (before < remaining && incl >= remaining) {  // exactly one lane
          int cum = before;
          for (int k = 0; k < 8; ++k) {
            const int bin = 255 - 8 * lane - k;
            if (cum + tot[bin] >= remaining) {
              sh_sel = static_cast<unsigned>(bin);
              sh_rem = remaining - cum;
              break;
            }
            cum += tot[bin];
          }
        }
      }
      __syncthreads();
      prefix |= sh_sel << shift;
      pmask |= 255u << shift;
      remaining = sh_rem;
      __syncthreads();
    }
    T = prefix;
    need_eq = remaining;
  }

  // CTA-wide exclusive scan of cnt[0 .. iters*32) in (j, warp) order
  auto scan_counts = [&](int* cnt) {
    const int n = iters * 32;
    const int per = (n + 1023) / 1024;
    int loc = 0;
    for (int k = 0; k < per; ++k) {
      const int e = tid * per + k;
      if (e < n) loc += cnt[e];
    }
    int total;
    int run = block_exclusive_sum_1024(loc, scan_ws, total);
    for (int k = 0; k < per; ++k) {
      const int e = tid * per + k;
      if (e < n) {
        const int c = cnt[e];
        cnt[e] = run;
        run += c;
      }
    }
    __syncthreads();
  };

  // rank of each key among the keys equal to T (index order)
  if (partial) {
    for (int j = 0; j < iters; ++j) {
      const int i = j * 1024 + tid;
      const unsigned bal = __ballot_sync(0xffffffffu, i < N && key(i) == T);
      if (lane == 0) ceq[j * 32 + w] = __popc(bal);
    }
    __syncthreads();
    scan_counts(ceq);
  }
  const unsigned lt = (1u << lane) - 1u;
  auto selected = [&](int j, int i) -> bool {  // warp-collective
    if (n_route <= 0) return false;
    if (n_route >= N) return i < N;
    const unsigned x = i < N ? key(i) : 0u;
    const bool eq = i < N && x == T;
    const unsigned beq = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = ceq[j * 32 + w] + __popc(beq & lt);
    return i < N && (x > T || (eq && eq_rank < need_eq));
  };
  // routed count per (j, warp), then their exclusive offsets
  for (int j = 0; j < iters; ++j) {
    const unsigned bal = __ballot_sync(0xffffffffu, selected(j, j * 1024 + tid));
    if (lane == 0) csel[j * 32 + w] = __popc(bal);
  }
  __syncthreads();
  scan_counts(csel);
  for (int j = 0; j < iters; ++j) {
    const int i = j * 1024 + tid;
    const bool sel = selected(j, i);
    const unsigned bal = __ballot_sync(0xffffffffu, sel);
    const int r = csel[j * 32 + w] + __popc(bal & lt);  // routed keys before i
    if (i < N) {
      // Counts are exact by construction; the guards only keep a corrupted
      // input (e.g. NaN sharpness) from writing past the buckets.
      if (sel) {
        if (r < n_route) rout[r] = i; else atomicCAS(status, 0, 1);
      } else {
        if (i - r < N - n_route) tout[i - r] = i; else atomicCAS(status, 0, 1);
      }
    }
  }
}

cudaError_t launch_route(const float* sharp, int32_t* routed, int32_t* taylor, int BH, int N, int n_route,
                         int* status, cudaStream_t st) {
  if (BH <= 0 || N <= 0) return cudaSuccess;
  const size_t counts = static_cast<size_t>(route_count_words(N)) * 4;
  const size_t resident = static_cast<size_t>(N) * 4 + counts;
  cudaError_t e;
  if (resident <= static_cast<size_t>(kRouteSmemBudget)) {
    e = cudaFuncSetAttribute(route_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kRouteSmemBudget);
    if (e != cudaSuccess) return e;
    route_kernel<true><<<BH, 1024, resident, st>>>(sharp, routed, taylor, N, n_route, status);
  } else {
    if (counts > static_cast<size_t>(kRouteSmemBudget)) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(route_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kRouteSmemBudget);
    if (e != cudaSuccess) return e;
    route_kernel<false><<<BH, 1024, counts, st>>>(sharp, routed, taylor, N, n_route, status);
  }
  return cudaGetLastError();
}

}  // namespace isa
