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
//
// route_cluster_kernel (used whenever a head's keys fit): the same select
// and compaction spread over a cluster of 8 CTAs per (b, h), each holding a
// contiguous eighth of the head's keys in shared memory.  Every radix pass
// builds the chunk's histogram, the cluster synchronises, and every CTA
// sums the 8 histograms over distributed shared memory and takes the same
// (deterministic) decision; the compaction offsets of a chunk come from
// the greater-than and equal-to-T counts of the chunks before it.  The
// index sets are identical to the single-CTA kernel's.
#include <cooperative_groups.h>

#include "block_scan.cuh"
#include "isa_internal.h"

namespace isa {

namespace cg = cooperative_groups;

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

constexpr int kRouteCluster = 8;    // CTAs per (b, h)
constexpr int kRouteCT = 512;       // threads per CTA
constexpr int kRouteNW = kRouteCT / 32;
constexpr int kRouteChunkCap = (200 * 1024) / 4 - 2048;  // keys per CTA held in shared memory

// Exclusive prefix sum of v over the kRouteCT threads in thread order, on
// 64-bit values (two 32-bit counts packed, low + high, which never carry);
// `total` receives the CTA-wide sum.  ws: >= kRouteNW words of shared
// memory, free for reuse when this returns.
__device__ __forceinline__ unsigned long long block_exclusive_sum_512(unsigned long long v, unsigned long long* ws,
                                                                      unsigned long long& total) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  unsigned long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) ws[w] = incl;
  __syncthreads();
  unsigned long long before = 0ull, all = 0ull;
#pragma unroll
  for (int ww = 0; ww < kRouteNW; ++ww) {  // every thread sums the warp totals (16 words, broadcast reads)
    const unsigned long long t = ws[ww];
    before += ww < w ? t : 0ull;
    all += t;
  }
  total = all;
  __syncthreads();  // ws may be reused right after
  return before + incl - v;
}

__global__ void __cluster_dims__(kRouteCluster, 1, 1) __launch_bounds__(kRouteCT)
    route_cluster_kernel(const float* __restrict__ sharp, int32_t* __restrict__ routed, int32_t* __restrict__ taylor,
                         int N, int n_route, int* __restrict__ status) {
  cg::cluster_group cl = cg::this_cluster();
  const int rank = static_cast<int>(cl.block_rank());
  const int bh = static_cast<int>(blockIdx.x) / kRouteCluster;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int chunk = (N + kRouteCluster - 1) / kRouteCluster;
  const int c0 = min(N, rank * chunk);
  const int n = max(0, min(N, c0 + chunk) - c0);  // keys of this CTA: [c0, c0 + n)
  const int trips = (chunk + kRouteCT - 1) / kRouteCT;
  extern __shared__ unsigned rkeys[];                        // [chunk]
  int* cgt = reinterpret_cast<int*>(rkeys + chunk);          // [trips][NW] keys > T, then their offsets
  int* ceq = cgt + trips * kRouteNW;                         // [trips][NW] keys == T, then their offsets
  __shared__ int whist[kRouteNW][257];                       // per warp, padded
  // every chunk's histogram, pushed by its CTA into all CTAs of the cluster
  // (remote stores before the cluster barrier; local reads after it), by
  // pass parity
  __shared__ int hist_all[2][kRouteCluster][256];
  __shared__ int tot[256];                                   // cluster-wide histogram of the pass
  __shared__ int cnt_all[kRouteCluster][2];                  // every chunk's keys > T, keys == T (pushed)
  __shared__ unsigned sh_sel[2];                             // each pass's decision, by pass parity
  __shared__ int sh_rem[2];
  __shared__ int sh_off[2];                                  // routed keys before this chunk, equal keys it takes
  __shared__ unsigned long long scan_ws[kRouteNW];
  const unsigned* u = reinterpret_cast<const unsigned*>(sharp + static_cast<size_t>(bh) * N);
  for (int i = tid; i < n; i += kRouteCT) rkeys[i] = __ldg(u + c0 + i);
  for (int e = tid; e < kRouteNW * 257; e += kRouteCT) (&whist[0][0])[e] = 0;
  __syncthreads();

  // Radix select, 4 passes of 8 bits.  Per pass: the warps' histograms
  // (barrier), their sum into this chunk's histogram by 256 threads, which
  // also clear them for the next pass (cluster barrier: every chunk's
  // histogram is complete, and every read of the buffer two passes back is
  // done), warp 0's decision over the 8 chunks (barrier).  The decision
  // words are double-buffered, so no barrier separates their reads from
  // the next pass's writes.
  unsigned T = 0u;
  int need_eq = 0;
  const bool partial = n_route > 0 && n_route < N;  // uniform over the cluster
  if (partial) {
    unsigned prefix = 0u, pmask = 0u;
    int remaining = n_route;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass, buf = pass & 1;
      for (int i = tid; i < n; i += kRouteCT) {
        const unsigned x = rkeys[i];
        if ((x & pmask) == prefix) atomicAdd(&whist[w][(x >> shift) & 255u], 1);
      }
      __syncthreads();
      if (tid < 256) {
        int t = 0;
#pragma unroll
        for (int ww = 0; ww < kRouteNW; ++ww) {
          t += whist[ww][tid];
          whist[ww][tid] = 0;
        }
        const uint32_t mine = static_cast<uint32_t>(__cvta_generic_to_shared(&hist_all[buf][rank][tid]));
#pragma unroll
        for (int r = 0; r < kRouteCluster; ++r)
          asm volatile("{\n\t.reg .b32 ra;\n\tmapa.shared::cluster.u32 ra, %0, %1;\n\tst.shared::cluster.u32 [ra], %2;\n\t}" ::"r"(mine), "r"(r), "r"(t)
                       : "memory");
      }
      // every chunk's histogram of this pass has arrived everywhere (and every
      // read of the other buffer, two passes back, is done)
      cl.sync();
      if (tid < 256) {
        int t = 0;
#pragma unroll
        for (int r = 0; r < kRouteCluster; ++r) t += hist_all[buf][r][tid];
        tot[tid] = t;
      }
      __syncthreads();
      if (w == 0) {
        // lane l owns bins 255-8l .. 248-8l (descending): the bin where the
        // count from the top reaches `remaining`
        int tl[8];
        int s = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          tl[k] = tot[255 - 8 * lane - k];
          s += tl[k];
        }
        int incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int nn = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += nn;
        }
        const int before = incl - s;
        if (before < remaining && incl >= remaining) {  // exactly one lane
          int cum = before;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if (cum + tl[k] >= remaining) {
              sh_sel[buf] = static_cast<unsigned>(255 - 8 * lane - k);
              sh_rem[buf] = remaining - cum;
              break;
            }
            cum += tl[k];
          }
        }
      }
      __syncthreads();
      prefix |= sh_sel[buf] << shift;
      pmask |= 255u << shift;
      remaining = sh_rem[buf];
    }
    T = prefix;
    need_eq = remaining;
  }

  // Ordered compaction.  Per (trip, warp): keys above T and keys equal to
  // T; one exclusive scan of both (packed) in (trip, warp) order gives
  // every key its counts of greater and of equal keys before it in the
  // chunk.  Equal keys are routed in index order up to need_eq over the
  // head, so a key's routed keys before it in the chunk are
  // gt_before + min(eq_before, take_eq).
  for (int j = 0; j < trips; ++j) {
    const int i = j * kRouteCT + tid;
    const unsigned x = i < n ? rkeys[i] : 0u;
    const unsigned bgt = __ballot_sync(0xffffffffu, partial && i < n && x > T);
    const unsigned beq = __ballot_sync(0xffffffffu, partial && i < n && x == T);
    if (lane == 0) {
      cgt[j * kRouteNW + w] = __popc(bgt);
      ceq[j * kRouteNW + w] = __popc(beq);
    }
  }
  __syncthreads();
  {
    const int ne = trips * kRouteNW;
    const int per = (ne + kRouteCT - 1) / kRouteCT;
    unsigned long long loc = 0ull;
    for (int k = 0; k < per; ++k) {
      const int e = tid * per + k;
      if (e < ne) loc += static_cast<unsigned long long>(cgt[e]) | (static_cast<unsigned long long>(ceq[e]) << 32);
    }
    unsigned long long total;
    unsigned long long run = block_exclusive_sum_512(loc, scan_ws, total);
    for (int k = 0; k < per; ++k) {
      const int e = tid * per + k;
      if (e < ne) {
        const int g = cgt[e], q = ceq[e];
        cgt[e] = static_cast<int>(run & 0xffffffffull);
        ceq[e] = static_cast<int>(run >> 32);
        run += static_cast<unsigned long long>(g) | (static_cast<unsigned long long>(q) << 32);
      }
    }
    if (tid < kRouteCluster) {  // this chunk's counts into every CTA of the cluster
      const uint32_t mine = static_cast<uint32_t>(__cvta_generic_to_shared(&cnt_all[rank][0]));
      const int g = static_cast<int>(total & 0xffffffffull), q = static_cast<int>(total >> 32);
      asm volatile("{\n\t.reg .b32 ra;\n\tmapa.shared::cluster.u32 ra, %0, %1;\n\tst.shared::cluster.v2.u32 [ra], {%2, %3};\n\t}" ::"r"(mine), "r"(tid), "r"(g), "r"(q)
                   : "memory");
    }
  }
  cl.sync();  // every chunk's counts have arrived (and this chunk's offsets are in place)
  if (tid == 0) {
    int sel_before = 0, eq_before = 0;
    for (int r = 0; r < rank; ++r) {
      const int r_gt = cnt_all[r][0], r_eq = cnt_all[r][1];
      sel_before += r_gt + min(r_eq, max(0, need_eq - eq_before));
      eq_before += r_eq;
    }
    sh_off[0] = n_route >= N ? c0 : (n_route <= 0 ? 0 : sel_before);
    sh_off[1] = min(cnt_all[rank][1], max(0, need_eq - eq_before));  // equal keys of this chunk that are routed
  }
  __syncthreads();
  const int sel_before = sh_off[0], take_eq = sh_off[1];
  const unsigned lt = (1u << lane) - 1u;
  int32_t* rout = routed + static_cast<size_t>(bh) * n_route;
  int32_t* tout = taylor + static_cast<size_t>(bh) * (N - n_route);
  for (int j = 0; j < trips; ++j) {
    const int i = j * kRouteCT + tid;
    const unsigned x = i < n ? rkeys[i] : 0u;
    bool sel;
    int r;  // routed keys before c0 + i over the head
    if (partial) {
      const bool gt = i < n && x > T, eq = i < n && x == T;
      const unsigned bgt = __ballot_sync(0xffffffffu, gt);
      const unsigned beq = __ballot_sync(0xffffffffu, eq);
      const int gt_b = cgt[j * kRouteNW + w] + __popc(bgt & lt);
      const int eq_b = ceq[j * kRouteNW + w] + __popc(beq & lt);
      sel = gt || (eq && eq_b < take_eq);
      r = sel_before + gt_b + min(eq_b, take_eq);
    } else {
      sel = n_route >= N && i < n;
      r = sel_before + (n_route >= N ? i : 0);
    }
    if (i < n) {
      // counts are exact by construction; the guards only keep a corrupted
      // input (e.g. NaN sharpness) from writing past the buckets
      const int gi = c0 + i;
      if (sel) {
        if (r < n_route) rout[r] = gi;
        else if (status != nullptr) atomicCAS(status, 0, 1);
      } else {
        if (gi - r >= 0 && gi - r < N - n_route) tout[gi - r] = gi;
        else if (status != nullptr) atomicCAS(status, 0, 1);
      }
    }
  }
  cl.sync();  // no CTA exits while a peer may still store into it
}

cudaError_t launch_route(const float* sharp, int32_t* routed, int32_t* taylor, int BH, int N, int n_route,
                         int* status, cudaStream_t st) {
  if (BH <= 0 || N <= 0) return cudaSuccess;
  cudaError_t e;
  const int chunk = (N + kRouteCluster - 1) / kRouteCluster;
  if (chunk <= kRouteChunkCap && static_cast<long long>(BH) * kRouteCluster <= 0x7fffffffLL) {
    const int trips = (chunk + kRouteCT - 1) / kRouteCT;
    const size_t smem = static_cast<size_t>(chunk) * 4 + static_cast<size_t>(2 * trips * kRouteNW) * 4;
    e = cudaFuncSetAttribute(route_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem < 48 * 1024 ? 48 * 1024 : smem));
    if (e != cudaSuccess) return e;
    route_cluster_kernel<<<BH * kRouteCluster, kRouteCT, smem, st>>>(sharp, routed, taylor, N, n_route, status);
    return cudaGetLastError();
  }
  const size_t counts = static_cast<size_t>(route_count_words(N)) * 4;
  const size_t resident = static_cast<size_t>(N) * 4 + counts;
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
