// route.cu -- ISA dynamic query grouping (stage 2, second half).
//
// "Lightning Unified Video Editing via In-Context Sparse Attention",
// abstract: high-error queries go to full attention, the rest to 0-th order
// Taylor attention, with query sharpness as the error proxy.  Reading: per
// (b, h) the n_route queries of largest sharpness (ties: lower index first)
// are routed; both buckets are written in ascending token order.
//
// One 1024-thread CTA per (b, h):
//  1. exact radix select (4 passes of 8 bits, MSB first) of the n_route-th
//     largest sharpness bit pattern T (sharpness is positive, so its bit
//     pattern orders like its value), with per-warp shared histograms;
//  2. one ordered pass: a query is routed if its key is above T, or equal to
//     T and among the first (n_route - #above) equal keys by index; ranks
//     come from warp ballots + popc and a scan of the 32 warp counts.
#include "block_scan.cuh"
#include "isa_internal.h"

namespace isa {

__global__ void __launch_bounds__(1024) route_kernel(const float* __restrict__ sharp, int32_t* __restrict__ routed,
                                                     int32_t* __restrict__ taylor, int N, int n_route,
                                                     int* __restrict__ status) {
  __shared__ int hist[32][256];
  __shared__ int tot[256];
  __shared__ unsigned sh_sel;
  __shared__ int sh_rem;
  __shared__ int scan_ws[33];
  const int bh = blockIdx.x, tid = threadIdx.x, w = tid >> 5;
  const unsigned* u = reinterpret_cast<const unsigned*>(sharp + static_cast<size_t>(bh) * N);
  int32_t* rout = routed + static_cast<size_t>(bh) * n_route;
  int32_t* tout = taylor + static_cast<size_t>(bh) * (N - n_route);

  unsigned T = 0u;
  int need_eq = 0;
  if (n_route > 0 && n_route < N) {
    unsigned prefix = 0u, pmask = 0u;
    int remaining = n_route;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int i = tid; i < 32 * 256; i += 1024) (&hist[0][0])[i] = 0;
      __syncthreads();
      for (int i = tid; i < N; i += 1024) {
        const unsigned x = __ldg(u + i);
        if ((x & pmask) == prefix) atomicAdd(&hist[w][(x >> shift) & 255u], 1);
      }
      __syncthreads();
      if (tid < 256) {
        int s = 0;
        for (int ww = 0; ww < 32; ++ww) s += hist[ww][tid];
        tot[tid] = s;
      }
      __syncthreads();
      if (tid == 0) {
        int cum = 0;
        unsigned sel = 0u;
        for (int bin = 255; bin >= 0; --bin) {
          if (cum + tot[bin] >= remaining) {
            sel = static_cast<unsigned>(bin);
            break;
          }
          cum += tot[bin];
        }
        sh_sel = sel;
        sh_rem = remaining - cum;
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

  int run_routed = 0, run_eq = 0;
  for (int base = 0; base < N; base += 1024) {
    const int i = base + tid;
    const bool in = i < N;
    bool sel;
    if (n_route == 0) {
      sel = false;
    } else if (n_route == N) {
      sel = in;
    } else {
      const unsigned x = in ? __ldg(u + i) : 0u;
      const bool eq = in && x == T;
      int eq_tot;
      const int eq_rank = block_rank_1024(eq, scan_ws, eq_tot) + run_eq;
      run_eq += eq_tot;
      sel = in && (x > T || (eq && eq_rank < need_eq));
    }
    int sel_tot;
    const int r = block_rank_1024(sel, scan_ws, sel_tot) + run_routed;
    if (in) {
      // Counts are exact by construction; the guards only keep a corrupted
      // input (e.g. NaN sharpness) from writing past the buckets.
      if (sel) {
        if (r < n_route) rout[r] = i; else atomicCAS(status, 0, 1);
      } else {
        if (i - r < N - n_route) tout[i - r] = i; else atomicCAS(status, 0, 1);
      }
    }
    run_routed += sel_tot;
  }
}

cudaError_t launch_route(const float* sharp, int32_t* routed, int32_t* taylor, int BH, int N, int n_route,
                         int* status, cudaStream_t st) {
  route_kernel<<<BH, 1024, 0, st>>>(sharp, routed, taylor, N, n_route, status);
  return cudaGetLastError();
}

}  // namespace isa
