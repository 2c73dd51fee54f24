// select.cu -- ISA stage 1, context pre-selection, and the gather of the
// kept block statistics used by stages 2 and 4.
//
// Reading of the pre-selection step of "Lightning Unified Video Editing via
// In-Context Sparse Attention" (abstract, first insight): the saliency of a
// key block c is the attention mass it receives at block level,
//   sal_c = sum_r cnt_r * softmax_c( s * Qbar_r . Kbar_c + ln cnt_c ) / N,
// over all key blocks c (source and context) and all query blocks r; the
// n_keep most salient context blocks are kept (higher saliency first, lower
// block number on ties), every source block is always kept.
//
// The saliency itself (per-row-tile partial column sums) comes from the
// tensor-core tile kernel of saliency_tc.cu.
// select_ctx_kernel: one 1024-thread CTA per (b, h); sums the row tiles'
//   partial column sums in a fixed order, divides by N, ranks every block
//   by counting the (saliency, block) keys above its own (no sort: nCB
//   comparisons per block, all threads reading the same key at once), and
//   writes the kept block numbers in ascending order.
// build_kept_kernel: one CTA per kept block slot; writes the bf16 hi/lo split
//   of Kbar, bf16 Vbar and log2(cnt) for the tensor-core stages; slots past
//   the kept count are zero with a -inf bias.  Vbar holds the context blocks
//   that the pre-selection kept (ksel, its record of them), so a kept set
//   that differs from it is reported (ISA_ERR_INVALID_ARG) rather than
//   computed on block means that were never pooled.
#include <cuda_bf16.h>

#include <cmath>

#include "block_scan.cuh"
#include "isa_internal.h"

namespace isa {

__device__ __forceinline__ int block_count(int b, int nSB, int N_src, int N_ctx, int blk) {
  return b < nSB ? min(blk, N_src - b * blk) : min(blk, N_ctx - (b - nSB) * blk);
}

__global__ void __launch_bounds__(1024) select_ctx_kernel(const float* __restrict__ partial, int n_chunks,
                                                          float* __restrict__ sal_ws, float* __restrict__ sal_user,
                                                          int32_t* __restrict__ kept, int nCB, int n_keep,
                                                          float inv_N) {
  __shared__ unsigned long long keys[kTopkCap];
  __shared__ unsigned char flag[kTopkCap];
  __shared__ int scan_ws[33];
  const int bh = blockIdx.x, tid = threadIdx.x;
  for (int c = tid; c < nCB; c += 1024) {
    float s = 0.f;
    const float* pp = partial + static_cast<size_t>(bh) * n_chunks * nCB + c;
    for (int ch = 0; ch < n_chunks; ++ch) s += pp[static_cast<size_t>(ch) * nCB];
    s *= inv_N;
    sal_ws[static_cast<size_t>(bh) * nCB + c] = s;
    if (sal_user) sal_user[static_cast<size_t>(bh) * nCB + c] = s;
    // non-negative float: its bit pattern orders like the value; the lower
    // block number ranks first on equal saliency (all keys distinct)
    keys[c] = (static_cast<unsigned long long>(__float_as_uint(s)) << 32) |
              static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<unsigned>(c));
  }
  __syncthreads();
  // a block is kept when fewer than n_keep blocks rank above it
  for (int c = tid; c < nCB; c += 1024) {
    const unsigned long long kc = keys[c];
    int above = 0;
    for (int o = 0; o < nCB; ++o) above += keys[o] > kc ? 1 : 0;  // every thread reads keys[o] together
    flag[c] = above < n_keep ? 1 : 0;
  }
  __syncthreads();
  int run = 0;
  for (int base = 0; base < nCB; base += 1024) {
    const int c = base + tid;
    const bool f = c < nCB && flag[c];
    int tot;
    const int pos = block_rank_1024(f, scan_ws, tot) + run;
    if (f) kept[static_cast<size_t>(bh) * n_keep + pos] = c;
    run += tot;
  }
}

template <int D>
__global__ void build_kept_kernel(const float* __restrict__ Kbar, const float* __restrict__ Vbar,
                                  const int32_t* __restrict__ kept, const int32_t* __restrict__ ksel,
                                  uint16_t* __restrict__ Khi,
                                  uint16_t* __restrict__ Klo, uint16_t* __restrict__ Vb, float* __restrict__ bias2,
                                  int N_src, int N_ctx, int blk, int nSB, int nB, int n_keep, int nKpad,
                                  int* __restrict__ status) {
  const int t = blockIdx.x, bh = blockIdx.y, col = threadIdx.x;
  int b = -1;
  if (t < nSB) {
    b = t;
  } else if (t < nSB + n_keep) {
    const size_t ki = static_cast<size_t>(bh) * n_keep + (t - nSB);
    const int c = kept[ki];
    if (c >= 0 && c < nB - nSB)
      b = nSB + c;
    else if (col == 0)
      atomicCAS(status, 0, 1 /* ISA_ERR_INVALID_ARG: kept block out of range, slot left empty */);
    if (col == 0 && c != __ldg(ksel + ki))
      atomicCAS(status, 0, 1 /* ISA_ERR_INVALID_ARG: not the pre-selection's kept set */);
  }
  const size_t dst = (static_cast<size_t>(bh) * nKpad + t) * D + col;
  if (b >= 0) {
    const float kb = Kbar[(static_cast<size_t>(bh) * nB + b) * D + col];
    const __nv_bfloat16 hi = __float2bfloat16_rn(kb);
    const __nv_bfloat16 lo = __float2bfloat16_rn(kb - __bfloat162float(hi));
    const __nv_bfloat16 vb = __float2bfloat16_rn(Vbar[(static_cast<size_t>(bh) * nB + b) * D + col]);
    Khi[dst] = __bfloat16_as_ushort(hi);
    Klo[dst] = __bfloat16_as_ushort(lo);
    Vb[dst] = __bfloat16_as_ushort(vb);
    if (col == 0)
      bias2[static_cast<size_t>(bh) * nKpad + t] = log2f(static_cast<float>(block_count(b, nSB, N_src, N_ctx, blk)));
  } else {
    Khi[dst] = 0;
    Klo[dst] = 0;
    Vb[dst] = 0;
    if (col == 0) bias2[static_cast<size_t>(bh) * nKpad + t] = -INFINITY;
  }
}

cudaError_t launch_select_ctx(const float* partial, int n_chunks, float* sal_ws, float* sal_user, int32_t* kept,
                              int BH, int N_src, int N_ctx, int blk, int n_keep, cudaStream_t st) {
  const int nCB = (N_ctx + blk - 1) / blk;
  if (nCB == 0) return cudaSuccess;
  select_ctx_kernel<<<BH, 1024, 0, st>>>(partial, n_chunks, sal_ws, sal_user, kept, nCB, n_keep,
                                          1.0f / static_cast<float>(N_src + N_ctx));
  return cudaGetLastError();
}

cudaError_t launch_build_kept(const float* Kbar, const float* Vbar, const int32_t* kept, const int32_t* ksel,
                              uint16_t* Khi, uint16_t* Klo, uint16_t* Vb, float* bias2, int BH, int N_src, int N_ctx,
                              int D, int blk, int n_keep, int nKpad, int* status, cudaStream_t st) {
  const int nSB = (N_src + blk - 1) / blk, nCB = (N_ctx + blk - 1) / blk, nB = nSB + nCB;
  const dim3 grid(nKpad, BH);
  if (D == 128)
    build_kept_kernel<128><<<grid, 128, 0, st>>>(Kbar, Vbar, kept, ksel, Khi, Klo, Vb, bias2, N_src, N_ctx, blk, nSB,
                                                 nB, n_keep, nKpad, status);
  else
    build_kept_kernel<64><<<grid, 64, 0, st>>>(Kbar, Vbar, kept, ksel, Khi, Klo, Vb, bias2, N_src, N_ctx, blk, nSB,
                                               nB, n_keep, nKpad, status);
  return cudaGetLastError();
}

}  // namespace isa
