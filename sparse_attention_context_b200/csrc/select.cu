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
// saliency_kernel: grid (ceil(nB/16), B*H); a CTA owns 16 query blocks,
//   computes their logits against every key block in fp32 (two passes: row
//   max and sum, then the column contributions; logits recomputed bit-
//   identically), and writes per-chunk partial column sums.
// select_ctx_kernel: one 1024-thread CTA per (b, h); sums the partials in a
//   fixed order, bitonic-sorts (saliency, block) keys in shared memory, and
//   writes the kept block numbers in ascending order.
// build_kept_kernel: one CTA per kept block slot; writes the bf16 hi/lo split
//   of Kbar, bf16 Vbar and log2(cnt) for the tensor-core stages; slots past
//   the kept count are zero with a -inf bias.
#include <cuda_bf16.h>

#include <cmath>

#include "block_scan.cuh"
#include "isa_internal.h"

namespace isa {

__device__ __forceinline__ int block_count(int b, int nSB, int N_src, int N_ctx, int blk) {
  return b < nSB ? min(blk, N_src - b * blk) : min(blk, N_ctx - (b - nSB) * blk);
}

template <int D>
__global__ void __launch_bounds__(256) saliency_kernel(const float* __restrict__ Qbar, const float* __restrict__ Kbar,
                                                       float* __restrict__ partial, int N_src, int N_ctx, int blk,
                                                       int nSB, int nB, float scale) {
  constexpr int RB = kSalRows;
  __shared__ __align__(16) float sQ[RB][D];
  __shared__ float red[RB][8];
  __shared__ float rowM[RB], rowS[RB];
  const int chunk = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nCB = nB - nSB;
  const int r0 = chunk * RB;
  const int nr = min(RB, nB - r0);
  for (int e = tid; e < RB * D; e += 256) {
    const int rr = e / D, col = e % D;
    sQ[rr][col] = rr < nr ? Qbar[(static_cast<size_t>(bh) * nB + r0 + rr) * D + col] : 0.f;
  }
  __syncthreads();
  const float* Kh = Kbar + static_cast<size_t>(bh) * nB * D;

  auto logits = [&](int c, float (&lg)[RB]) {
    float acc[RB];
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) acc[rr] = 0.f;
    const float4* kc = reinterpret_cast<const float4*>(Kh + static_cast<size_t>(c) * D);
#pragma unroll 4
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 kv = __ldg(kc + d4);
#pragma unroll
      for (int rr = 0; rr < RB; ++rr) {
        const float4 qv = *reinterpret_cast<const float4*>(&sQ[rr][4 * d4]);
        acc[rr] = fmaf(qv.x, kv.x, acc[rr]);
        acc[rr] = fmaf(qv.y, kv.y, acc[rr]);
        acc[rr] = fmaf(qv.z, kv.z, acc[rr]);
        acc[rr] = fmaf(qv.w, kv.w, acc[rr]);
      }
    }
    const float lc = logf(static_cast<float>(block_count(c, nSB, N_src, N_ctx, blk)));
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) lg[rr] = fmaf(scale, acc[rr], lc);
  };

  // Pass 1: per-row max and sum of exp over all key blocks.
  float mloc[RB], sloc[RB];
#pragma unroll
  for (int rr = 0; rr < RB; ++rr) {
    mloc[rr] = -INFINITY;
    sloc[rr] = 0.f;
  }
  for (int c = tid; c < nB; c += 256) {
    float lg[RB];
    logits(c, lg);
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) {
      const float mn = fmaxf(mloc[rr], lg[rr]);
      sloc[rr] = sloc[rr] * expf(mloc[rr] - mn) + expf(lg[rr] - mn);
      mloc[rr] = mn;
    }
  }
#pragma unroll
  for (int rr = 0; rr < RB; ++rr) {
    float mm = mloc[rr];
#pragma unroll
    for (int o = 16; o; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, o));
    float ss = (mloc[rr] == -INFINITY) ? 0.f : sloc[rr] * expf(mloc[rr] - mm);
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) {
      red[rr][w] = mm;
      rowS[rr] = 0.f;
    }
    mloc[rr] = mm;
    sloc[rr] = ss;
  }
  __syncthreads();
  if (tid < RB) {
    float mm = -INFINITY;
    for (int i = 0; i < 8; ++i) mm = fmaxf(mm, red[tid][i]);
    rowM[tid] = mm;
  }
  __syncthreads();
#pragma unroll
  for (int rr = 0; rr < RB; ++rr) {
    if (lane == 0) red[rr][w] = sloc[rr] * expf(mloc[rr] - rowM[rr]);
  }
  __syncthreads();
  if (tid < RB) {
    float ss = 0.f;
    for (int i = 0; i < 8; ++i) ss += red[tid][i];
    rowS[tid] = ss;
  }
  __syncthreads();

  // Pass 2: column contributions sum_r cnt_r * P_rc for context blocks.
  float wr[RB];
#pragma unroll
  for (int rr = 0; rr < RB; ++rr)
    wr[rr] = rr < nr ? static_cast<float>(block_count(r0 + rr, nSB, N_src, N_ctx, blk)) / rowS[rr] : 0.f;
  float* out = partial + (static_cast<size_t>(bh) * gridDim.x + chunk) * nCB;
  for (int c = nSB + tid; c < nB; c += 256) {
    float lg[RB];
    logits(c, lg);
    float col = 0.f;
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) col = fmaf(wr[rr], expf(lg[rr] - rowM[rr]), col);
    out[c - nSB] = col;
  }
}

__global__ void __launch_bounds__(1024) select_ctx_kernel(const float* __restrict__ partial, int n_chunks,
                                                          float* __restrict__ sal_ws, float* __restrict__ sal_user,
                                                          int32_t* __restrict__ kept, int nCB, int n_keep,
                                                          float inv_N) {
  __shared__ unsigned long long keys[kTopkCap];
  __shared__ unsigned char flag[kTopkCap];
  __shared__ int scan_ws[33];
  const int bh = blockIdx.x, tid = threadIdx.x;
  int P = 2;
  while (P < nCB) P <<= 1;
  for (int c = tid; c < P; c += 1024) {
    unsigned long long key = 0ull;
    if (c < nCB) {
      float s = 0.f;
      const float* pp = partial + static_cast<size_t>(bh) * n_chunks * nCB + c;
      for (int ch = 0; ch < n_chunks; ++ch) s += pp[static_cast<size_t>(ch) * nCB];
      s *= inv_N;
      sal_ws[static_cast<size_t>(bh) * nCB + c] = s;
      if (sal_user) sal_user[static_cast<size_t>(bh) * nCB + c] = s;
      // non-negative float: its bit pattern orders like the value; lower
      // block number ranks first on equal saliency.
      key = (static_cast<unsigned long long>(__float_as_uint(s)) << 32) |
            static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<unsigned>(c));
    }
    keys[c] = key;
    flag[c] = 0;
  }
  __syncthreads();
  // Bitonic sort, descending.
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P; i += 1024) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = keys[i], b = keys[ixj];
          const bool desc = (i & k) == 0;
          if (desc ? (a < b) : (a > b)) {
            keys[i] = b;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < n_keep; i += 1024) {
    const unsigned c = 0xFFFFFFFFu - static_cast<unsigned>(keys[i] & 0xFFFFFFFFull);
    if (c < static_cast<unsigned>(nCB)) flag[c] = 1;
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
                                  const int32_t* __restrict__ kept, uint16_t* __restrict__ Khi,
                                  uint16_t* __restrict__ Klo, uint16_t* __restrict__ Vb, float* __restrict__ bias2,
                                  int N_src, int N_ctx, int blk, int nSB, int nB, int n_keep, int nKpad,
                                  int* __restrict__ status) {
  const int t = blockIdx.x, bh = blockIdx.y, col = threadIdx.x;
  int b = -1;
  if (t < nSB) {
    b = t;
  } else if (t < nSB + n_keep) {
    const int c = kept[static_cast<size_t>(bh) * n_keep + (t - nSB)];
    if (c >= 0 && c < nB - nSB)
      b = nSB + c;
    else if (col == 0)
      atomicCAS(status, 0, 1 /* ISA_ERR_INVALID_ARG: kept block out of range, slot left empty */);
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

cudaError_t launch_saliency(const float* Qbar, const float* Kbar, float* partial, int BH, int N_src, int N_ctx,
                            int D, int blk, float scale, cudaStream_t st) {
  const int nSB = (N_src + blk - 1) / blk, nCB = (N_ctx + blk - 1) / blk, nB = nSB + nCB;
  if (nCB == 0) return cudaSuccess;
  const dim3 grid((nB + kSalRows - 1) / kSalRows, BH);
  if (D == 128)
    saliency_kernel<128><<<grid, 256, 0, st>>>(Qbar, Kbar, partial, N_src, N_ctx, blk, nSB, nB, scale);
  else
    saliency_kernel<64><<<grid, 256, 0, st>>>(Qbar, Kbar, partial, N_src, N_ctx, blk, nSB, nB, scale);
  return cudaGetLastError();
}

cudaError_t launch_select_ctx(const float* partial, float* sal_ws, float* sal_user, int32_t* kept, int BH,
                              int N_src, int N_ctx, int blk, int n_keep, cudaStream_t st) {
  const int nSB = (N_src + blk - 1) / blk, nCB = (N_ctx + blk - 1) / blk, nB = nSB + nCB;
  if (nCB == 0) return cudaSuccess;
  const int n_chunks = (nB + kSalRows - 1) / kSalRows;
  select_ctx_kernel<<<BH, 1024, 0, st>>>(partial, n_chunks, sal_ws, sal_user, kept, nCB, n_keep,
                                          1.0f / static_cast<float>(N_src + N_ctx));
  return cudaGetLastError();
}

cudaError_t launch_build_kept(const float* Kbar, const float* Vbar, const int32_t* kept, uint16_t* Khi,
                              uint16_t* Klo, uint16_t* Vb, float* bias2, int BH, int N_src, int N_ctx, int D,
                              int blk, int n_keep, int nKpad, int* status, cudaStream_t st) {
  const int nSB = (N_src + blk - 1) / blk, nCB = (N_ctx + blk - 1) / blk, nB = nSB + nCB;
  const dim3 grid(nKpad, BH);
  if (D == 128)
    build_kept_kernel<128><<<grid, 128, 0, st>>>(Kbar, Vbar, kept, Khi, Klo, Vb, bias2, N_src, N_ctx, blk, nSB, nB,
                                                 n_keep, nKpad, status);
  else
    build_kept_kernel<64><<<grid, 64, 0, st>>>(Kbar, Vbar, kept, Khi, Klo, Vb, bias2, N_src, N_ctx, blk, nSB, nB,
                                               n_keep, nKpad, status);
  return cudaGetLastError();
}

}  // namespace isa
