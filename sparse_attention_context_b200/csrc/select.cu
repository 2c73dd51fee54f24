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
// saliency_kernel: grid (ceil(nB/32), B*H); a CTA owns 32 query blocks and
//   walks the key blocks in tiles of 64 staged in shared memory (each K-bar
//   row is read from L2 once per CTA), computing the logits in fp32 (pass 1:
//   row max and sum; pass 2: the column contributions of the context
//   blocks), and writes per-chunk partial column sums.  Pass 1 keeps its
//   logits in shared memory when 32 x nB floats fit, so pass 2 reads them
//   back instead of recomputing them; larger shapes recompute them
//   bit-identically.
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

// Shared-memory tile sizes of saliency_kernel.
constexpr int kSalColTile = 64;  // key blocks staged per tile
template <int D>
constexpr int sal_smem_bytes() {
  return (kSalRows * D + kSalColTile * (D + 4) + 16 * kSalColTile) * 4;
}
// Shared memory of the logit cache: kSalRows rows of nB logits, padded to
// whole column tiles.
inline size_t sal_cache_bytes(int nB) {
  return static_cast<size_t>(kSalRows) * ((nB + kSalColTile - 1) / kSalColTile * kSalColTile) * 4;
}

template <int D, bool CACHE>
__global__ void __launch_bounds__(256) saliency_kernel(const float* __restrict__ Qbar, const float* __restrict__ Kbar,
                                                       float* __restrict__ partial, int N_src, int N_ctx, int blk,
                                                       int nSB, int nB, float scale) {
  constexpr int RB = kSalRows;     // query blocks of this CTA
  constexpr int CT = kSalColTile;  // key blocks per staged tile
  constexpr int KP = D + 4;        // padded row of the staged tile (conflict-free float4 columns)
  extern __shared__ __align__(16) float sal_sm[];
  float* sQ = sal_sm;               // [RB][D]
  float* sK = sQ + RB * D;          // [CT][KP]
  float* sRed = sK + CT * KP;       // [16][CT] column partial sums of the 16 row pairs
  float* sL = sRed + 16 * CT;       // CACHE: [RB][nBp] logits of pass 1
  const int nBp = (nB + CT - 1) / CT * CT;
  const int chunk = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;  // rows 2ty, 2ty+1; tile columns tx + 16m
  const int nCB = nB - nSB;
  const int r0 = chunk * RB;
  const int nr = min(RB, nB - r0);
  const float* Kh = Kbar + static_cast<size_t>(bh) * nB * D;
  for (int e = tid; e < RB * D / 4; e += 256) {
    const int rr = e / (D / 4), q4 = e % (D / 4);
    const float4 v = rr < nr ? __ldg(reinterpret_cast<const float4*>(Qbar + (static_cast<size_t>(bh) * nB + r0 + rr) * D) + q4)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(sQ + rr * D + 4 * q4) = v;
  }
  // K rows [c0, c0 + CT) into sK (zero past nB); the caller syncs around it
  auto stage = [&](int c0) {
    for (int e = tid; e < CT * D / 4; e += 256) {
      const int rr = e / (D / 4), q4 = e % (D / 4);
      const int c = c0 + rr;
      const float4 v = c < nB ? __ldg(reinterpret_cast<const float4*>(Kh + static_cast<size_t>(c) * D) + q4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(sK + rr * KP + 4 * q4) = v;
    }
  };
  // logits of rows 2ty, 2ty+1 against tile columns tx + 16m (-inf past nB);
  // each dot product accumulates over d in order, as a plain loop would
  auto tile_logits = [&](int c0, float (&lg)[2][4]) {
    float acc[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[i][m] = 0.f;
#pragma unroll 8
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 qa = *reinterpret_cast<const float4*>(sQ + (2 * ty) * D + 4 * d4);
      const float4 qb = *reinterpret_cast<const float4*>(sQ + (2 * ty + 1) * D + 4 * d4);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 kv = *reinterpret_cast<const float4*>(sK + (tx + 16 * m) * KP + 4 * d4);
        acc[0][m] = fmaf(qa.x, kv.x, acc[0][m]);
        acc[0][m] = fmaf(qa.y, kv.y, acc[0][m]);
        acc[0][m] = fmaf(qa.z, kv.z, acc[0][m]);
        acc[0][m] = fmaf(qa.w, kv.w, acc[0][m]);
        acc[1][m] = fmaf(qb.x, kv.x, acc[1][m]);
        acc[1][m] = fmaf(qb.y, kv.y, acc[1][m]);
        acc[1][m] = fmaf(qb.z, kv.z, acc[1][m]);
        acc[1][m] = fmaf(qb.w, kv.w, acc[1][m]);
      }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int c = c0 + tx + 16 * m;
      const float lc = c < nB ? logf(static_cast<float>(block_count(c, nSB, N_src, N_ctx, blk))) : 0.f;
#pragma unroll
      for (int i = 0; i < 2; ++i) lg[i][m] = c < nB ? fmaf(scale, acc[i][m], lc) : -INFINITY;
    }
  };

  // Pass 1: max and sum of exp of each row over all key blocks (online per
  // thread over its columns, then merged across the 16 threads of a row pair)
  float rm[2] = {-INFINITY, -INFINITY}, rs[2] = {0.f, 0.f};
  for (int c0 = 0; c0 < nB; c0 += CT) {
    __syncthreads();
    stage(c0);
    __syncthreads();
    float lg[2][4];
    tile_logits(c0, lg);
    if constexpr (CACHE) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int m = 0; m < 4; ++m) sL[(2 * ty + i) * nBp + c0 + tx + 16 * m] = lg[i][m];
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float mn = fmaxf(rm[i], lg[i][m]);
        if (mn != -INFINITY) {
          rs[i] = rs[i] * expf(rm[i] - mn) + expf(lg[i][m] - mn);
          rm[i] = mn;
        }
      }
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float mm = rm[i];
#pragma unroll
    for (int o = 8; o; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, o));
    float ss = rm[i] == -INFINITY ? 0.f : rs[i] * expf(rm[i] - mm);
#pragma unroll
    for (int o = 8; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    rm[i] = mm;
    rs[i] = ss;
  }
  // weight of each row: cnt_r / S_r (zero for rows past the last block)
  float wr[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = 2 * ty + i;
    wr[i] = r < nr ? static_cast<float>(block_count(r0 + r, nSB, N_src, N_ctx, blk)) / rs[i] : 0.f;
  }

  // Pass 2: column contributions sum_r cnt_r * P_rc for the context blocks
  float* out = partial + (static_cast<size_t>(bh) * gridDim.x + chunk) * nCB;
  for (int c0 = nSB; c0 < nB; c0 += CT) {
    float lg[2][4];
    if constexpr (CACHE) {
      // the logits of pass 1: the same rows, columns possibly written by
      // another thread of the row pair (pass 2 tiles start at nSB); the
      // barrier makes them visible and also guards sRed of the previous tile
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int c = c0 + tx + 16 * m;
          lg[i][m] = c < nB ? sL[(2 * ty + i) * nBp + c] : -INFINITY;
        }
    } else {
      __syncthreads();
      stage(c0);
      __syncthreads();
      tile_logits(c0, lg);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float col = 0.f;
#pragma unroll
      for (int i = 0; i < 2; ++i) col = fmaf(wr[i], expf(lg[i][m] - rm[i]), col);
      sRed[ty * CT + tx + 16 * m] = col;
    }
    __syncthreads();
    if (tid < CT && c0 + tid < nB) {
      float col = 0.f;
#pragma unroll
      for (int y = 0; y < 16; ++y) col += sRed[y * CT + tid];
      out[c0 + tid - nSB] = col;
    }
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
  cudaError_t e;
  auto run = [&](auto kern, size_t smem) -> cudaError_t {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    kern<<<grid, 256, smem, st>>>(Qbar, Kbar, partial, N_src, N_ctx, blk, nSB, nB, scale);
    return cudaGetLastError();
  };
  constexpr size_t kMax = 227 * 1024;
  if (D == 128) {
    const size_t base = sal_smem_bytes<128>(), cached = base + sal_cache_bytes(nB);
    e = cached <= kMax ? run(saliency_kernel<128, true>, cached) : run(saliency_kernel<128, false>, base);
  } else {
    const size_t base = sal_smem_bytes<64>(), cached = base + sal_cache_bytes(nB);
    e = cached <= kMax ? run(saliency_kernel<64, true>, cached) : run(saliency_kernel<64, false>, base);
  }
  return e;
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
