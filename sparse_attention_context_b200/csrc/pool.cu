// pool.cu -- block means of q, k, v (ISA stage 1 input; also the keys and
// values of the 0-th order Taylor path).
//
// Blocks are taken per segment: source blocks b < nSB cover rows
// [b*blk, min((b+1)*blk, N_src)), context blocks cover the context rows the
// same way; the last block of each segment may be partial.  One CTA reduces
// one block of one (b, h): 16-byte vector loads (8 bf16), fp32 accumulation
// in a fixed order: each thread sums one 8-column chunk over a strided set
// of rows, then the row groups' partial sums are added through shared
// memory.  HBM-bound.  q and k are pooled over every block (the block
// saliency takes all of them); v only over the source blocks, since Vbar is
// read only for kept blocks (source blocks and the kept context blocks):
// pool_kept_v_kernel pools v over the kept context blocks once the
// selection has chosen them, in the same summation order (the same bits as
// pooling every block would give).  The other context rows of v are never
// read.
#include <cuda_bf16.h>

#include "isa_internal.h"
#include "tc_ptx.cuh"

namespace isa {

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4& w) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[2 * i + 0] += __uint_as_float(u[i] << 16);
    a[2 * i + 1] += __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                                   const uint16_t* __restrict__ v, float* __restrict__ Qbar,
                                                   float* __restrict__ Kbar, float* __restrict__ Vbar,
                                                   uint16_t* __restrict__ QKsplit, int N_src, int N_ctx, int blk,
                                                   int nSB, int nB, int nBp) {
  constexpr int CPR = D / 8;          // 16-byte chunks per row
  constexpr int RG = 256 / CPR;       // row groups (rows in flight per pass)
  __shared__ float red[3][RG][D + 4];
  const int b = blockIdx.x, bh = blockIdx.y;
  // bf16 hi + lo of Qbar and Kbar for the tensor-core saliency: four
  // [BH, nBp, D] arrays (Qhi, Qlo, Khi, Klo); rows nB..nBp-1 are not written
  // (the saliency kernel masks them)
  const size_t split_plane = static_cast<size_t>(gridDim.y) * nBp * D;
  uint16_t* split_row = QKsplit + (static_cast<size_t>(bh) * nBp + b) * D;
  const int N = N_src + N_ctx;
  const int start = b < nSB ? b * blk : N_src + (b - nSB) * blk;
  const int cnt = b < nSB ? min(blk, N_src - b * blk) : min(blk, N_ctx - (b - nSB) * blk);
  const int ch = threadIdx.x % CPR, rg = threadIdx.x / CPR;
  const size_t base = (static_cast<size_t>(bh) * N + start) * D + ch * 8;
  float aq[8] = {0}, ak[8] = {0}, av[8] = {0};
  if (b < nSB) {
#pragma unroll 4
    for (int r = rg; r < cnt; r += RG) {
      const size_t off = base + static_cast<size_t>(r) * D;
      const uint4 wq = __ldg(reinterpret_cast<const uint4*>(q + off));
      const uint4 wk = __ldg(reinterpret_cast<const uint4*>(k + off));
      const uint4 wv = __ldg(reinterpret_cast<const uint4*>(v + off));
      acc_bf16x8(aq, wq);
      acc_bf16x8(ak, wk);
      acc_bf16x8(av, wv);
    }
  } else {
#pragma unroll 4
    for (int r = rg; r < cnt; r += RG) {
      const size_t off = base + static_cast<size_t>(r) * D;
      const uint4 wq = __ldg(reinterpret_cast<const uint4*>(q + off));
      const uint4 wk = __ldg(reinterpret_cast<const uint4*>(k + off));
      acc_bf16x8(aq, wq);
      acc_bf16x8(ak, wk);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    red[0][rg][ch * 8 + i] = aq[i];
    red[1][rg][ch * 8 + i] = ak[i];
    red[2][rg][ch * 8 + i] = av[i];
  }
  __syncthreads();
  const float fcnt = static_cast<float>(cnt);
  // two adjacent columns per thread: 8-byte fp32 and 4-byte bf16x2 stores
  for (int e = threadIdx.x; e < 3 * D / 2; e += 256) {
    const int t = (2 * e) / D, col = (2 * e) % D;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) {
      s0 += red[t][g][col];
      s1 += red[t][g][col + 1];
    }
    const float m0 = s0 / fcnt, m1 = s1 / fcnt;
    float* dst = t == 0 ? Qbar : (t == 1 ? Kbar : (b < nSB ? Vbar : nullptr));  // Qbar may be null
    if (dst != nullptr) *reinterpret_cast<float2*>(dst + (static_cast<size_t>(bh) * nB + b) * D + col) = make_float2(m0, m1);
    if (t < 2) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(m0), h1 = __float2bfloat16_rn(m1);
      const __nv_bfloat16 l0 = __float2bfloat16_rn(m0 - __bfloat162float(h0));
      const __nv_bfloat16 l1 = __float2bfloat16_rn(m1 - __bfloat162float(h1));
      *reinterpret_cast<uint32_t*>(split_row + (2 * t) * split_plane + col) =
          static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
      *reinterpret_cast<uint32_t*>(split_row + (2 * t + 1) * split_plane + col) =
          static_cast<uint32_t>(__bfloat16_as_ushort(l0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
    }
  }
}

// Vbar of the kept context blocks: one CTA per (kept slot, b*H + h), the
// reduction of pool_kernel on v alone; slots with an index outside the
// context are skipped (the operand build reports them).  The kept set is
// recorded in ksel, against which the operand build checks the set it is
// given.
template <int D>
__global__ void __launch_bounds__(256) pool_kept_v_kernel(const uint16_t* __restrict__ v,
                                                          const int32_t* __restrict__ kept, int32_t* __restrict__ ksel,
                                                          float* __restrict__ Vbar, int N_src, int N_ctx, int blk,
                                                          int nSB, int nB, int n_keep) {
  constexpr int CPR = D / 8;
  constexpr int RG = 256 / CPR;
  __shared__ float red[RG][D + 4];
  const int slot = blockIdx.x, bh = blockIdx.y;
  const int c = __ldg(kept + static_cast<size_t>(bh) * n_keep + slot);
  if (threadIdx.x == 0) ksel[static_cast<size_t>(bh) * n_keep + slot] = c;
  if (c < 0 || c >= nB - nSB) return;
  const int N = N_src + N_ctx;
  const int start = N_src + c * blk;
  const int cnt = min(blk, N_ctx - c * blk);
  const int ch = threadIdx.x % CPR, rg = threadIdx.x / CPR;
  const size_t base = (static_cast<size_t>(bh) * N + start) * D + ch * 8;
  float av[8] = {0};
#pragma unroll 4
  for (int r = rg; r < cnt; r += RG)
    acc_bf16x8(av, __ldg(reinterpret_cast<const uint4*>(v + base + static_cast<size_t>(r) * D)));
#pragma unroll
  for (int i = 0; i < 8; ++i) red[rg][ch * 8 + i] = av[i];
  __syncthreads();
  const float fcnt = static_cast<float>(cnt);
  for (int e = threadIdx.x; e < D / 2; e += 256) {
    const int col = 2 * e;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) {
      s0 += red[g][col];
      s1 += red[g][col + 1];
    }
    *reinterpret_cast<float2*>(Vbar + (static_cast<size_t>(bh) * nB + nSB + c) * D + col) =
        make_float2(s0 / fcnt, s1 / fcnt);
  }
}

cudaError_t launch_pool_kept_v(const uint16_t* v, const int32_t* kept, int32_t* ksel, float* Vbar, int BH,
                               int N_src, int N_ctx, int D, int blk, int n_keep, cudaStream_t st) {
  const int nSB = (N_src + blk - 1) / blk, nCB = (N_ctx + blk - 1) / blk;
  if (n_keep <= 0 || nCB <= 0 || BH <= 0) return cudaSuccess;
  const dim3 grid(n_keep, BH);
  if (D == 128)
    pool_kept_v_kernel<128><<<grid, 256, 0, st>>>(v, kept, ksel, Vbar, N_src, N_ctx, blk, nSB, nSB + nCB, n_keep);
  else
    pool_kept_v_kernel<64><<<grid, 256, 0, st>>>(v, kept, ksel, Vbar, N_src, N_ctx, blk, nSB, nSB + nCB, n_keep);
  return cudaGetLastError();
}

cudaError_t launch_pool(const uint16_t* q, const uint16_t* k, const uint16_t* v, float* Qbar, float* Kbar,
                        float* Vbar, uint16_t* QKsplit, int BH, int N_src, int N_ctx, int D, int blk,
                        cudaStream_t st) {
  const int nSB = (N_src + blk - 1) / blk, nCB = (N_ctx + blk - 1) / blk;
  const int nB = nSB + nCB;
  const int nBp = (nB + 127) / 128 * 128;
  const dim3 grid(nB, BH);
  if (D == 128)
    pool_kernel<128><<<grid, 256, 0, st>>>(q, k, v, Qbar, Kbar, Vbar, QKsplit, N_src, N_ctx, blk, nSB, nB, nBp);
  else
    pool_kernel<64><<<grid, 256, 0, st>>>(q, k, v, Qbar, Kbar, Vbar, QKsplit, N_src, N_ctx, blk, nSB, nB, nBp);
  return cudaGetLastError();
}

}  // namespace isa
