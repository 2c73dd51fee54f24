// route_blocks.cu -- ISA dynamic query grouping by whole query blocks.
//
// "Lightning Unified Video Editing via In-Context Sparse Attention",
// abstract: queries whose Taylor approximation error is high (sharp
// queries) are grouped for full attention.  The abstract does not fix the
// unit that is grouped; this variant groups the per-segment token blocks
// that the keys already use: a query block scores the mean sharpness of its
// cnt_b queries, and the n_rb = ceil(rho*nB - min(1e-6*nB, 0.5)) best blocks (ties:
// lower block index first) are routed whole.  A routed group is then a run
// of consecutive rows, so full attention needs no scattered query set.
//
// One 1024-thread CTA per (b, h):
//  1. block means of the head's sharpness: one warp per block, lane-strided
//     sums and a fixed shuffle tree (deterministic), scores kept in shared
//     memory;
//  2. exact top-n_rb by rank counting (a block is routed when fewer than
//     n_rb blocks rank ahead of it: higher score, or equal score and lower
//     index); routed blocks compacted in ascending order with a CTA-wide
//     ballot rank;
//  3. expansion into the row list of the full-attention pass: n_rb * blk
//     entries per head, entry r*blk + t = start of routed block r + t, or
//     -1 where t >= cnt of that block (a partial block's missing rows).
#include "block_scan.cuh"
#include "isa_internal.h"

namespace isa {

__device__ __forceinline__ void block_span(int b, int N_src, int N_ctx, int blk, int nSB, int& start, int& cnt) {
  if (b < nSB) {
    start = b * blk;
    cnt = min(blk, N_src - start);
  } else {
    const int c = b - nSB;
    start = N_src + c * blk;
    cnt = min(blk, N_ctx - c * blk);
  }
}

__global__ void __launch_bounds__(1024) route_blocks_kernel(const float* __restrict__ sharp,
                                                            int32_t* __restrict__ routed_blk,
                                                            int32_t* __restrict__ routed_rows,
                                                            float* __restrict__ score_out, int N, int N_src,
                                                            int N_ctx, int blk, int nSB, int nB, int n_rb,
                                                            int* __restrict__ status) {
  extern __shared__ float score[];                                // [nB]
  int* sel_blk = reinterpret_cast<int*>(score + nB);              // [n_rb]
  __shared__ int scan_ws[33];
  const int bh = blockIdx.x, tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const float* s = sharp + static_cast<size_t>(bh) * N;

  for (int b = w; b < nB; b += 32) {
    int start, cnt;
    block_span(b, N_src, N_ctx, blk, nSB, start, cnt);
    float acc = 0.f;
    for (int j = lane; j < cnt; j += 32) acc += __ldg(s + start + j);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) score[b] = acc / static_cast<float>(cnt);
  }
  for (int r = tid; r < n_rb; r += 1024) sel_blk[r] = -1;
  __syncthreads();
  if (score_out != nullptr)
    for (int b = tid; b < nB; b += 1024) score_out[static_cast<size_t>(bh) * nB + b] = score[b];

  int base = 0;
  for (int c0 = 0; c0 < nB; c0 += 1024) {
    const int b = c0 + tid;
    bool sel = false;
    if (b < nB && n_rb > 0) {
      const float x = score[b];
      int ahead = 0;
      for (int c = 0; c < nB && ahead < n_rb; ++c) {
        const float y = score[c];
        ahead += (y > x) || (y == x && c < b);
      }
      sel = ahead < n_rb;
    }
    int total;
    const int r = base + block_rank_1024(sel, scan_ws, total);
    if (sel) {
      // exact by construction; the guard keeps a corrupted input (NaN
      // sharpness) from writing past the list
      if (r < n_rb) sel_blk[r] = b;
      else if (status != nullptr) atomicCAS(status, 0, 1);
    }
    base += total;
  }
  __syncthreads();
  if (tid == 0 && base < n_rb && status != nullptr) atomicCAS(status, 0, 1);  // unfilled slots stay -1

  int32_t* rb = routed_blk + static_cast<size_t>(bh) * n_rb;
  for (int r = tid; r < n_rb; r += 1024) rb[r] = sel_blk[r];
  const int n_rows = n_rb * blk;
  int32_t* rows = routed_rows + static_cast<size_t>(bh) * n_rows;
  for (int e = tid; e < n_rows; e += 1024) {
    const int r = e / blk, t = e - r * blk;
    const int b = sel_blk[r];
    int row = -1;
    if (b >= 0) {
      int start, cnt;
      block_span(b, N_src, N_ctx, blk, nSB, start, cnt);
      if (t < cnt) row = start + t;
    }
    rows[e] = row;
  }
}

cudaError_t launch_route_blocks(const float* sharp, int32_t* routed_blk, int32_t* routed_rows, float* score_out,
                                int BH, int N_src, int N_ctx, int blk, int n_rb, int* status, cudaStream_t st) {
  const int nSB = (N_src + blk - 1) / blk, nCB = (N_ctx + blk - 1) / blk, nB = nSB + nCB;
  if (BH <= 0 || nB <= 0 || nB > kRouteBlocksCap || n_rb < 0 || n_rb > nB) return cudaErrorInvalidValue;
  const size_t smem = static_cast<size_t>(nB) * 4 + static_cast<size_t>(n_rb) * 4;
  cudaError_t e = cudaFuncSetAttribute(route_blocks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem < 48 * 1024 ? 48 * 1024 : smem));
  if (e != cudaSuccess) return e;
  route_blocks_kernel<<<BH, 1024, smem, st>>>(sharp, routed_blk, routed_rows, score_out, N_src + N_ctx, N_src,
                                               N_ctx, blk, nSB, nB, n_rb, status);
  return cudaGetLastError();
}

}  // namespace isa
