// saliency_tc.cu -- ISA stage 1, context pre-selection: the block-level
// saliency on the tensor cores.
//
// Reading of the pre-selection step of "Lightning Unified Video Editing via
// In-Context Sparse Attention" (abstract, first insight): the saliency of a
// key block c is the attention mass it receives at block level,
//   sal_c = sum_r cnt_r * softmax_c( s * Qbar_r . Kbar_c + ln cnt_c ) / N,
// over all key blocks c (source and context) and all query blocks r.
//
// The block means arrive from the pooling kernel as bf16 hi + lo pairs
// (x = hi + lo to about 16 mantissa bits) in row-major [BH, nBp, D] arrays,
// nBp = nB rounded up to 128 (pad rows masked).  A CTA owns one 128 x 128 tile
// (query blocks of row tile rt, key blocks of column tile ct) of one (b, h)
// and computes its logits with three UMMA chains into one fp32 TMEM
// accumulator,  Qhi.Khi + Qhi.Klo + Qlo.Khi  (the lo.lo term is below fp32
// rounding), which makes the logits fp32-grade: the ranking that picks the
// kept context blocks sees the same values a float64 evaluation does to
// about 1e-6 relative.
//
// Two launches of the same tile kernel (a two-phase row softmax):
//  PASS 1 writes each row's (max, sum of 2^(x - max)) over its tile, x the
//         logit in log2 units;
//  PASS 2 recomputes the tile (the same UMMAs, bit-identical logits),
//         combines the row's statistics over all column tiles into its
//         softmax normaliser, and writes the tile's column sums of
//         cnt_r * 2^(x_rc - M_r) / S_r over its rows for the context
//         columns; the selection kernel adds the row tiles' sums in order
//         and divides by N.
// One thread per query row (TMEM lane); one thread issues the TMA loads and
// the UMMAs; every wait is bounded (status word on expiry).
#include <cmath>

#include "isa_internal.h"
#include "tc_ptx.cuh"

namespace isa {

namespace {

__device__ __forceinline__ int sal_block_count(int b, int nSB, int N_src, int N_ctx, int blk) {
  return b < nSB ? min(blk, N_src - b * blk) : min(blk, N_ctx - (b - nSB) * blk);
}

template <int D>
struct SalCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;  // one operand tile: 128 rows x D bf16
  static constexpr int RED_BYTES = 128 * 129 * 4;  // column-sum transpose (reuses the operand tiles)
  static constexpr int OPS = 4 * TILE_BYTES > RED_BYTES ? 4 * TILE_BYTES : (RED_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_BAR = OPS;             // after Qhi, Qlo, Khi, Klo
  static constexpr int OFF_LC = OFF_BAR + 64;     // log2 cnt of the tile's 128 columns
  static constexpr int SMEM = OFF_LC + 128 * 4 + 1024;
};

}  // namespace

template <int D, int PASS>
__global__ void __launch_bounds__(128, 1)
    sal_tile_kernel(const __grid_constant__ CUtensorMap tmQhi, const __grid_constant__ CUtensorMap tmQlo,
                    const __grid_constant__ CUtensorMap tmKhi, const __grid_constant__ CUtensorMap tmKlo,
                    float2* __restrict__ stats, float* __restrict__ partial, int N_src, int N_ctx, int blk, int nSB,
                    int nB, int nBp, float scale_log2, int* __restrict__ status) {
  using C = SalCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_done = bar_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_full + 2);
  int* sflag = reinterpret_cast<int*>(bar_full + 3);
  float* lc = reinterpret_cast<float*>(smem + C::OFF_LC);
  const int ct = blockIdx.x, rt = blockIdx.y, bh = blockIdx.z;
  const int nCT = gridDim.x, nRT = gridDim.y;
  const int tid = threadIdx.x, warp = tid >> 5;

  if (tid == 0) {
    mbar_init(bar_full, 1);
    mbar_init(bar_done, 1);
    *sflag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQhi);
    tma_prefetch_desc(&tmQlo);
    tma_prefetch_desc(&tmKhi);
    tma_prefetch_desc(&tmKlo);
  }
  {
    const int c = ct * 128 + tid;  // this thread's column: its key block's log2 cnt
    lc[tid] = c < nB ? log2f(static_cast<float>(sal_block_count(c, nSB, N_src, N_ctx, blk))) : -INFINITY;
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    const CUtensorMap* maps[4] = {&tmQhi, &tmQlo, &tmKhi, &tmKlo};
    mbar_arrive_expect_tx(bar_full, 4 * C::TILE_BYTES);
    for (int a = 0; a < 4; ++a) {
      const int row = bh * nBp + (a < 2 ? rt : ct) * 128;
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_2d(smem + a * C::TILE_BYTES + c * (128 * 128), maps[a], bar_full, c * 64, row);
    }
    if (mbar_wait_bounded(bar_full, 0, nullptr, kWaitLimitNs) == 0) {
      tc_fence_after();
      constexpr uint32_t IDS = idesc_bf16(128, 128, 0);
      const uint32_t qh = smem_u32(smem), ql = qh + C::TILE_BYTES, kh = ql + C::TILE_BYTES, kl = kh + C::TILE_BYTES;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t o = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
        umma_bf16(tmem, desc_k_sw128(qh + o), desc_k_sw128(kh + o), IDS, kk > 0 ? 1u : 0u);
        umma_bf16(tmem, desc_k_sw128(qh + o), desc_k_sw128(kl + o), IDS, 1u);
        umma_bf16(tmem, desc_k_sw128(ql + o), desc_k_sw128(kh + o), IDS, 1u);
      }
    } else {
      *reinterpret_cast<volatile int*>(sflag) = 1;
      if (status != nullptr) atomicCAS(status, 0, 5 /* ISA_ERR_DEVICE_TIMEOUT */);
    }
    umma_commit(bar_done);  // arrives once every UMMA issued above is done (at once if none)
  }
  __syncwarp();
  const bool done = mbar_wait_bounded(bar_done, 0, nullptr, kWaitLimitNs) == 0;
  if (!done && status != nullptr) atomicCAS(status, 0, 5);
  tc_fence_after();
  const bool ok = __all_sync(0xffffffffu, done) && *reinterpret_cast<volatile int*>(sflag) == 0;

  const int r = tid;                // row of the tile = TMEM lane
  const int grow = rt * 128 + r;    // query block
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  // logits of this row for columns [32j, 32j + 32) of the tile, log2 units;
  // columns past nB (zero or stale pad rows of Kbar) are -inf
  auto logits = [&](int j, float (&x)[32]) {
    uint32_t u[32];
    tmem_ld32(tmem + lane_base + j * 32, u);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float l = lc[j * 32 + i];
      x[i] = l == -INFINITY ? -INFINITY : fmaf(__uint_as_float(u[i]), scale_log2, l);
    }
  };
  if constexpr (PASS == 1) {
    if (ok) {
      float m = -INFINITY;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        float x[32];
        logits(j, x);
#pragma unroll
        for (int i = 0; i < 32; ++i) m = fmaxf(m, x[i]);
      }
      float s = 0.f;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        float x[32];
        logits(j, x);
#pragma unroll
        for (int i = 0; i < 32; ++i) s += exp2f(x[i] - m);  // -inf columns add 0
      }
      if (grow < nB) stats[(static_cast<size_t>(bh) * nCT + ct) * nBp + grow] = make_float2(m, s);
    }
  } else {
    // the row's softmax normaliser from every column tile's (max, sum)
    float w = 0.f, M = 0.f;
    if (ok && grow < nB) {
      M = -INFINITY;
      for (int t = 0; t < nCT; ++t) M = fmaxf(M, stats[(static_cast<size_t>(bh) * nCT + t) * nBp + grow].x);
      float S = 0.f;
      for (int t = 0; t < nCT; ++t) {
        const float2 ms = stats[(static_cast<size_t>(bh) * nCT + t) * nBp + grow];
        S += ms.y * exp2f(ms.x - M);
      }
      w = static_cast<float>(sal_block_count(grow, nSB, N_src, N_ctx, blk)) / S;
    }
    __syncthreads();  // the operand tiles are free (every UMMA completed before bar_done)
    float* red = reinterpret_cast<float*>(smem);  // [column][row], rows padded to 129
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
      float x[32];
      if (ok) logits(j, x);
#pragma unroll
      for (int i = 0; i < 32; ++i) red[(j * 32 + i) * 129 + r] = w > 0.f ? w * exp2f(x[i] - M) : 0.f;
    }
    __syncthreads();
    const int c = ct * 128 + tid;  // this thread's column
    if (ok && c >= nSB && c < nB) {
      float colsum = 0.f;
      for (int rr = 0; rr < 128; ++rr) colsum += red[tid * 129 + rr];  // rows in order
      partial[(static_cast<size_t>(bh) * nRT + rt) * (nB - nSB) + (c - nSB)] = colsum;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

cudaError_t launch_saliency_tc(const uint16_t* Qhi, const uint16_t* Qlo, const uint16_t* Khi, const uint16_t* Klo,
                               float2* stats, float* partial, int BH, int N_src, int N_ctx, int D, int blk,
                               float scale, int* status, cudaStream_t st) {
  const int nSB = (N_src + blk - 1) / blk, nCB = (N_ctx + blk - 1) / blk, nB = nSB + nCB;
  if (nCB == 0) return cudaSuccess;
  const int nBp = (nB + 127) / 128 * 128;
  CUtensorMap tm[4];
  const uint16_t* src[4] = {Qhi, Qlo, Khi, Klo};
  for (int a = 0; a < 4; ++a)
    if (!make_tmap_bf16(&tm[a], src[a], static_cast<uint64_t>(BH) * nBp, D, 128)) return cudaErrorInvalidValue;
  const dim3 grid(nBp / 128, nBp / 128, BH);
  const float sl2 = scale * 1.4426950408889634f;
  cudaError_t e;
  auto run = [&](auto kern, int smem) -> cudaError_t {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    kern<<<grid, 128, smem, st>>>(tm[0], tm[1], tm[2], tm[3], stats, partial, N_src, N_ctx, blk, nSB, nB, nBp, sl2,
                                  status);
    return cudaGetLastError();
  };
  if (D == 128) {
    if ((e = run(sal_tile_kernel<128, 1>, SalCfg<128>::SMEM)) != cudaSuccess) return e;
    return run(sal_tile_kernel<128, 2>, SalCfg<128>::SMEM);
  }
  if (D == 64) {
    if ((e = run(sal_tile_kernel<64, 1>, SalCfg<64>::SMEM)) != cudaSuccess) return e;
    return run(sal_tile_kernel<64, 2>, SalCfg<64>::SMEM);
  }
  return cudaErrorInvalidValue;
}

}  // namespace isa
