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
// nBp = nB rounded up to 128 (pad rows masked).  Each 128 x 128 tile of
// logits (the query blocks of a row tile against the key blocks of a column
// tile) is three UMMA chains into one fp32 TMEM accumulator,
// Qhi.Khi + Qhi.Klo + Qlo.Khi  (the lo.lo term is below fp32
// rounding), which makes the logits fp32-grade: the ranking that picks the
// kept context blocks sees the same values a float64 evaluation does to
// about 1e-6 relative.
//
// One CTA per 128-row tile of query blocks of one (b, h) (grid: row tiles x
// B*H, 576 threads).  Warp 16 streams the Kbar tiles (TMA, two stages), warp
// 17 issues the UMMAs into two 128-column score buffers in tensor memory, so
// the logits of the next column tile are computed while the current one is
// read.  Warps 0-15 read the scores: warp w takes TMEM lanes (rows)
// 32*(w%4) .. +31 and the 32 columns 32*(w/4) .. +31 of each tile, four
// warps per SM sub-partition to hide the exponentials' latency.
//  pass 1 (every column tile, in order) keeps per row and column quarter a
//         running (max, sum of 2^(x - max)), x the logit in log2 units; the
//         four quarters are combined once, through shared memory, into the
//         row's softmax normaliser;
//  pass 2 (the column tiles that hold context blocks, last first) takes the
//         tile's column sums of cnt_r * 2^(x_rc - M_r) / S_r over its 128
//         rows: a butterfly reduce-scatter per warp, then the four row
//         groups' sums in order.  The last tile of pass 1 is still in
//         registers and is not recomputed.  The selection kernel adds the
//         row tiles' sums in order and divides by N.
// Every wait is bounded (status word and CTA abort flag on expiry).
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
  static constexpr int TILE_BYTES = 128 * D * 2;            // one operand tile: 128 rows x D bf16
  static constexpr int OFF_Q = 0;                           // Qhi, Qlo
  static constexpr int OFF_K = 2 * TILE_BYTES;              // two stages of Khi, Klo
  static constexpr int OFF_RED = OFF_K + 4 * TILE_BYTES;    // [2 buffers][4 row groups][128 columns] fp32
  static constexpr int OFF_STAT = OFF_RED + 2 * 4 * 128 * 4;  // [4 column quarters][128 rows] (max, sum)
  static constexpr int OFF_BAR = OFF_STAT + 4 * 128 * 8;
  static constexpr int SMEM = OFF_BAR + 128 + 1024;         // + alignment slack
  static constexpr int EPI_WARPS = 16;
  static constexpr int THREADS = (EPI_WARPS + 2) * 32;
};

struct SalBars {
  uint64_t q_full;
  uint64_t k_full[2];
  uint64_t k_empty[2];  // K stage free: the UMMAs reading it are done
  uint64_t s_full[2];   // score buffer written
  uint64_t s_free[2];   // score buffer read by all 128 rows
  uint64_t teardown;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool sal_wait(uint64_t* bar, uint32_t par, SalBars* bars, int* status) {
  const int r = mbar_wait_bounded(bar, par, reinterpret_cast<volatile int*>(&bars->abort), kWaitLimitNs);
  if (r == 2) {
    *reinterpret_cast<volatile int*>(&bars->abort) = 1;
    if (status != nullptr) atomicCAS(status, 0, 5 /* ISA_ERR_DEVICE_TIMEOUT */);
  }
  return r == 0;
}

// Lane L of the warp returns the sum over the warp's 32 lanes of v[L]
// (v is consumed).  Five halving steps: at step w each lane keeps the half
// of its columns selected by lane bit w and adds the partner's copy of it.
__device__ __forceinline__ float warp_reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = upper ? v[i] : v[i + w];
      const float keep = upper ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(SalCfg<D>::THREADS, 1)
    sal_row_kernel(const __grid_constant__ CUtensorMap tmQhi, const __grid_constant__ CUtensorMap tmQlo,
                   const __grid_constant__ CUtensorMap tmKhi, const __grid_constant__ CUtensorMap tmKlo,
                   float* __restrict__ partial, int N_src, int N_ctx, int blk, int nSB, int nB, int nBp,
                   float scale_log2, int* __restrict__ status) {
  using C = SalCfg<D>;
  constexpr int W_LOAD = C::EPI_WARPS, W_MMA = C::EPI_WARPS + 1;
  constexpr int EPI_THREADS = C::EPI_WARPS * 32;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  SalBars* bars = reinterpret_cast<SalBars*>(smem + C::OFF_BAR);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  float2* qstat = reinterpret_cast<float2*>(smem + C::OFF_STAT);
  const int rt = blockIdx.x, bh = blockIdx.y;
  const int nCT = nBp / 128;   // column tiles (= row tiles)
  const int ct0 = nSB / 128;   // first column tile holding a context block
  const int nE = 2 * nCT - 1 - ct0;  // tile evaluations: pass 1, then pass 2 less the last tile
  // column tile of evaluation e: 0 .. nCT-1, then nCT-2 down to ct0
  auto ct_of = [&](int e) { return e < nCT ? e : nCT - 2 - (e - nCT); };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->s_free[s], EPI_THREADS);
    }
    mbar_init(&bars->teardown, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(&bars->tmem_base, 256);
    tmem_relinquish();
  }
  if (warp == W_LOAD && lane == 0) {
    tma_prefetch_desc(&tmQhi);
    tma_prefetch_desc(&tmQlo);
    tma_prefetch_desc(&tmKhi);
    tma_prefetch_desc(&tmKlo);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == W_LOAD) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars->q_full, 2 * C::TILE_BYTES);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_2d(smem + C::OFF_Q + c * (128 * 128), &tmQhi, &bars->q_full, c * 64, bh * nBp + rt * 128);
        tma_load_2d(smem + C::OFF_Q + C::TILE_BYTES + c * (128 * 128), &tmQlo, &bars->q_full, c * 64,
                    bh * nBp + rt * 128);
      }
      int issued = 0;
      for (int e = 0; e < nE; ++e) {
        const int s = e & 1;
        if (e >= 2 && !sal_wait(&bars->k_empty[s], ((e >> 1) - 1) & 1, bars, status)) break;
        uint8_t* kb = smem + C::OFF_K + s * 2 * C::TILE_BYTES;
        const int row = bh * nBp + ct_of(e) * 128;
        mbar_arrive_expect_tx(&bars->k_full[s], 2 * C::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_2d(kb + c * (128 * 128), &tmKhi, &bars->k_full[s], c * 64, row);
          tma_load_2d(kb + C::TILE_BYTES + c * (128 * 128), &tmKlo, &bars->k_full[s], c * 64, row);
        }
        issued = e + 1;
      }
      for (int e = issued > 2 ? issued - 2 : 0; e < issued; ++e)  // drain own copies
        mbar_wait_bounded(&bars->k_full[e & 1], (e >> 1) & 1, nullptr, kWaitLimitNs);
      mbar_wait_bounded(&bars->q_full, 0, nullptr, kWaitLimitNs);
    }
  } else if (warp == W_MMA) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t IDS = idesc_bf16(128, 128, 0);
      const uint32_t qh = smem_u32(smem + C::OFF_Q), ql = qh + C::TILE_BYTES;
      bool ok = sal_wait(&bars->q_full, 0, bars, status);
      for (int e = 0; ok && e < nE; ++e) {
        const int s = e & 1;
        if (!(ok = sal_wait(&bars->k_full[s], (e >> 1) & 1, bars, status))) break;
        if (e >= 2 && !(ok = sal_wait(&bars->s_free[s], ((e >> 1) - 1) & 1, bars, status))) break;
        tc_fence_after();
        // logits Qhi.Khi + Qhi.Klo + Qlo.Khi (lo.lo is below fp32 rounding)
        const uint32_t kh = smem_u32(smem + C::OFF_K + s * 2 * C::TILE_BYTES), kl = kh + C::TILE_BYTES;
        const uint32_t dS = tmem + s * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          umma_bf16(dS, desc_k_sw128(qh + o), desc_k_sw128(kh + o), IDS, kk > 0 ? 1u : 0u);
          umma_bf16(dS, desc_k_sw128(qh + o), desc_k_sw128(kl + o), IDS, 1u);
          umma_bf16(dS, desc_k_sw128(ql + o), desc_k_sw128(kh + o), IDS, 1u);
        }
        umma_commit(&bars->s_full[s]);
        umma_commit(&bars->k_empty[s]);
      }
      umma_commit(&bars->teardown);  // every UMMA issued above is done
      mbar_wait_bounded(&bars->teardown, 0, nullptr, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------------- rows: softmax, column sums
    const int lg = warp & 3;          // row group: TMEM lanes 32*lg .. +31
    const int qc = warp >> 2;         // column quarter of each tile
    const int r = lg * 32 + lane;     // row of the tile = TMEM lane
    const int grow = rt * 128 + r;    // query block
    const uint32_t taddr = tmem + (static_cast<uint32_t>(lg * 32) << 16) + qc * 32;
    const float l_full = log2f(static_cast<float>(blk));
    const float l_src_last = log2f(static_cast<float>(sal_block_count(nSB - 1, nSB, N_src, N_ctx, blk)));
    const float l_ctx_last = log2f(static_cast<float>(sal_block_count(nB - 1, nSB, N_src, N_ctx, blk)));
    float m = -INFINITY, ssum = 0.f, M = 0.f, w = 0.f;
    bool ok = true;
    for (int e = 0; e < nE; ++e) {
      const int b = e & 1;
      const int cq = ct_of(e) * 128 + qc * 32;  // first column of this warp's quarter
      float x[32];
      if (ok) ok = __all_sync(0xffffffffu, sal_wait(&bars->s_full[b], (e >> 1) & 1, bars, status));
      if (ok) {
        uint32_t u[32];
        tc_fence_after();
        tmem_ld32(taddr + b * 128, u);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->s_free[b]);
        // logits in log2 units with the key block's log2 cnt; columns past
        // nB (pad rows of Kbar) are -inf
        if (cq + 32 < nB && (nSB - 1 < cq || nSB - 1 >= cq + 32)) {  // full blocks only
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = fmaf(__uint_as_float(u[i]), scale_log2, l_full);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int c = cq + i;
            const float lc = c == nSB - 1 ? l_src_last : (c == nB - 1 ? l_ctx_last : l_full);
            x[i] = c < nB ? fmaf(__uint_as_float(u[i]), scale_log2, lc) : -INFINITY;
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = -INFINITY;
      }
      if (e < nCT) {
        // pass 1: running (max, sum) of this row's column quarter
        if (ok) {
          float tm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int i = 0; i < 32; ++i) tm[i & 3] = fmaxf(tm[i & 3], x[i]);
          const float m_new = fmaxf(m, fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3])));
          if (m_new != -INFINITY) {  // a quarter of pad columns only adds nothing
            float ts[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 32; ++i) ts[i & 3] += exp2f(x[i] - m_new);  // -inf adds 0
            ssum = ssum * exp2f(m - m_new) + ((ts[0] + ts[1]) + (ts[2] + ts[3]));  // m = -inf at first: 0
            m = m_new;
          }
        }
        if (e < nCT - 1) continue;
        // the row's normaliser from its four quarters, in quarter order
        qstat[qc * 128 + r] = make_float2(m, ssum);
        asm volatile("bar.sync 1, %0;" ::"r"(EPI_THREADS) : "memory");
        float MM = -INFINITY;
#pragma unroll
        for (int q = 0; q < 4; ++q) MM = fmaxf(MM, qstat[q * 128 + r].x);
        float S = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 st = qstat[q * 128 + r];
          S += st.x == -INFINITY ? 0.f : st.y * exp2f(st.x - MM);
        }
        M = MM;
        w = (ok && grow < nB) ? static_cast<float>(sal_block_count(grow, nSB, N_src, N_ctx, blk)) / S : 0.f;
      }
      // pass 2: this tile's column sums over the 128 rows (every warp takes
      // part in each exchange, also after a failed wait, so that the named
      // barriers are reached equally often by all sixteen warps)
      float* rb = red + b * 4 * 128;
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] = (ok && w > 0.f) ? w * exp2f(x[i] - M) : 0.f;
      rb[lg * 128 + qc * 32 + lane] = warp_reduce_scatter32(x, lane);
      asm volatile("bar.sync 1, %0;" ::"r"(EPI_THREADS) : "memory");
      if (tid < 128) {
        const int c = ct_of(e) * 128 + tid;  // this thread's column
        if (ok && c >= nSB && c < nB)
          partial[(static_cast<size_t>(bh) * nCT + rt) * (nB - nSB) + (c - nSB)] =
              ((rb[tid] + rb[128 + tid]) + rb[256 + tid]) + rb[384 + tid];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

cudaError_t launch_saliency_tc(const uint16_t* Qhi, const uint16_t* Qlo, const uint16_t* Khi, const uint16_t* Klo,
                               float* partial, int BH, int N_src, int N_ctx, int D, int blk, float scale,
                               int* status, cudaStream_t st) {
  const int nSB = (N_src + blk - 1) / blk, nCB = (N_ctx + blk - 1) / blk, nB = nSB + nCB;
  if (nCB == 0) return cudaSuccess;
  const int nBp = (nB + 127) / 128 * 128;
  CUtensorMap tm[4];
  const uint16_t* src[4] = {Qhi, Qlo, Khi, Klo};
  for (int a = 0; a < 4; ++a)
    if (!make_tmap_bf16(&tm[a], src[a], static_cast<uint64_t>(BH) * nBp, D, 128)) return cudaErrorInvalidValue;
  const dim3 grid(nBp / 128, BH);
  const float sl2 = scale * 1.4426950408889634f;
  auto run = [&](auto kern, int smem) -> cudaError_t {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    kern<<<grid, SalCfg<128>::THREADS, smem, st>>>(tm[0], tm[1], tm[2], tm[3], partial, N_src, N_ctx, blk, nSB, nB,
                                                   nBp, sl2, status);
    return cudaGetLastError();
  };
  if (D == 128) return run(sal_row_kernel<128>, SalCfg<128>::SMEM);
  if (D == 64) return run(sal_row_kernel<64>, SalCfg<64>::SMEM);
  return cudaErrorInvalidValue;
}

}  // namespace isa
