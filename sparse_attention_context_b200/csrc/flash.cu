// flash.cu -- the one-tile tcgen05 attention engine (the SHARP and TAYLOR
// kernels of the stage-by-stage ABI; the dense, routed-full and fused
// sharpness+Taylor kernels use the two-tile engine of flash2.cu).
//
// One CTA owns 128 query rows of one (b, h) and streams key tiles of BN
// rows through shared memory (TMA, 128-byte swizzle, two stages).  The
// score tile S = Q K^T and the output O += P V are tcgen05 UMMAs with fp32
// accumulators in tensor memory; softmax runs in registers, one query row
// per thread.  Modes:
//   DENSE   all N keys of the head, contiguous queries (in-house baseline).
//   FULL    ISA stage 3: gathered routed queries, keys of every source
//           block plus the kept context blocks (one block per tile, BN =
//           block, partial blocks masked by their token count).
//   TAYLOR  ISA stage 4: gathered Taylor queries, keys = kept block means
//           (bf16), values = kept block-mean values, +log2(cnt) bias.
//   SHARP   ISA stage 2: contiguous queries, keys = kept block means split
//           into bf16 hi + lo parts (two UMMAs into one accumulator, fp32-
//           grade logits), +log2(cnt) bias; writes max softmax probability.
// Method source: "Lightning Unified Video Editing via In-Context Sparse
// Attention", abstract (full attention for high-error queries, 0-th order
// Taylor sparse attention for the rest, sharpness as the error proxy).
//
// Warp roles (192 threads): warps 0-3 load Q, run softmax and the epilogue
// (thread i <-> query row i <-> TMEM lane i); warp 4 issues TMA loads;
// warp 5 allocates TMEM and one lane issues every UMMA.
// TMEM columns: S double buffer [0, 2*BN), O [2*BN, 2*BN + D).
// Every mbarrier wait is bounded; on expiry the kernel records
// ISA_ERR_DEVICE_TIMEOUT, raises a CTA-wide abort flag, drains its own
// in-flight copies and MMAs, frees TMEM and returns.
#include <cmath>

#include "gather.cuh"
#include "isa_internal.h"
#include "tc_ptx.cuh"

namespace isa {

template <int D, int BN, int MODE>
struct FlashCfg {
  static constexpr int BM = 128;
  static constexpr int STAGES = 2;
  static constexpr bool kPV = MODE != MODE_SHARP;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int P_BYTES = kPV ? BM * BN * 2 : 0;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_P = OFF_V + STAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;  // + barriers + alignment slack
  static constexpr int TMEM_NEED = 2 * BN + (kPV ? D : 0);
  static constexpr int TMEM_COLS = TMEM_NEED <= 32    ? 32
                                   : TMEM_NEED <= 64  ? 64
                                   : TMEM_NEED <= 128 ? 128
                                   : TMEM_NEED <= 256 ? 256
                                                      : 512;
  static constexpr int THREADS = 192;
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BN == 64 || BN == 128, "key tile");
};

struct FlashBars {
  uint64_t q_full;
  uint64_t k_full[2];
  uint64_t v_full[2];
  uint64_t kv_empty[2];
  uint64_t s_full[2];
  uint64_t p_full[2];  // one per S buffer: softmax may run a tile ahead of the issuer
  uint64_t o_done;
  uint64_t teardown;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void raise_timeout(FlashBars* bars, const FlashParams& p) {
  *reinterpret_cast<volatile int*>(&bars->abort) = 1;
  if (p.status != nullptr) atomicCAS(p.status, 0, 5 /* ISA_ERR_DEVICE_TIMEOUT */);
}

// Bounded wait by a single thread; true when the phase completed.
__device__ __forceinline__ bool wait1(uint64_t* bar, uint32_t par, FlashBars* bars, const FlashParams& p) {
  const int r = mbar_wait_bounded(bar, par, reinterpret_cast<volatile int*>(&bars->abort), kWaitLimitNs);
  if (r == 2) raise_timeout(bars, p);
  return r == 0;
}
// Bounded wait by a whole warp; the verdict is made warp-uniform so that the
// warp-collective tcgen05.ld/st that follow never diverge.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t par, FlashBars* bars, const FlashParams& p) {
  const bool ok = wait1(bar, par, bars, p);
  return __all_sync(0xffffffffu, ok);
}

template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

template <int BN, int MODE>
__device__ __forceinline__ int kv_row0(const FlashParams& p, int bh, int t) {
  if constexpr (MODE == MODE_FULL) {
    const int start = (t < p.nSB) ? t * p.blk
                                  : p.N_src + __ldg(p.kept_ctx + static_cast<size_t>(bh) * p.n_keep + (t - p.nSB)) * p.blk;
    return bh * p.N + start;
  } else if constexpr (MODE == MODE_DENSE) {
    return bh * p.N + t * BN;
  } else {
    return bh * p.kv_rows_per_head + t * BN;
  }
}

template <int BN, int MODE>
__device__ __forceinline__ int kv_valid(const FlashParams& p, int bh, int t) {
  if constexpr (MODE == MODE_FULL) {
    if (t < p.nSB) return min(p.blk, p.N_src - t * p.blk);
    const int c = __ldg(p.kept_ctx + static_cast<size_t>(bh) * p.n_keep + (t - p.nSB));
    return min(p.blk, p.N_ctx - c * p.blk);
  } else if constexpr (MODE == MODE_DENSE) {
    return min(BN, p.N - t * BN);
  } else {
    return BN;
  }
}

template <int D, int BN, int MODE>
__global__ void __launch_bounds__(192, 1)
    flash_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const FlashParams p) {
  using C = FlashCfg<D, BN, MODE>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  FlashBars* bars = reinterpret_cast<FlashBars*>(smem + C::OFF_BAR);
  const uint32_t aQ = smem_u32(smem + C::OFF_Q);
  const uint32_t aK = smem_u32(smem + C::OFF_K);
  const uint32_t aV = smem_u32(smem + C::OFF_V);
  const uint32_t aP = smem_u32(smem + C::OFF_P);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, bh = blockIdx.y;
  const int nT = p.n_kv_tiles;

  if (tid == 0) {
    mbar_init(&bars->q_full, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
    }
    mbar_init(&bars->p_full[0], 128);
    mbar_init(&bars->p_full[1], 128);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->teardown, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int t = 0; t < nT; ++t) {
        const int st = t % STAGES;
        if (t >= STAGES && !wait1(&bars->kv_empty[st], ((t / STAGES) - 1) & 1, bars, p)) break;
        const int row0 = kv_row0<BN, MODE>(p, bh, t);
        const uint32_t koff = C::OFF_K + st * C::KV_BYTES, voff = C::OFF_V + st * C::KV_BYTES;
        mbar_arrive_expect_tx(&bars->k_full[st], C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) tma_load_2d(smem + koff + c * (BN * 128), &tmK, &bars->k_full[st], c * 64, row0);
        mbar_arrive_expect_tx(&bars->v_full[st], C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) tma_load_2d(smem + voff + c * (BN * 128), &tmV, &bars->v_full[st], c * 64, row0);
        issued = t + 1;
      }
      // Drain: every copy this thread issued has landed before the CTA exits.
      for (int t = issued > STAGES ? issued - STAGES : 0; t < issued; ++t) {
        const int st = t % STAGES;
        const uint32_t par = (t / STAGES) & 1;
        mbar_wait_bounded(&bars->k_full[st], par, nullptr, kWaitLimitNs);
        mbar_wait_bounded(&bars->v_full[st], par, nullptr, kWaitLimitNs);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t IDS = idesc_bf16(128, BN, 0);
      constexpr uint32_t IDO = idesc_bf16(128, D, 1);
      bool ok = wait1(&bars->q_full, 0, bars, p);
      tc_fence_after();
      auto issue_S = [&](int t) -> bool {
        const int st = t % STAGES;
        const uint32_t par = (t / STAGES) & 1;
        if (!wait1(&bars->k_full[st], par, bars, p)) return false;
        if constexpr (MODE == MODE_SHARP) {
          if (!wait1(&bars->v_full[st], par, bars, p)) return false;
        }
        tc_fence_after();
        const uint32_t dS = tmem + (t & 1) * BN;
        const uint32_t kb = aK + st * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = desc_k_sw128(aQ + (kk >> 2) * (128 * 128) + (kk & 3) * 32);
          const uint64_t b = desc_k_sw128(kb + (kk >> 2) * (BN * 128) + (kk & 3) * 32);
          umma_bf16(dS, a, b, IDS, kk > 0 ? 1u : 0u);
        }
        if constexpr (MODE == MODE_SHARP) {  // + Q * Klo^T
          const uint32_t lb = aV + st * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = desc_k_sw128(aQ + (kk >> 2) * (128 * 128) + (kk & 3) * 32);
            const uint64_t b = desc_k_sw128(lb + (kk >> 2) * (BN * 128) + (kk & 3) * 32);
            umma_bf16(dS, a, b, IDS, 1u);
          }
        }
        umma_commit(&bars->s_full[t & 1]);
        if constexpr (MODE == MODE_SHARP) umma_commit(&bars->kv_empty[st]);
        return true;
      };
      if (ok && nT > 0) ok = issue_S(0);
      for (int t = 0; ok && t < nT; ++t) {
        if (t + 1 < nT && !(ok = issue_S(t + 1))) break;
        if (!(ok = wait1(&bars->p_full[t & 1], (t >> 1) & 1, bars, p))) break;
        if constexpr (C::kPV) {
          const int st = t % STAGES;
          if (!(ok = wait1(&bars->v_full[st], (t / STAGES) & 1, bars, p))) break;
          tc_fence_after();
          const uint32_t vb = aV + st * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t a = desc_k_sw128(aP + (kk >> 2) * (128 * 128) + (kk & 3) * 32);
            const uint64_t b = desc_mn_sw128(vb + kk * 16 * 128, BN * 128);
            umma_bf16(tmem + 2 * BN, a, b, IDO, (t > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars->o_done);
          umma_commit(&bars->kv_empty[st]);
        }
      }
      // Every UMMA issued above completes before TMEM is released.
      umma_commit(&bars->teardown);
      mbar_wait_bounded(&bars->teardown, 0, nullptr, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------------- Q load, softmax, epilogue
    const int r0 = tile * 128;
    gather_rows_sw128<D>(p.q, p.row_idx, bh, p.n_rows, p.N, r0, tid, aQ, false, p.status);
    fence_proxy_async_smem();
    mbar_arrive(&bars->q_full);

    const int r = tid;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    if (p.inject != nullptr && (__ldg(p.inject) & 1)) {  // test hook: behave as if S never arrived
      raise_timeout(bars, p);
      ok = false;
    }
    for (int t = 0; ok && t < nT; ++t) {
      if (!(ok = wait_warp(&bars->s_full[t & 1], (t >> 1) & 1, bars, p))) break;
      tc_fence_after();
      float x[BN];
      {
        uint32_t u[BN / 32][32];
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) tmem_ld32(tmem + lane_base + (t & 1) * BN + j * 32, u[j]);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) {
          reg_fence(u[j]);
#pragma unroll
          for (int i = 0; i < 32; ++i) x[j * 32 + i] = __uint_as_float(u[j][i]);
        }
      }
      float mt = -INFINITY;
      if constexpr (MODE == MODE_TAYLOR || MODE == MODE_SHARP) {
        const float4* bp = reinterpret_cast<const float4*>(p.bias2 + static_cast<size_t>(bh) * p.kv_rows_per_head + t * BN);
#pragma unroll
        for (int c4 = 0; c4 < BN / 4; ++c4) {
          const float4 b = __ldg(bp + c4);
          x[4 * c4 + 0] = fmaf(x[4 * c4 + 0], p.scale_log2, b.x);
          x[4 * c4 + 1] = fmaf(x[4 * c4 + 1], p.scale_log2, b.y);
          x[4 * c4 + 2] = fmaf(x[4 * c4 + 2], p.scale_log2, b.z);
          x[4 * c4 + 3] = fmaf(x[4 * c4 + 3], p.scale_log2, b.w);
        }
#pragma unroll
        for (int c = 0; c < BN; ++c) mt = fmaxf(mt, x[c]);
      } else {
        const int valid = kv_valid<BN, MODE>(p, bh, t);
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          x[c] = (c < valid) ? x[c] * p.scale_log2 : -INFINITY;
          mt = fmaxf(mt, x[c]);
        }
      }

      if constexpr (MODE == MODE_SHARP) {
        const float m_new = fmaxf(m, mt);
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < BN; ++c) sum += ex2(x[c] - m_new);
        l = l * ex2(m - m_new) + sum;
        m = m_new;
        tc_fence_before();
        mbar_arrive(&bars->p_full[t & 1]);
      } else {
        if (t > 0) {
          if (!(ok = wait_warp(&bars->o_done, (t - 1) & 1, bars, p))) break;
          tc_fence_after();
        }
        const float m_new = fmaxf(m, mt);
        // Rescale only when the running maximum grew by more than 2^8: the
        // stale reference keeps every p <= 256, exact after the final 1/l.
        const bool need = m_new > m + 8.0f;
        if (t > 0 && __any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2(m - m_new) : 1.f;
#pragma unroll
          for (int j = 0; j < D / 32; ++j) {
            uint32_t u[32];
            tmem_ld32(tmem + lane_base + 2 * BN + j * 32, u);
            tmem_wait_ld();
            reg_fence(u);
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
            tmem_st32(tmem + lane_base + 2 * BN + j * 32, u);
          }
          tmem_wait_st();
        }
        if (need) {
          l *= ex2(m - m_new);
          m = m_new;
        }
        const float mref = (m == -INFINITY) ? 0.f : m;
        float sum = 0.f;
#pragma unroll
        for (int a = 0; a < BN / 64; ++a) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float e[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              e[i] = ex2(x[a * 64 + j * 8 + i] - mref);
              sum += e[i];
            }
            st_shared_v4(aP + a * (128 * 128) + sw128(r, j), pack_bf16(e[0], e[1]), pack_bf16(e[2], e[3]),
                         pack_bf16(e[4], e[5]), pack_bf16(e[6], e[7]));
          }
        }
        l += sum;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->p_full[t & 1]);
      }
    }

    const int g = r0 + r;
    const bool valid_row = g < p.n_rows;
    if constexpr (MODE == MODE_SHARP) {
      if (ok && valid_row) p.sharp[static_cast<size_t>(bh) * p.N + g] = 1.f / l;
    } else {
      if (ok && nT > 0 && wait_warp(&bars->o_done, (nT - 1) & 1, bars, p)) {
        tc_fence_after();
        int dst = valid_row ? (p.row_idx ? __ldg(p.row_idx + static_cast<size_t>(bh) * p.n_rows + g) : g) : 0;
        const bool store = valid_row && static_cast<unsigned>(dst) < static_cast<unsigned>(p.N);
        if (!store) dst = 0;
        uint16_t* orow = p.out + (static_cast<size_t>(bh) * p.N + dst) * D;
        const float inv = 1.f / l;
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
          uint32_t u[32];
          tmem_ld32(tmem + lane_base + 2 * BN + j * 32, u);
          tmem_wait_ld();
          reg_fence(u);
          if (store) {
            uint4* o4 = reinterpret_cast<uint4*>(orow + j * 32);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(u[8 * q4 + 0]) * inv, __uint_as_float(u[8 * q4 + 1]) * inv);
              w.y = pack_bf16(__uint_as_float(u[8 * q4 + 2]) * inv, __uint_as_float(u[8 * q4 + 3]) * inv);
              w.z = pack_bf16(__uint_as_float(u[8 * q4 + 4]) * inv, __uint_as_float(u[8 * q4 + 5]) * inv);
              w.w = pack_bf16(__uint_as_float(u[8 * q4 + 6]) * inv, __uint_as_float(u[8 * q4 + 7]) * inv);
              o4[q4] = w;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// At most `k` CTAs of this kernel may share an SM (TMEM budget): request
// enough dynamic shared memory that a (k+1)-th cannot fit.
static int smem_request(int need, int tmem_cols) {
  const int per_sm = 233472;  // 228 KiB shared memory per SM
  const int k = 512 / tmem_cols;
  const int floor_bytes = per_sm / (k + 1) - 1024 + 16;
  return need > floor_bytes ? need : floor_bytes;
}

template <int D, int BN, int MODE>
static cudaError_t launch_t(const CUtensorMap& tmK, const CUtensorMap& tmV, const FlashParams& p, int BH,
                            cudaStream_t st) {
  using C = FlashCfg<D, BN, MODE>;
  const int smem = smem_request(C::SMEM, C::TMEM_COLS);
  auto kern = flash_kernel<D, BN, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((p.n_rows + 127) / 128, BH);
  kern<<<grid, C::THREADS, smem, st>>>(tmK, tmV, p);
  return cudaGetLastError();
}

cudaError_t launch_flash(int D, int BN, int mode, const CUtensorMap& tmK, const CUtensorMap& tmV,
                         const FlashParams& p, int BH, cudaStream_t st) {
  if (p.n_rows <= 0 || BH <= 0) return cudaSuccess;
#define ISA_FLASH_CASE(d_, bn_, m_) \
  if (D == d_ && BN == bn_ && mode == m_) return launch_t<d_, bn_, m_>(tmK, tmV, p, BH, st);
  ISA_FLASH_CASE(128, 128, MODE_TAYLOR)
  ISA_FLASH_CASE(128, 128, MODE_SHARP)
  ISA_FLASH_CASE(64, 128, MODE_TAYLOR)
  ISA_FLASH_CASE(64, 128, MODE_SHARP)
#undef ISA_FLASH_CASE
  return cudaErrorInvalidValue;
}

}  // namespace isa
