// taylor1.cu -- first-order Taylor sparse attention, a variant of ISA stage 4.
//
// Method ("Lightning Unified Video Editing via In-Context Sparse
// Attention", abstract): queries that are not routed to full attention get
// a 0-th order Taylor approximation, exp(s q.k_j) -> exp(s q.Kbar_b) inside
// every kept block b.  The next order keeps the linear term,
//   exp(s q.k_j) ~= exp(s q.Kbar_b) (1 + s q.(k_j - Kbar_b)),
// whose block sums give
//   o_i = [sum_b cnt_b e_ib Vbar_b + s sum_b e_ib C_b^T q_i] / sum_b cnt_b e_ib
// with e_ib = exp(s q_i.Kbar_b) and C_b = sum_{j in b} (k_j - Kbar_b) v_j^T
// (the linear terms cancel in the denominator: deviations from a mean sum
// to zero).
//
// Two kernels:
//  * cbuild_kernel: one CTA per (b, h, kept block) computes C_b with one
//    tcgen05 UMMA, K_b^T V_b (A = K_b^T read MN-major straight from the TMA
//    tile, B = V_b MN-major), then subtracts cnt_b Kbar_b Vbar_b^T in fp32
//    and stores C_b as bf16, row-major [d_in][d_out] (the layout the second
//    kernel reads as an MN-major B operand).  Rows of a partial block past
//    its count are zeroed in V before the product.
//  * taylor1_kernel: one CTA per 256 gathered query rows of one (b, h), two
//    128-row tiles (thread <-> row <-> TMEM lane).  Per key tile of 128 kept
//    blocks: S = Q Kbar^T (UMMA), the softmax warps form the biased weights
//    P0 = cnt_b 2^(l - m) (bf16 into TMEM, A of O += P0 Vbar) and the
//    unbiased ones w = s 2^(l - m) (bf16 pairs, per-thread local memory);
//    then for every kept block b the warps write A_b = w_b q (their own q
//    row, bf16) into one of two 64-column TMEM slots and the issuer adds
//    O += A_b C_b (UMMA, A from TMEM, C_b staged by TMA in a ring shared by
//    both tiles).  The Vbar tile of a key tile travels through the same
//    ring, as the element before the key tile's C_b, so the ring is as deep
//    as shared memory allows.  Every MMA accumulates into one O per tile, so the
//    epilogue is O / l.  The running maximum m is re-based only when it
//    grows by 2^32 (then O is rescaled in TMEM; every earlier MMA is known
//    complete once S of the next key tile has landed).
//
// Warps (320 threads): 0-3 tile 0, 4-7 tile 1, 8 TMA producer, 9 TMEM
// allocator + the single UMMA issuer.  TMEM (512 columns): region of tile i
// at [128i, 128i + 128) holds S, then P0 in its first 64 columns, then the
// A slots [128i + 64s, 128i + 64s + 64), s = 0, 1; O of tile i at
// [256 + D i, 256 + D i + D).  Every wait is bounded (2 s of %globaltimer,
// then the device status word and a CTA abort flag, as in flash2.cu).
#include <cuda_bf16.h>

#include <cmath>

#include "gather.cuh"
#include "isa_internal.h"
#include "tc_ptx.cuh"

namespace isa {

namespace {

// kind::f16 instruction descriptor with A read MN-major as well as B.
__host__ __device__ constexpr uint32_t idesc_ab_mn(int M, int N) {
  return idesc_bf16(M, N, 1) | (1u << 15);
}

__device__ __forceinline__ void wg_bar_sync(int id) {  // the 128 threads of one tile
  asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a), y = *reinterpret_cast<__nv_bfloat162*>(&b);
  __nv_bfloat162 z = __hmul2(x, y);
  return *reinterpret_cast<uint32_t*>(&z);
}

template <int N>
__device__ __forceinline__ void keep_regs(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// ----------------------------------------------------------------- C_b build
template <int D>
struct CBCfg {
  static constexpr int ROWS = 128;                   // token rows staged (block <= 128)
  static constexpr int CHUNK = ROWS * 128;           // one 64-column box of 128 rows
  static constexpr int OFF_K = 0;                    // 2 chunks: K (D = 64: K + zeros)
  static constexpr int OFF_V = 2 * CHUNK;            // D / 64 chunks
  static constexpr int OFF_BAR = OFF_V + (D / 64) * CHUNK;
  static constexpr int SMEM = OFF_BAR + 64 + 1024;
};

}  // namespace

template <int D>
__global__ void __launch_bounds__(128) cbuild_kernel(const __grid_constant__ CUtensorMap tmK,
                                                     const __grid_constant__ CUtensorMap tmV,
                                                     const float* __restrict__ Kbar, const float* __restrict__ Vbar,
                                                     const int32_t* __restrict__ kept, uint16_t* __restrict__ Cout,
                                                     int N, int N_src, int N_ctx, int blk, int nSB, int nB,
                                                     int n_keep, int nK, int* status) {
  using C = CBCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* done = full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full + 2);
  const int r = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5;

  // the r-th kept block: every source block, then the kept context blocks
  int kb, start, cnt;
  if (r < nSB) {
    kb = r;
    start = r * blk;
    cnt = min(blk, N_src - start);
  } else {
    const int c = __ldg(kept + static_cast<size_t>(bh) * n_keep + (r - nSB));
    if (c < 0 || nSB + c >= nB) {  // corrupted kept set: report, write nothing
      if (tid == 0 && status != nullptr) atomicCAS(status, 0, 1);
      return;
    }
    kb = nSB + c;
    start = N_src + c * blk;
    cnt = min(blk, N_ctx - c * blk);
  }

  if (tid == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, D);
    tmem_relinquish();
  }
  if constexpr (D == 64) {  // M is padded to 128: the second 64-wide group of A reads zeros
    uint4* z = reinterpret_cast<uint4*>(smem + C::OFF_K + blk * 128);
    for (int e = tid; e < blk * 8; e += 128) z[e] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int row = bh * N + start;
  if (tid == 0) {
    mbar_arrive_expect_tx(full, 2u * (D / 64) * blk * 128);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_2d(smem + C::OFF_K + c * blk * 128, &tmK, full, c * 64, row);
      tma_load_2d(smem + C::OFF_V + c * blk * 128, &tmV, full, c * 64, row);
    }
  }
  bool ok = mbar_wait_bounded(full, 0, nullptr, kWaitLimitNs) == 0;
  if (!ok && tid == 0 && status != nullptr) atomicCAS(status, 0, 5);
  if (ok && cnt < blk) {  // rows past the block's count hold other tokens: zero them in V
    const int nz = (blk - cnt) * 8;
    for (int e = tid; e < nz * (D / 64); e += 128) {
      const int c = e / nz, rr = cnt + (e % nz) / 8, piece = e % 8;
      reinterpret_cast<uint4*>(smem + C::OFF_V + c * blk * 128 + rr * 128)[piece] = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  if (ok && tid == 0) {
    tc_fence_after();
    constexpr uint32_t ID = idesc_ab_mn(128, D);
    const uint32_t aK = smem_u32(smem + C::OFF_K), aV = smem_u32(smem + C::OFF_V);
    for (int kk = 0; kk < blk / 16; ++kk)
      umma_bf16(tmem, desc_mn_sw128(aK + kk * 16 * 128, blk * 128), desc_mn_sw128(aV + kk * 16 * 128, blk * 128), ID,
                kk > 0 ? 1u : 0u);
    umma_commit(done);
  }
  if (ok) {
    ok = mbar_wait_bounded(done, 0, nullptr, kWaitLimitNs) == 0;
    if (!ok && tid == 0 && status != nullptr) atomicCAS(status, 0, 5);
  }
  if (ok) {
    tc_fence_after();
    const int m = tid;  // d_in index = TMEM lane
    const size_t mean_row = (static_cast<size_t>(bh) * nB + kb) * D;
    const float km = m < D ? __ldg(Kbar + mean_row + m) * static_cast<float>(cnt) : 0.f;
    uint16_t* crow = Cout + ((static_cast<size_t>(bh) * nK + r) * D + (m < D ? m : 0)) * D;
#pragma unroll
    for (int j = 0; j < D / 32; ++j) {
      uint32_t u[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + j * 32, u);
      tmem_wait_ld();
      keep_regs(u);
      if (m < D) {
        uint4* o4 = reinterpret_cast<uint4*>(crow + j * 32);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t w[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int e = j * 32 + q4 * 8 + 2 * h;
            const float c0 = __uint_as_float(u[q4 * 8 + 2 * h]) - km * __ldg(Vbar + mean_row + e);
            const float c1 = __uint_as_float(u[q4 * 8 + 2 * h + 1]) - km * __ldg(Vbar + mean_row + e + 1);
            w[h] = pack_bf16(c0, c1);
          }
          o4[q4] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, D);
  }
}

// ------------------------------------------------------- first-order Taylor
namespace {

template <int D>
struct T1Cfg {
  static constexpr int BN = 128;                 // kept blocks per key tile
  static constexpr int Q_BYTES = 128 * D * 2;    // one 128-row query tile
  static constexpr int KT_BYTES = BN * D * 2;    // one Kbar / Vbar tile
  static constexpr int C_BYTES = D * D * 2;      // one correction matrix
  // ring of Vbar tiles and correction matrices (one slot holds either)
  static constexpr int SLOT = KT_BYTES > C_BYTES ? KT_BYTES : C_BYTES;
  static constexpr int R = D == 128 ? 4 : 8;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * Q_BYTES;
  static constexpr int OFF_C = OFF_K + KT_BYTES;
  static constexpr int OFF_BIAS = OFF_C + R * SLOT;  // [2][BN] log2 cnt (ring by key tile parity)
  static constexpr int OFF_BAR = OFF_BIAS + 2 * BN * 4;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(2 * BN + 2 * D <= 512, "TMEM budget");
};

struct T1Bars {
  uint64_t q_full[2];
  uint64_t k_full, k_empty;
  uint64_t c_full[8], c_empty[8];  // ring of Vbar tiles and correction matrices
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t a_full[2][2];  // [tile][slot]: A written by the tile's 128 threads
  uint64_t a_free[2][2];  // [tile][slot]: the MMA that read the slot is done
  uint64_t o_done[2];
  uint64_t teardown;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(T1Bars) <= 512, "barrier block");

__device__ __forceinline__ void t1raise(T1Bars* bars, const FlashParams& p) {
  *reinterpret_cast<volatile int*>(&bars->abort) = 1;
  if (p.status != nullptr) atomicCAS(p.status, 0, 5 /* ISA_ERR_DEVICE_TIMEOUT */);
}
__device__ __forceinline__ bool t1w(uint64_t* bar, uint32_t par, T1Bars* bars, const FlashParams& p) {
  const int r = mbar_wait_bounded(bar, par, reinterpret_cast<volatile int*>(&bars->abort), kWaitLimitNs);
  if (r == 2) t1raise(bars, p);
  return r == 0;
}
__device__ __forceinline__ bool t1warp(uint64_t* bar, uint32_t par, T1Bars* bars, const FlashParams& p) {
  const bool ok = t1w(bar, par, bars, p);
  return __all_sync(0xffffffffu, ok);
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(320, 1)
    taylor1_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmC, const FlashParams p, int nK, float scale) {
  using C = T1Cfg<D>;
  constexpr int BN = C::BN;
  constexpr int R = C::R;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  T1Bars* bars = reinterpret_cast<T1Bars*>(smem + C::OFF_BAR);
  const uint32_t aQ = smem_u32(smem + C::OFF_Q);
  const uint32_t aK = smem_u32(smem + C::OFF_K);
  const uint32_t aC = smem_u32(smem + C::OFF_C);
  const float* bias_sm = reinterpret_cast<const float*>(smem + C::OFF_BIAS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = static_cast<int>(blockIdx.x);
  const int bh = item / p.pairs_per_head;
  const int row0 = (item % p.pairs_per_head) * 256;
  const int nT = p.n_kv_tiles;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], 128);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 128);
      mbar_init(&bars->o_done[i], 1);
      for (int s = 0; s < 2; ++s) {
        mbar_init(&bars->a_full[i][s], 128);
        mbar_init(&bars->a_free[i][s], 1);
      }
    }
    mbar_init(&bars->k_full, 1);
    mbar_init(&bars->k_empty, 1);
    for (int r = 0; r < R; ++r) {
      mbar_init(&bars->c_full[r], 1);
      mbar_init(&bars->c_empty[r], 1);
    }
    mbar_init(&bars->teardown, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmC);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // ring elements issued: per key tile its Vbar tile, then its C_b
      // (unsigned, so that % R and / R are bit operations)
      unsigned ge = 0u;
      bool ok = true;
      int k_issued = 0;
      auto slot_ready = [&](unsigned e) -> bool {  // wait until ring slot e % R is free
        return e < R || t1w(&bars->c_empty[e % R], ((e / R) - 1) & 1, bars, p);
      };
      for (int t = 0; ok && t < nT; ++t) {
        if (t > 0 && !(ok = t1w(&bars->k_empty, (t - 1) & 1, bars, p))) break;
        const int kr = bh * p.kv_rows_per_head + t * BN;
        mbar_arrive_expect_tx(&bars->k_full, C::KT_BYTES + BN * 4);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) tma_load_2d(smem + C::OFF_K + c * (BN * 128), &tmK, &bars->k_full, c * 64, kr);
        bulk_load(smem + C::OFF_BIAS + (t & 1) * BN * 4, p.bias2 + kr, BN * 4, &bars->k_full);
        k_issued = t + 1;
        if (!(ok = slot_ready(ge))) break;
        {
          const int r = static_cast<int>(ge % R);
          mbar_arrive_expect_tx(&bars->c_full[r], C::KT_BYTES);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_2d(smem + C::OFF_C + r * C::SLOT + c * (BN * 128), &tmV, &bars->c_full[r], c * 64, kr);
          ++ge;
        }
        const int nb = min(BN, nK - t * BN);
        for (int b = 0; b < nb; ++b) {
          if (!(ok = slot_ready(ge))) break;
          const int r = static_cast<int>(ge % R);
          mbar_arrive_expect_tx(&bars->c_full[r], C::C_BYTES);
          const int crow = (bh * nK + t * BN + b) * D;
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_2d(smem + C::OFF_C + r * C::SLOT + c * (D * 128), &tmC, &bars->c_full[r], c * 64, crow);
          ++ge;
        }
      }
      // drain this thread's copies still in flight before the CTA may exit
      if (k_issued > 0) mbar_wait_bounded(&bars->k_full, (k_issued - 1) & 1, nullptr, kWaitLimitNs);
      for (unsigned e = ge > R ? ge - R : 0u; e < ge; ++e)
        mbar_wait_bounded(&bars->c_full[e % R], (e / R) & 1, nullptr, kWaitLimitNs);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t IDS = idesc_bf16(128, BN, 0);
      constexpr uint32_t IDO = idesc_bf16(128, D, 1);
      bool ok = t1w(&bars->q_full[0], 0, bars, p) && t1w(&bars->q_full[1], 0, bars, p);
      unsigned ge = 0u;  // ring elements consumed (same order as the producer; unsigned: bit-op % R)
      int na[2][2] = {{0, 0}, {0, 0}};
      for (int t = 0; ok && t < nT; ++t) {
        if (!(ok = t1w(&bars->k_full, t & 1, bars, p))) break;
        tc_fence_after();
        for (int i = 0; i < 2; ++i) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_bf16(tmem + i * BN, desc_k_sw128(aQ + i * C::Q_BYTES + (kk >> 2) * (128 * 128) + (kk & 3) * 32),
                      desc_k_sw128(aK + (kk >> 2) * (BN * 128) + (kk & 3) * 32), IDS, kk > 0 ? 1u : 0u);
          umma_commit(&bars->s_full[i]);
        }
        umma_commit(&bars->k_empty);
        const int rv = static_cast<int>(ge % R);
        if (!(ok = t1w(&bars->c_full[rv], (ge / R) & 1, bars, p))) break;
        const uint32_t aV = aC + rv * C::SLOT;
        for (int i = 0; i < 2 && ok; ++i) {
          if (!(ok = t1w(&bars->p_full[i], t & 1, bars, p))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            umma_bf16_tmem_a(tmem + 2 * BN + i * D, tmem + i * BN + kk * 8,
                             desc_mn_sw128(aV + kk * 16 * 128, BN * 128), IDO, (t > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&bars->a_free[i][0]);
        }
        if (!ok) break;
        umma_commit(&bars->c_empty[rv]);
        ++ge;
        const int nb = min(BN, nK - t * BN);
        for (int b = 0; ok && b < nb; ++b, ++ge) {
          const int r = static_cast<int>(ge % R), s = b & 1;
          if (!(ok = t1w(&bars->c_full[r], (ge / R) & 1, bars, p))) break;
          const uint32_t cb = aC + r * C::SLOT;
          for (int i = 0; i < 2; ++i) {
            if (!(ok = t1w(&bars->a_full[i][s], na[i][s] & 1, bars, p))) break;
            ++na[i][s];
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              umma_bf16_tmem_a(tmem + 2 * BN + i * D, tmem + i * BN + s * 64 + kk * 8,
                               desc_mn_sw128(cb + kk * 16 * 128, D * 128), IDO, 1u);
            umma_commit(&bars->a_free[i][s]);
          }
          if (ok) umma_commit(&bars->c_empty[r]);
        }
      }
      if (ok) {
        umma_commit(&bars->o_done[0]);
        umma_commit(&bars->o_done[1]);
      }
      umma_commit(&bars->teardown);
      mbar_wait_bounded(&bars->teardown, 0, nullptr, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------ tile i: weights, A operands, epilogue
    const int i = warp >> 2;
    const int r = tid & 127;
    const int g = row0 + i * 128 + r;
    {
      // gather the tile's query rows into shared memory (K-major, 128B swizzle)
      gather_rows_sw128<D>(p.q, p.row_idx, bh, p.n_rows, p.N, row0 + i * 128, r, aQ + i * C::Q_BYTES, true, p.status);
      fence_proxy_async_smem();
      mbar_arrive(&bars->q_full[i]);
    }
    wg_bar_sync(1 + i);
    // this thread's own query row, bf16 pairs (the A operands scale it)
    uint32_t qr[D / 2];
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint4 v4 = lds128(aQ + i * C::Q_BYTES + (c >> 3) * (128 * 128) + sw128(r, c & 7));
      qr[4 * c] = v4.x;
      qr[4 * c + 1] = v4.y;
      qr[4 * c + 2] = v4.z;
      qr[4 * c + 3] = v4.w;
    }

    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t sS = tmem + lane_base + i * BN;
    const uint32_t sO = tmem + lane_base + 2 * BN + i * D;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    if (p.inject != nullptr && (__ldg(p.inject) & 1)) {  // test hook: behave as if S never arrived
      t1raise(bars, p);
      ok = false;
    }
    uint4 wl[BN / 8];  // w of the current key tile, 8 blocks per entry (indexed by block group)
    int f[2] = {0, 0};  // uses of A slot 0 / 1 so far (P0 counts as a use of slot 0)
    for (int t = 0; ok && t < nT; ++t) {
      if (!(ok = t1warp(&bars->s_full[i], t & 1, bars, p))) break;
      tc_fence_after();
      const float* bias = bias_sm + (t & 1) * BN;
      float mt = -INFINITY;
#pragma unroll
      for (int j = 0; j < BN / 32; ++j) {
        uint32_t u[32];
        tmem_ld32(sS + j * 32, u);
        tmem_wait_ld();
        keep_regs(u);
#pragma unroll
        for (int c = 0; c < 32; ++c) mt = fmaxf(mt, fmaf(__uint_as_float(u[c]), p.scale_log2, bias[j * 32 + c]));
      }
      const float m_new = fmaxf(m, mt);
      const bool need = m_new > m + 32.0f;  // re-base only on a 2^32 growth (see flash2.cu)
      const float alpha = need ? ex2(m - m_new) : 1.f;
      if (need) {
        l *= alpha;
        m = m_new;
      }
      if (t > 0 && __any_sync(0xffffffffu, need)) {
        // every MMA into O issued before S(t) is complete: S(t)'s commit covers them
#pragma unroll 1
        for (int j = 0; j < D / 16; ++j) {
          uint32_t u[16];
          tmem_ld16(sO + j * 16, u);
          tmem_wait_ld();
          keep_regs(u);
#pragma unroll
          for (int c = 0; c < 16; ++c) u[c] = __float_as_uint(__uint_as_float(u[c]) * alpha);
          tmem_st16(sO + j * 16, u);
        }
      }
      const float mref = (m == -INFINITY) ? 0.f : m;
      // slot 0 receives P0: its previous use (the last even A of the
      // previous key tile) is complete, waited on so the phases stay in step
      if (f[0] > 0 && !(ok = t1warp(&bars->a_free[i][0], (f[0] - 1) & 1, bars, p))) break;
      float ls = 0.f;
#pragma unroll
      for (int j = 0; j < BN / 32; ++j) {
        uint32_t u[32];
        tmem_ld32(sS + j * 32, u);
        tmem_wait_ld();
        keep_regs(u);
        uint32_t pw[16], ww[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float b0 = bias[j * 32 + 2 * c], b1 = bias[j * 32 + 2 * c + 1];
          const float x0 = fmaf(__uint_as_float(u[2 * c]), p.scale_log2, -mref);
          const float x1 = fmaf(__uint_as_float(u[2 * c + 1]), p.scale_log2, -mref);
          const float p0 = ex2(x0 + b0), p1 = ex2(x1 + b1);
          const float e0 = b0 == -INFINITY ? 0.f : ex2(x0) * scale;
          const float e1 = b1 == -INFINITY ? 0.f : ex2(x1) * scale;
          ls += p0 + p1;
          pw[c] = pack_bf16(p0, p1);
          ww[c] = pack_bf16(e0, e1);
        }
        // P0 of this quarter into columns [16j, 16j + 16): their scores were
        // read by this quarter or an earlier one
        tmem_st16(sS + j * 16, pw);
#pragma unroll
        for (int k = 0; k < 4; ++k) wl[j * 4 + k] = make_uint4(ww[4 * k], ww[4 * k + 1], ww[4 * k + 2], ww[4 * k + 3]);
      }
      l += ls;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[i]);
      ++f[0];
      const int nb = min(BN, nK - t * BN);
#pragma unroll 1
      for (int gi = 0; ok && gi * 8 < nb; ++gi) {
        const uint4 wv = wl[gi];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int b = gi * 8 + k;
          if (b >= nb) break;
          const int s = k & 1;
          if (f[s] > 0 && !(ok = t1warp(&bars->a_free[i][s], (f[s] - 1) & 1, bars, p))) break;
          tc_fence_after();
          const uint32_t word = (k >> 1) == 0 ? wv.x : (k >> 1) == 1 ? wv.y : (k >> 1) == 2 ? wv.z : wv.w;
          const uint32_t h = s ? (word >> 16) : (word & 0xffffu);
          const uint32_t wpair = h | (h << 16);
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh) {
            uint32_t a[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) a[c] = bf16x2_mul(qr[hh * 32 + c], wpair);
            tmem_st32(sS + s * 64 + hh * 32, a);
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&bars->a_full[i][s]);
          ++f[s];
        }
      }
    }

    const bool valid_row = g < p.n_rows;
    if (ok && nT > 0 && t1warp(&bars->o_done[i], 0, bars, p)) {
      tc_fence_after();
      int dst = valid_row ? (p.row_idx ? __ldg(p.row_idx + static_cast<size_t>(bh) * p.n_rows + g) : g) : 0;
      const bool store = valid_row && static_cast<unsigned>(dst) < static_cast<unsigned>(p.N);
      if (!store) dst = 0;
      uint16_t* orow = p.out + (static_cast<size_t>(bh) * p.N + dst) * D;
      const float inv = 1.f / l;
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        uint32_t u[32];
        tmem_ld32(sO + j * 32, u);
        tmem_wait_ld();
        keep_regs(u);
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

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_cbuild(int D, const CUtensorMap& tmK, const CUtensorMap& tmV, const float* Kbar,
                          const float* Vbar, const int32_t* kept, uint16_t* Cout, int BH, int N_src, int N_ctx,
                          int blk, int n_keep, int* status, cudaStream_t st) {
  const int nSB = (N_src + blk - 1) / blk, nCB = (N_ctx + blk - 1) / blk;
  const int nK = nSB + n_keep;
  if (BH <= 0 || nK <= 0) return cudaSuccess;
  if (blk > 128 || BH > 65535) return cudaErrorInvalidValue;
  const dim3 grid(nK, BH);
  const int N = N_src + N_ctx;
  cudaError_t e;
  if (D == 128) {
    e = cudaFuncSetAttribute(cbuild_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, CBCfg<128>::SMEM);
    if (e != cudaSuccess) return e;
    cbuild_kernel<128><<<grid, 128, CBCfg<128>::SMEM, st>>>(tmK, tmV, Kbar, Vbar, kept, Cout, N, N_src, N_ctx, blk,
                                                            nSB, nSB + nCB, n_keep, nK, status);
  } else if (D == 64) {
    e = cudaFuncSetAttribute(cbuild_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, CBCfg<64>::SMEM);
    if (e != cudaSuccess) return e;
    cbuild_kernel<64><<<grid, 128, CBCfg<64>::SMEM, st>>>(tmK, tmV, Kbar, Vbar, kept, Cout, N, N_src, N_ctx, blk, nSB,
                                                          nSB + nCB, n_keep, nK, status);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_taylor1(int D, const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmC,
                           const FlashParams& p0, int nK, float scale, int BH, cudaStream_t st) {
  if (p0.n_rows <= 0 || BH <= 0) return cudaSuccess;
  FlashParams p = p0;
  p.pairs_per_head = (p.n_rows + 255) / 256;
  const long long items = static_cast<long long>(BH) * p.pairs_per_head;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e;
  if (D == 128) {
    e = cudaFuncSetAttribute(taylor1_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, T1Cfg<128>::SMEM);
    if (e != cudaSuccess) return e;
    taylor1_kernel<128><<<static_cast<unsigned>(items), 320, T1Cfg<128>::SMEM, st>>>(tmK, tmV, tmC, p, nK, scale);
  } else if (D == 64) {
    int smem = T1Cfg<64>::SMEM;
    if (smem < 116 * 1024) smem = 116 * 1024;  // one CTA per SM (all 512 TMEM columns)
    e = cudaFuncSetAttribute(taylor1_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    taylor1_kernel<64><<<static_cast<unsigned>(items), 320, smem, st>>>(tmK, tmV, tmC, p, nK, scale);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace isa
