// fused.cu -- persistent tcgen05 kernel for ISA sharpness + 0-th order
// Taylor attention over every query (stages 2 and 4 in one pass).
//
// Method ("Lightning Unified Video Editing via In-Context Sparse Attention",
// abstract): a query's sharpness is the largest probability of its block
// distribution over the kept blocks, and the queries that are not routed to
// full attention get the 0-th order Taylor output, whose keys and values
// are the block means.  Both come from the same logits
//   l_ib = s * q_i . Kbar_b + log cnt_b   over the kept blocks b:
//   sharp_i = max_b softmax_b(l_i)  and  o_i = softmax_b(l_i) . Vbar.
// The logits use Kbar split as bf16 hi + lo (two UMMAs, fp32-grade) so the
// routing decision matches a float64 evaluation; the log2 cnt key biases
// (-inf on padding) are read per key tile; Vbar is the bf16 V operand.
//
// A work item is 256 query rows of one (b, h) (two 128-row tiles) against
// the head's nK_pad gathered kept blocks (a few 128-key tiles).  With so few
// key tiles per item, a CTA per item spends most of its life loading Q from
// HBM and storing O, one CTA per SM.  Here one CTA per SM loops over items
// (stride = grid size): Q of the next item is loaded into a second buffer
// while the current item computes, and the epilogue of one item overlaps the
// QK^T products of the next: O goes from TMEM through registers into the
// item's own Q buffer (free once its last QK^T is done) and leaves with one
// TMA store per tile, issued by a warp of its own, so the softmax threads
// neither issue stores nor wait for them.  The same warp loads the Q of
// item k + 2 into that buffer as soon as the store has read it out, so the
// K / V producer never waits on an output store.
//
// Warps (352 threads): 0-3 softmax of tile 0, 4-7 tile 1 (thread <-> query
// row <-> TMEM lane), 8 TMA producer, 9 TMEM allocator + the single UMMA
// issuer, 10 Q loads and O stores (TMA) through the two Q buffers.  TMEM: S/P of tile i at [128i, 128i + 128), O of tile i at
// [256 + D*i, 256 + D*i + D).  Tensor pipe order per key tile g (counted
// across the CTA's items): PV0(g), S0(g+1), PV1(g), S1(g+1); S_i(g+1)
// overwrites the P_i(g) columns PV_i(g) reads and is issued after it by the
// same thread (UMMAs from one thread execute in order).  The first PV of an
// item overwrites O, so the issuer waits until the softmax warps have read
// the previous item's O out of TMEM (o_free).
//
// Barrier phases are counted per use across items; every wait is bounded
// (2 s of %globaltimer, then the device status word and a CTA abort flag).
#include <cmath>

#include "isa_internal.h"
#include "tc_ptx.cuh"

namespace isa {

namespace {

template <int D>
struct FusedCfg {
  static constexpr int TILE = 128;
  static constexpr int BN = 128;
  static constexpr int Q_BYTES = TILE * D * 2;   // one 128-row tile
  static constexpr int KT_BYTES = BN * D * 2;    // one key (or value) tile
  static constexpr int OFF_Q = 0;                // [buffer][tile]
  static constexpr int OFF_K = 4 * Q_BYTES;      // K hi, K lo
  // K arrives and is released in 64-column chunks (hi chunks, then lo), the
  // order in which the QK^T UMMAs read it: chunk j of key tile g+1 loads as
  // soon as S_1(g) is done with chunk j, under S_1(g)'s later chunks and
  // PV_0(g), instead of after the whole of S_1(g)
  static constexpr int NKC = 2 * (D / 64);
  static constexpr int KC_BYTES = BN * 128;      // one chunk: BN rows x 64 bf16
  static constexpr int OFF_V = OFF_K + 2 * KT_BYTES;
  static constexpr int OFF_BIAS = OFF_V + KT_BYTES;  // [2][BN] log2 cnt of key tiles g (ring by g & 1)
  static constexpr int OFF_BAR = OFF_BIAS + 2 * BN * 4;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;  // + alignment slack
  static constexpr int THREADS = 352;
  static_assert(2 * BN + 2 * D <= 512, "TMEM budget");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct FusedBars {
  uint64_t q_full[2][2];  // [buffer][tile]
  uint64_t o_staged[2];   // O of tile i written into the staging buffer (128 arrivals)
  uint64_t k_full[4], k_empty[4];  // per K chunk (hi c0, hi c1, lo c0, lo c1)
  uint64_t v_full, v_empty;
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t o_free[2];     // O of tile i read out by its softmax warps
  uint64_t teardown;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(FusedBars) <= 256, "barrier block");

__device__ __forceinline__ void fraise(FusedBars* bars, const FlashParams& p) {
  *reinterpret_cast<volatile int*>(&bars->abort) = 1;
  if (p.status != nullptr) atomicCAS(p.status, 0, 5 /* ISA_ERR_DEVICE_TIMEOUT */);
}
__device__ __forceinline__ bool fw1(uint64_t* bar, uint32_t par, FusedBars* bars, const FlashParams& p) {
  const int r = mbar_wait_bounded(bar, par, reinterpret_cast<volatile int*>(&bars->abort), kWaitLimitNs);
  if (r == 2) fraise(bars, p);
  return r == 0;
}
__device__ __forceinline__ bool fwarp(uint64_t* bar, uint32_t par, FusedBars* bars, const FlashParams& p) {
  const bool ok = fw1(bar, par, bars, p);
  return __all_sync(0xffffffffu, ok);
}
template <int N>
__device__ __forceinline__ void fregs_after(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(352, 1)
    fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKhi,
                 const __grid_constant__ CUtensorMap tmKlo, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmO, const FlashParams p, int n_items, int n_heads) {
  using C = FusedCfg<D>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  FusedBars* bars = reinterpret_cast<FusedBars*>(smem + C::OFF_BAR);
  const uint32_t aQ = smem_u32(smem + C::OFF_Q);
  const uint32_t aK = smem_u32(smem + C::OFF_K);
  const uint32_t aV = smem_u32(smem + C::OFF_V);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = static_cast<int>(gridDim.x);
  const int my_items = n_items > static_cast<int>(blockIdx.x) ? (n_items - 1 - static_cast<int>(blockIdx.x)) / G + 1 : 0;
  const int nT = p.n_kv_tiles;
  const int total = my_items * nT;  // key tiles this CTA walks, over all its items
  // The CTAs' k-th items are consecutive in a head-minor order, so the ~148
  // items in flight at once span every head (a few per head) instead of
  // all being one head's: each head's Kbar / Vbar tiles are then read by a
  // few SMs at a time, not by all of them from the same L2 lines.
  auto item_of = [&](int k) {
    const int lin = static_cast<int>(blockIdx.x) + k * G;
    return (lin % n_heads) * p.pairs_per_head + lin / n_heads;
  };

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->q_full[b][0], 1);
      mbar_init(&bars->q_full[b][1], 1);
    }
    for (int cc = 0; cc < 4; ++cc) {
      mbar_init(&bars->k_full[cc], 1);
      mbar_init(&bars->k_empty[cc], 1);
    }
    mbar_init(&bars->v_full, 1);
    mbar_init(&bars->v_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 128);
      mbar_init(&bars->o_done[i], 1);
      mbar_init(&bars->o_free[i], 128);
      mbar_init(&bars->o_staged[i], 128);
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
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmKhi);
    tma_prefetch_desc(&tmKlo);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      int g_issued = 0;
      int t = 0, row_base = 0;  // key tile of g within its item, first K/V row of the item's head
      for (int g = 0; ok && g < total; ++g, ++t) {
        if (t == nT) t = 0;
        if (t == 0) row_base = item_of(g / nT) / p.pairs_per_head * p.kv_rows_per_head;
        const int r = row_base + t * BN;
#pragma unroll
        for (int cc = 0; cc < C::NKC; ++cc) {
          if (g >= 1 && !(ok = fw1(&bars->k_empty[cc], (g - 1) & 1, bars, p))) break;
          const bool lo = cc >= D / 64;
          const int c = lo ? cc - D / 64 : cc;
          mbar_arrive_expect_tx(&bars->k_full[cc], C::KC_BYTES + (cc == 0 ? BN * 4 : 0));
          // key biases of tile g ride with its first chunk: slot g & 1 (the
          // softmax warps of tile g-2 read it, and both handed their P over
          // before PV_1(g-2), which precedes S_1(g-1) in the tensor pipe)
          if (cc == 0)
            bulk_load(smem + C::OFF_BIAS + (g & 1) * BN * 4, p.bias2 + static_cast<size_t>(r), BN * 4,
                      &bars->k_full[0]);
          tma_load_2d(smem + C::OFF_K + (lo ? C::KT_BYTES : 0) + c * C::KC_BYTES, lo ? &tmKlo : &tmKhi,
                      &bars->k_full[cc], c * 64, r);
        }
        if (!ok) break;
        if (g >= 1 && !(ok = fw1(&bars->v_empty, (g - 1) & 1, bars, p))) break;
        mbar_arrive_expect_tx(&bars->v_full, C::KT_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) tma_load_2d(smem + C::OFF_V + c * (BN * 128), &tmV, &bars->v_full, c * 64, r);
        g_issued = g + 1;
      }
      // drain own copies still in flight
      if (g_issued > 0) {
        for (int cc = 0; cc < C::NKC; ++cc)
          mbar_wait_bounded(&bars->k_full[cc], (g_issued - 1) & 1, nullptr, kWaitLimitNs);
        mbar_wait_bounded(&bars->v_full, (g_issued - 1) & 1, nullptr, kWaitLimitNs);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t IDS = idesc_bf16(128, BN, 0);
      constexpr uint32_t IDO = idesc_bf16(128, D, 1);
      bool ok = true;
      // S_i(g) = Q_i (hi + lo) of key tile g, chunk by chunk of K: S_0 waits
      // for each chunk to land, S_1 (its last reader) releases each one;
      // commits s_full[i] (false: a wait gave up)
      // (the issuing thread paces the tensor pipe: no divisions on its path;
      // the item k and key tile t of g are carried along)
      auto issue_S = [&](int i, int g, int k) -> bool {
        const uint32_t qa = aQ + ((k & 1) * 2 + i) * C::Q_BYTES;
        const uint32_t dS = tmem + i * BN;
#pragma unroll
        for (int cc = 0; cc < C::NKC; ++cc) {
          const int c = cc % (D / 64);
          const uint32_t kb = aK + (cc >= D / 64 ? C::KT_BYTES : 0) + c * C::KC_BYTES;
          if (i == 0) {
            if (!fw1(&bars->k_full[cc], g & 1, bars, p)) return false;
            tc_fence_after();
          }
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            umma_bf16(dS, desc_k_sw128(qa + c * (128 * 128) + k4 * 32), desc_k_sw128(kb + k4 * 32), IDS,
                      (cc > 0 || k4 > 0) ? 1u : 0u);
          if (i == 1) umma_commit(&bars->k_empty[cc]);
        }
        umma_commit(&bars->s_full[i]);
        return true;
      };
      // waits for the Q of item k (before its first key tile)
      auto q_ready = [&](int k) -> bool {
        return fw1(&bars->q_full[k & 1][0], (k >> 1) & 1, bars, p) &&
               fw1(&bars->q_full[k & 1][1], (k >> 1) & 1, bars, p);
      };
      auto issue_PV = [&](int i, int g, int k, int t) -> bool {
        if (t == 0 && k > 0 && !fw1(&bars->o_free[i], (k - 1) & 1, bars, p)) return false;
        if (!fw1(&bars->p_full[i], g & 1, bars, p)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_bf16_tmem_a(tmem + 2 * BN + i * D, tmem + i * BN + kk * 8, desc_mn_sw128(aV + kk * 16 * 128, BN * 128),
                           IDO, (t > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&bars->o_done[i]);
        return true;
      };
      if (total > 0) ok = q_ready(0) && issue_S(0, 0, 0) && issue_S(1, 0, 0);
      int k = 0, t = 0;  // item and key tile of g
      for (int g = 0; ok && g < total; ++g) {
        const bool more = g + 1 < total;
        int k1 = k, t1 = t + 1;  // of g + 1
        if (t1 == nT) {
          t1 = 0;
          ++k1;
        }
        if (!(ok = fw1(&bars->v_full, g & 1, bars, p))) break;
        if (!(ok = issue_PV(0, g, k, t))) break;
        if (more && !(ok = (t1 != 0 || q_ready(k1)) && issue_S(0, g + 1, k1))) break;
        if (!(ok = issue_PV(1, g, k, t))) break;
        umma_commit(&bars->v_empty);
        if (more && !(ok = issue_S(1, g + 1, k1))) break;
        k = k1;
        t = t1;
      }
      umma_commit(&bars->teardown);
      mbar_wait_bounded(&bars->teardown, 0, nullptr, kWaitLimitNs);
    }
  } else if (warp == 10) {
    // ---------------------------------- Q loads and O stores of each item
    if (lane == 0) {
      int q_issued = 0;
      auto load_q = [&](int k) {  // Q of item k into buffer k & 1
        const int b = k & 1;
        const int item = item_of(k);
        const int bh = item / p.pairs_per_head, row0 = (item % p.pairs_per_head) * 256;
        for (int i = 0; i < 2; ++i) {
          mbar_arrive_expect_tx(&bars->q_full[b][i], C::Q_BYTES);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_2d(smem + C::OFF_Q + (b * 2 + i) * C::Q_BYTES + c * (128 * 128), &tmQ, &bars->q_full[b][i],
                        c * 64, bh * p.N + row0 + i * 128);
        }
        q_issued = k + 1;
      };
      for (int k = 0; k < 2 && k < my_items; ++k) load_q(k);
      for (int k = 0; k < my_items; ++k) {
        const int item = item_of(k);
        const int bh = item / p.pairs_per_head, b = k & 1;
        bool ok = true;
        for (int i = 0; i < 2 && ok; ++i) {
          if (!(ok = fw1(&bars->o_staged[i], k & 1, bars, p))) break;
          const int row0 = (item % p.pairs_per_head) * 256 + i * 128;
          uint8_t* stage = smem + C::OFF_Q + (b * 2 + i) * C::Q_BYTES;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) tma_store_3d(&tmO, stage + c * (128 * 128), c * 64, row0, bh);
        }
        bulk_commit_group();
        if (!ok) break;
        if (k + 2 < my_items) {
          bulk_wait_read_all();  // buffer b is free once the stores have read it
          load_q(k + 2);
        }
      }
      bulk_wait_all();  // stores complete before the CTA ends
      for (int k = q_issued > 2 ? q_issued - 2 : 0; k < q_issued; ++k) {  // and own loads (error paths)
        mbar_wait_bounded(&bars->q_full[k & 1][0], (k >> 1) & 1, nullptr, kWaitLimitNs);
        mbar_wait_bounded(&bars->q_full[k & 1][1], (k >> 1) & 1, nullptr, kWaitLimitNs);
      }
    }
  } else {
    // ------------------------------------------ softmax warpgroup of tile i
    const int i = warp >> 2;
    const int r = tid & 127;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t sS = tmem + lane_base + i * BN;
    const uint32_t sO = tmem + lane_base + 2 * BN + i * D;
    bool ok = true;
    if (p.inject != nullptr && (__ldg(p.inject) & 1)) {  // test hook: behave as if S never arrived
      fraise(bars, p);
      ok = false;
    }
    for (int k = 0; ok && k < my_items; ++k) {
      const int item = item_of(k);
      const int bh = item / p.pairs_per_head;
      const int g_row = (item % p.pairs_per_head) * 256 + i * 128 + r;  // query row in the head
      float m = -INFINITY, l = 0.f, mx = -INFINITY;
      for (int t = 0; t < nT; ++t) {
        const int g = k * nT + t;
        if (!(ok = fwarp(&bars->s_full[i], g & 1, bars, p))) break;
        tc_fence_after();
        const float* bias = reinterpret_cast<const float*>(smem + C::OFF_BIAS + (g & 1) * BN * 4);
        // every S column of the tile in flight at once; the raw scores stay
        // in registers for both passes.  Logits in log2 units:
        // x = s*log2(e)*S + log2 cnt (key bias, -inf on padding).
        uint32_t sreg[BN / 32][32];
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) tmem_ld32(sS + j * 32, sreg[j]);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) fregs_after(sreg[j]);
        const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
        float pm[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) pm[c] = -INFINITY;
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) {
          const float4* bp = reinterpret_cast<const float4*>(bias + j * 32);
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 b = bp[c4];
            const float2 x01 = __ffma2_rn(
                make_float2(__uint_as_float(sreg[j][4 * c4]), __uint_as_float(sreg[j][4 * c4 + 1])), sl2,
                make_float2(b.x, b.y));
            const float2 x23 = __ffma2_rn(
                make_float2(__uint_as_float(sreg[j][4 * c4 + 2]), __uint_as_float(sreg[j][4 * c4 + 3])), sl2,
                make_float2(b.z, b.w));
            pm[c4] = fmax3(pm[c4], x01.x, x01.y);
            pm[c4] = fmax3(pm[c4], x23.x, x23.y);
          }
        }
        const float mt = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                               fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        mx = fmaxf(mx, mt);
        const float m_new = fmaxf(m, mt);
        // rescale only when the running maximum grew by more than 2^32 (every
        // p stays <= 2^32; exact after the final 1/l)
        const bool need = m_new > m + 32.0f;
        const float alpha = need ? ex2(m - m_new) : 1.f;
        if (need) {
          l *= alpha;
          m = m_new;
        }
        const float mref = (m == -INFINITY) ? 0.f : m;
        const float2 nm2 = make_float2(-mref, -mref);
        float2 ps2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) {
          // quarter j: P to columns [16j, 16j + 16) (their scores are in registers)
          const float2* bp = reinterpret_cast<const float2*>(bias + j * 32);
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float2 x = __ffma2_rn(
                make_float2(__uint_as_float(sreg[j][2 * c]), __uint_as_float(sreg[j][2 * c + 1])), sl2, bp[c]);
            const float2 a = __fadd2_rn(x, nm2);
            const float e0 = ex2(a.x), e1 = ex2(a.y);
            ps2[c & 3] = __fadd2_rn(ps2[c & 3], make_float2(e0, e1));
            w[c] = pack_bf16(e0, e1);
          }
          tmem_st16(sS + j * 16, w);
        }
        float ps[8];
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) {
          ps[2 * k2] = ps2[k2].x;
          ps[2 * k2 + 1] = ps2[k2].y;
        }
        l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        // O_i rescale (PV_i(g-1) is complete, PV_i(g) not yet issued)
        if (t > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int j = 0; j < D / 32; ++j) {
            uint32_t u[32];
            tmem_ld32(sO + j * 32, u);
            tmem_wait_ld();
            fregs_after(u);
#pragma unroll
            for (int c = 0; c < 32; ++c) u[c] = __float_as_uint(__uint_as_float(u[c]) * alpha);
            tmem_st32(sO + j * 32, u);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[i]);
      }
      if (!ok) break;
      // epilogue of item k: sharpness and Taylor output of this row.  O_i
      // leaves TMEM through registers into Q buffer k & 1 (its last QK^T,
      // S_1 of the item's last key tile, completed before PV_0 of that tile
      // did, hence before o_done) in the TMA box layout; the store warp
      // sends the tile out (rows past N are clipped by the map).
      if (!(ok = fwarp(&bars->o_done[i], (k * nT + nT - 1) & 1, bars, p))) break;
      tc_fence_after();
      const int b = k & 1;
      uint8_t* stage = smem + C::OFF_Q + (b * 2 + i) * C::Q_BYTES;
      const float inv = 1.f / l;
      if (g_row < p.n_rows) p.sharp[static_cast<size_t>(bh) * p.N + g_row] = ex2(mx - m) * inv;  // max_b softmax_b
      // all of O_i in flight at once, one wait; then the next item's first
      // PV may overwrite it
      uint32_t ou[D / 32][32];
#pragma unroll
      for (int j = 0; j < D / 32; ++j) tmem_ld32(sO + j * 32, ou[j]);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < D / 32; ++j) fregs_after(ou[j]);
      tc_fence_before();
      mbar_arrive(&bars->o_free[i]);
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        const uint32_t (&u)[32] = ou[j];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint32_t x = pack_bf16(__uint_as_float(u[8 * q4 + 0]) * inv, __uint_as_float(u[8 * q4 + 1]) * inv);
          const uint32_t y = pack_bf16(__uint_as_float(u[8 * q4 + 2]) * inv, __uint_as_float(u[8 * q4 + 3]) * inv);
          const uint32_t z = pack_bf16(__uint_as_float(u[8 * q4 + 4]) * inv, __uint_as_float(u[8 * q4 + 5]) * inv);
          const uint32_t w = pack_bf16(__uint_as_float(u[8 * q4 + 6]) * inv, __uint_as_float(u[8 * q4 + 7]) * inv);
          // 16-byte chunk (j*4 + q4) of the row: 64-column box j/2, chunk (j%2)*4 + q4 of its 128-byte row
          st_shared_v4(smem_u32(stage) + (j >> 1) * (128 * 128) + sw128(r, (j & 1) * 4 + q4), x, y, z, w);
        }
      }
      fence_proxy_async_smem();  // the generic-proxy writes above, for the TMA store
      mbar_arrive(&bars->o_staged[i]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_fused(int D, const CUtensorMap& tmQ, const CUtensorMap& tmKhi, const CUtensorMap& tmKlo,
                         const CUtensorMap& tmV, const CUtensorMap& tmO, const FlashParams& p0, int BH,
                         cudaStream_t st) {
  if (p0.n_rows <= 0 || BH <= 0 || p0.n_kv_tiles <= 0) return cudaSuccess;
  FlashParams p = p0;
  p.pairs_per_head = (p.n_rows + 255) / 256;
  const long long items = static_cast<long long>(BH) * p.pairs_per_head;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  int dev = 0, nsm = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = static_cast<int>(items < nsm ? items : nsm);
  if (D == 128) {
    using C = FusedCfg<128>;
    if ((e = cudaFuncSetAttribute(fused_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM)) !=
        cudaSuccess)
      return e;
    fused_kernel<128><<<grid, C::THREADS, C::SMEM, st>>>(tmQ, tmKhi, tmKlo, tmV, tmO, p, static_cast<int>(items), BH);
  } else if (D == 64) {
    using C = FusedCfg<64>;
    const int smem = C::SMEM < 116 * 1024 ? 116 * 1024 : C::SMEM;  // one CTA per SM (all 512 TMEM columns)
    if ((e = cudaFuncSetAttribute(fused_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return e;
    fused_kernel<64><<<grid, C::THREADS, smem, st>>>(tmQ, tmKhi, tmKlo, tmV, tmO, p, static_cast<int>(items), BH);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace isa
