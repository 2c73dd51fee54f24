// flash2.cu -- two-tile (ping-pong) tcgen05 attention engine.
//
// One CTA owns 256 query rows of one (b, h) as two 128-row tiles.  Each tile
// has its own softmax warpgroup, its own S tile and its own O accumulator in
// tensor memory; the tensor core alternates between the tiles, so one
// tile's softmax overlaps the other tile's QK^T and PV products.  The bf16
// probabilities P are written back into the first BN/2 columns of the
// tile's own S region (tcgen05.st, two bf16 per column) and consumed from
// there as the A operand of the PV UMMA; V is the MN-major B operand in
// 128B-swizzled shared memory.
//
// Modes (method: "Lightning Unified Video Editing via In-Context Sparse
// Attention", abstract):
//   DENSE  all N keys, contiguous queries (the in-house baseline).
//   FULL   ISA full attention for routed queries: gathered Q rows, keys of
//          every source block then of the kept context blocks, one block
//          per key tile, partial blocks masked by their token count.  A row
//          index of -1 is a padding entry (a partial block's missing rows
//          in the block-granular grouping): computed on zeros, never stored.
// (Sharpness + Taylor over every query runs in the persistent kernel of
// fused.cu, built on the same pipeline.)
//
// Work items: 256 query rows of one (b, h); whole waves of items run as
// one launch, the items of a partial last wave are split along the key
// tiles over all SMs and merged by combine_kernel (no idle tail wave).
//
// Warps (320 threads): 0-3 softmax of tile 0, 4-7 softmax of tile 1 (thread
// <-> query row <-> TMEM lane), 8 TMA producer, 9 TMEM allocator + UMMA
// issuer.  TMEM: S/P of tile i at [i*BN, i*BN+BN), O of tile i at
// [2*BN + i*D, 2*BN + i*D + D).
//
// Ordering: the issuer runs the tensor pipe as PV0(t), S0(t+1), PV1(t),
// S1(t+1), so each tile's softmax overlaps two MMAs of the other tile.
// The softmax hands P_i(t) over in parts of 64 keys (one mbarrier each);
// the issuer starts PV_i(t) on the first part while the later ones are
// still being exponentiated, so the tensor pipe waits only for the last.
// S_i(t+1) overwrites the columns PV_i(t) reads as P_i(t); it is issued
// behind PV_i(t) by the same thread and UMMAs from one thread execute in
// order.  The commit that signals S_i(t+1) fires only when every earlier
// UMMA (PV_i(t) included) is complete, so a softmax warpgroup that sees
// S_i(t+1) may rescale O_i and overwrite the S_i columns with P_i(t+1).
// Every mbarrier wait is bounded (status word + CTA abort flag, as in
// flash.cu).
#include <cmath>

#include "gather.cuh"
#include "isa_internal.h"
#include "tc_ptx.cuh"

namespace isa {

template <int D, int BN, int MODE>
struct Attn2Cfg {
  static constexpr int TILE = 128;
  static constexpr bool kTmaQ = MODE != MODE_FULL;  // contiguous query rows
  static constexpr int Q_BYTES = TILE * D * 2;      // one tile
  static constexpr int KT_BYTES = BN * D * 2;       // one key (or value) tile
  static constexpr int NKT = 2;                     // tiles per stage: K, V
  // P hand-off in parts of 64 keys (one barrier each), so PV starts on the
  // first keys while the softmax still exponentiates the rest (32-key parts
  // measured no faster: twice the issuer's waits).
  static constexpr int NP = BN / 64;
  static constexpr int STAGE_BYTES = NKT * KT_BYTES;
  static constexpr int BUDGET = 225 * 1024;
  static constexpr int ST_FIT = (BUDGET - 2 * Q_BYTES - 1024 - 256) / STAGE_BYTES;
  static constexpr int STAGES = ST_FIT >= 3 ? 3 : (ST_FIT >= 2 ? 2 : 1);
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + STAGES * STAGE_BYTES;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;  // + alignment slack
  static constexpr int THREADS = 320;
  static_assert(2 * BN + 2 * D <= 512, "TMEM budget");
  static_assert(ST_FIT >= 1, "shared memory budget");
};

struct Attn2Bars {
  uint64_t q_full[2];
  uint64_t k_full[3];
  uint64_t v_full[3];
  uint64_t k_empty[3];  // K slot free: S_1 of its tile done
  uint64_t v_empty[3];  // V slot free: PV_1 of its tile done
  uint64_t s_full[2];
  uint64_t p_part[2][4];
  uint64_t o_done[2];
  uint64_t teardown;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void raise2(Attn2Bars* bars, const FlashParams& p) {
  *reinterpret_cast<volatile int*>(&bars->abort) = 1;
  if (p.status != nullptr) atomicCAS(p.status, 0, 5 /* ISA_ERR_DEVICE_TIMEOUT */);
}
__device__ __forceinline__ bool w1(uint64_t* bar, uint32_t par, Attn2Bars* bars, const FlashParams& p) {
  const int r = mbar_wait_bounded(bar, par, reinterpret_cast<volatile int*>(&bars->abort), kWaitLimitNs);
  if (r == 2) raise2(bars, p);
  return r == 0;
}
__device__ __forceinline__ bool wwarp(uint64_t* bar, uint32_t par, Attn2Bars* bars, const FlashParams& p) {
  const bool ok = w1(bar, par, bars, p);
  return __all_sync(0xffffffffu, ok);
}
template <int N>
__device__ __forceinline__ void regs_after(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

template <int BN, int MODE>
__device__ __forceinline__ int kv_row(const FlashParams& p, int bh, int t) {
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
__device__ __forceinline__ int kv_count(const FlashParams& p, int bh, int t) {
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
__global__ void __launch_bounds__(320, 1)
    attn2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV,
                 const FlashParams p) {
  using C = Attn2Cfg<D, BN, MODE>;
  constexpr int ST = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  Attn2Bars* bars = reinterpret_cast<Attn2Bars*>(smem + C::OFF_BAR);
  const uint32_t aQ = smem_u32(smem + C::OFF_Q);
  const uint32_t aKV = smem_u32(smem + C::OFF_KV);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool split = p.split_pieces > 0;
  const int item = p.item_base + (split ? static_cast<int>(blockIdx.x) / p.split_pieces : static_cast<int>(blockIdx.x));
  const int piece = split ? static_cast<int>(blockIdx.x) % p.split_pieces : 0;
  const int pieces = split ? p.split_pieces : 1;
  const int bh = item / p.pairs_per_head;
  const int row0 = (item % p.pairs_per_head) * 256;
  // key tiles [kv0, kv0 + nT) of this CTA (all of them unless key-split)
  const int kv0 = piece * p.n_kv_tiles / pieces;
  const int nT = (piece + 1) * p.n_kv_tiles / pieces - kv0;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], C::kTmaQ ? 1 : 128);
      mbar_init(&bars->s_full[i], 1);
      for (int q = 0; q < 4; ++q) mbar_init(&bars->p_part[i][q], 128);
      mbar_init(&bars->o_done[i], 1);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_empty[s], 1);
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
    if constexpr (C::kTmaQ) tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      if constexpr (C::kTmaQ) {
        for (int i = 0; i < 2; ++i) {
          mbar_arrive_expect_tx(&bars->q_full[i], C::Q_BYTES);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_2d(smem + C::OFF_Q + i * C::Q_BYTES + c * (128 * 128), &tmQ, &bars->q_full[i], c * 64,
                        bh * p.N + row0 + i * 128);
        }
      }
      int issued = 0;
      for (int t = 0; t < nT; ++t) {
        const int st = t % ST;
        // K and V slots are released separately: K(t) is last read by
        // S_1(t), V(t) by PV_1(t) two MMAs later, so K(t + ST) loads early
        if (t >= ST && !w1(&bars->k_empty[st], ((t / ST) - 1) & 1, bars, p)) break;
        const int r = kv_row<BN, MODE>(p, bh, kv0 + t);
        uint8_t* base = smem + C::OFF_KV + st * C::STAGE_BYTES;
        mbar_arrive_expect_tx(&bars->k_full[st], C::KT_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) tma_load_2d(base + c * (BN * 128), &tmK, &bars->k_full[st], c * 64, r);
        uint8_t* vb = base + (C::NKT - 1) * C::KT_BYTES;
        if (t >= ST && !w1(&bars->v_empty[st], ((t / ST) - 1) & 1, bars, p)) break;
        mbar_arrive_expect_tx(&bars->v_full[st], C::KT_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) tma_load_2d(vb + c * (BN * 128), &tmV, &bars->v_full[st], c * 64, r);
        issued = t + 1;
      }
      for (int t = issued > ST ? issued - ST : 0; t < issued; ++t) {  // drain own copies
        const int st = t % ST;
        const uint32_t par = (t / ST) & 1;
        mbar_wait_bounded(&bars->k_full[st], par, nullptr, kWaitLimitNs);
        mbar_wait_bounded(&bars->v_full[st], par, nullptr, kWaitLimitNs);
      }
      if constexpr (C::kTmaQ) {
        mbar_wait_bounded(&bars->q_full[0], 0, nullptr, kWaitLimitNs);
        mbar_wait_bounded(&bars->q_full[1], 0, nullptr, kWaitLimitNs);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t IDS = idesc_bf16(128, BN, 0);
      constexpr uint32_t IDO = idesc_bf16(128, D, 1);
      bool ok = w1(&bars->q_full[0], 0, bars, p) && w1(&bars->q_full[1], 0, bars, p);
      tc_fence_after();
      auto issue_S = [&](int i, int t) {
        const int st = t % ST;
        const uint32_t kb = aKV + st * C::STAGE_BYTES;
        const uint32_t qa = aQ + i * C::Q_BYTES;
        const uint32_t dS = tmem + i * BN;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(dS, desc_k_sw128(qa + (kk >> 2) * (128 * 128) + (kk & 3) * 32),
                    desc_k_sw128(kb + (kk >> 2) * (BN * 128) + (kk & 3) * 32), IDS, kk > 0 ? 1u : 0u);
        umma_commit(&bars->s_full[i]);
      };
      // PV_i(t), part by part as the softmax hands P over (false: a wait gave up)
      auto issue_PV = [&](int i, int t) -> bool {
        const int st = t % ST;
        const uint32_t vb = aKV + st * C::STAGE_BYTES + (C::NKT - 1) * C::KT_BYTES;
        constexpr int KS = BN / 16 / C::NP;  // k-steps per part
#pragma unroll
        for (int qp = 0; qp < C::NP; ++qp) {
          if (!w1(&bars->p_part[i][qp], t & 1, bars, p)) return false;
          tc_fence_after();
#pragma unroll
          for (int k2 = 0; k2 < KS; ++k2) {
            const int kk = qp * KS + k2;
            umma_bf16_tmem_a(tmem + 2 * BN + i * D, tmem + i * BN + kk * 8,
                             desc_mn_sw128(vb + kk * 16 * 128, BN * 128), IDO, (t > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&bars->o_done[i]);
        return true;
      };
      if (ok && nT > 0) {
        ok = w1(&bars->k_full[0], 0, bars, p);
        if (ok) {
          tc_fence_after();
          issue_S(0, 0);
          issue_S(1, 0);
          umma_commit(&bars->k_empty[0]);
        }
      }
      for (int t = 0; ok && t < nT; ++t) {
        const int st = t % ST;
        const bool more = t + 1 < nT;
        if (!(ok = w1(&bars->v_full[st], (t / ST) & 1, bars, p))) break;
        if constexpr (ST >= 2) {
          // Tensor-pipe order PV0(t), S0(t+1), PV1(t), S1(t+1): each softmax
          // warpgroup has the other tile's PV and S (two MMAs) to hide behind.
          // S_i(t+1) overwrites the P_i(t) columns that PV_i(t), issued just
          // before it, reads: UMMAs issued by one thread execute in order.
          if (!(ok = issue_PV(0, t))) break;
          if (more) {
            if (!(ok = w1(&bars->k_full[(t + 1) % ST], ((t + 1) / ST) & 1, bars, p))) break;
            tc_fence_after();
            issue_S(0, t + 1);
          }
          if (!(ok = issue_PV(1, t))) break;
          umma_commit(&bars->v_empty[st]);
          if (more) {
            issue_S(1, t + 1);
            umma_commit(&bars->k_empty[(t + 1) % ST]);
          }
        } else {
          // One stage: V(t+1) lands only after PV(t) of both tiles released
          // its slot, so both PVs go first (K(t+1) loads once S_1(t) is done).
          if (!(ok = issue_PV(0, t))) break;
          if (!(ok = issue_PV(1, t))) break;
          umma_commit(&bars->v_empty[st]);
          if (more) {
            if (!(ok = w1(&bars->k_full[0], ((t + 1) / ST) & 1, bars, p))) break;
            tc_fence_after();
            issue_S(0, t + 1);
            issue_S(1, t + 1);
            umma_commit(&bars->k_empty[0]);
          }
        }
      }
      umma_commit(&bars->teardown);
      mbar_wait_bounded(&bars->teardown, 0, nullptr, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------ softmax warpgroup of tile i
    const int i = warp >> 2;
    const int r = tid & 127;
    const int g = row0 + i * 128 + r;  // query row within the launch's row list
    if constexpr (!C::kTmaQ) {
      gather_rows_sw128<D>(p.q, p.row_idx, bh, p.n_rows, p.N, row0 + i * 128, r, aQ + i * C::Q_BYTES, true, p.status);
      fence_proxy_async_smem();
      mbar_arrive(&bars->q_full[i]);
    }

    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t sS = tmem + lane_base + i * BN;
    const uint32_t sO = tmem + lane_base + 2 * BN + i * D;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    if (p.inject != nullptr && (__ldg(p.inject) & 1)) {  // test hook: behave as if S never arrived
      raise2(bars, p);
      ok = false;
    }
    int valid_next = nT > 0 ? kv_count<BN, MODE>(p, bh, kv0) : 0;
    for (int t = 0; ok && t < nT; ++t) {
      const int valid = valid_next;
      if (t + 1 < nT) valid_next = kv_count<BN, MODE>(p, bh, kv0 + t + 1);  // prefetched under the wait below
      if (!(ok = wwarp(&bars->s_full[i], t & 1, bars, p))) break;
      tc_fence_after();
      uint32_t sreg[BN / 32][32];
      float mt = -INFINITY;
      {
        // every S column of the tile in flight at once; max of the raw
        // scores (the scale is positive), columns past `valid` excluded.
        // The scores stay in registers for the exponent pass below.
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) tmem_ld32(sS + j * 32, sreg[j]);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) regs_after(sreg[j]);
        float pm[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) pm[k] = -INFINITY;
        if (valid >= BN) {  // three-input max: 64 instructions for 128 scores
#pragma unroll
          for (int c = 0; c < BN; c += 2)
            pm[(c >> 1) & 7] = fmax3(pm[(c >> 1) & 7], __uint_as_float(sreg[c >> 5][c & 31]),
                                     __uint_as_float(sreg[c >> 5][(c + 1) & 31]));
        } else {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c < valid) pm[c & 7] = fmaxf(pm[c & 7], __uint_as_float(sreg[c >> 5][c & 31]));
        }
        const float raw = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        mt = raw * p.scale_log2;
      }
      const float m_new = fmaxf(m, mt);
      // Rescale only when the running maximum grew by more than 2^32: with
      // the stale reference every p stays <= 2^32 (bf16 and fp32 hold that
      // with the same relative precision; l <= n_keys * 2^32 is far from
      // fp32 overflow) and the result is exact after the final 1/l.  A small
      // threshold would make some warp rescale O on most key tiles when the
      // logits span tens of units (sharp routed queries).
      const bool need = m_new > m + 32.0f;
      // factor for the accumulated O and l when the reference moves
      const float alpha = need ? ex2(m - m_new) : 1.f;
      if (need) {
        l *= alpha;
        m = m_new;
      }
      const float mref = (m == -INFINITY) ? 0.f : m;
      float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float2 ps2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      {
        // quarters of 32 columns; P of quarter q goes to columns [16q, 16q+16)
        // (the scores are already in registers)
        const float nm = -mref;
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(nm, nm);
#pragma unroll
        for (int qq = 0; qq < BN / 32; ++qq) {
          uint32_t w[16];
          if (valid >= BN) {
            // packed fp32x2 FMA (argument) and add (row sum): half the instructions
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float2 a = __ffma2_rn(
                  make_float2(__uint_as_float(sreg[qq][2 * c]), __uint_as_float(sreg[qq][2 * c + 1])), sc2, nm2);
              float2 e;
              if (c % 5 == 4) {  // 3 of 16 pairs on the FMA pipe, the rest on MUFU (measured best of 0-8)
                e = ex2_poly2(a);
              } else {
                e.x = ex2(a.x);
                e.y = ex2(a.y);
              }
              ps2[c & 3] = __fadd2_rn(ps2[c & 3], e);
              w[c] = pack_bf16(e.x, e.y);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int col = qq * 32 + 2 * c;
              const float e0 = col < valid ? ex2(fmaf(__uint_as_float(sreg[qq][2 * c]), p.scale_log2, nm)) : 0.f;
              const float e1 =
                  col + 1 < valid ? ex2(fmaf(__uint_as_float(sreg[qq][2 * c + 1]), p.scale_log2, nm)) : 0.f;
              ps[c & 7] += e0 + e1;
              w[c] = pack_bf16(e0, e1);
            }
          }
          // hand the previous two quarters' P to the issuer: their stores
          // have had this quarter's exponentials to complete
          if (qq > 0 && (qq & 1) == 0) {
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_part[i][qq / 2 - 1]);
          }
          tmem_st16(sS + qq * 16, w);
          if (qq == 0 && t > 0 && __any_sync(0xffffffffu, need)) {
            // O_i rescale (PV_i(t-1) is complete, no part of PV_i(t) issued
            // yet), once the first quarter's scores have left the registers;
            // 16 columns at a time beside the 96 scores still held
#pragma unroll 1
            for (int j = 0; j < D / 16; ++j) {
              uint32_t u[16];
              tmem_ld16(sO + j * 16, u);
              tmem_wait_ld();
              regs_after(u);
#pragma unroll
              for (int c = 0; c < 16; ++c) u[c] = __float_as_uint(__uint_as_float(u[c]) * alpha);
              tmem_st16(sO + j * 16, u);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_part[i][BN / 64 - 1]);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) ps[k] += ps2[k].x + ps2[k].y;
      l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
    }

    const bool valid_row = g < p.n_rows;
    if (ok && nT > 0 && wwarp(&bars->o_done[i], (nT - 1) & 1, bars, p)) {
      tc_fence_after();
      int dst = valid_row ? (p.row_idx ? __ldg(p.row_idx + static_cast<size_t>(bh) * p.n_rows + g) : g) : 0;
      const bool store = valid_row && static_cast<unsigned>(dst) < static_cast<unsigned>(p.N);
      if (!store) dst = 0;
      if (split) {
        // unnormalised partial accumulator of this key range (+ its m, l)
        const size_t prow = static_cast<size_t>(blockIdx.x) * 256 + i * 128 + r;
        p.ml_part[prow] = make_float2(m, l);
        float4* op = reinterpret_cast<float4*>(p.o_part + prow * D);
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
          uint32_t u[32];
          tmem_ld32(sO + j * 32, u);
          tmem_wait_ld();
          regs_after(u);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            op[j * 8 + q4] = make_float4(__uint_as_float(u[4 * q4]), __uint_as_float(u[4 * q4 + 1]),
                                         __uint_as_float(u[4 * q4 + 2]), __uint_as_float(u[4 * q4 + 3]));
        }
      } else {
      uint16_t* orow = p.out + (static_cast<size_t>(bh) * p.N + dst) * D;
      const float inv = 1.f / l;
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        uint32_t u[32];
        tmem_ld32(sO + j * 32, u);
        tmem_wait_ld();
        regs_after(u);
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
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge of key-split partials: row r of split item s is
// sum_p 2^(m_p - M) O_p / sum_p 2^(m_p - M) l_p with M = max_p m_p.
// One warp per query row; grid covers n_items * 256 rows.
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ o_part,
                                                      const float2* __restrict__ ml_part, int pieces, int item_base,
                                                      int n_items, const FlashParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr_all = blockIdx.x * 8 + warp;
  if (rr_all >= n_items * 256) return;
  // A piece that gave up on a bounded wait wrote no partials: leave the rows
  // unwritten rather than merge whatever the buffers held before.
  if (p.status != nullptr && *reinterpret_cast<const volatile int*>(p.status) != 0) return;
  const int s = rr_all / 256, rr = rr_all % 256;
  const int item = item_base + s;
  const int bh = item / p.pairs_per_head;
  const int g = (item % p.pairs_per_head) * 256 + rr;
  if (g >= p.n_rows) return;
  int dst = p.row_idx ? __ldg(p.row_idx + static_cast<size_t>(bh) * p.n_rows + g) : g;
  if (static_cast<unsigned>(dst) >= static_cast<unsigned>(p.N)) {
    if (dst != -1 && lane == 0 && p.status != nullptr) atomicCAS(p.status, 0, 1);  // -1: padding
    return;
  }
  float M = -INFINITY;
  for (int q = 0; q < pieces; ++q) M = fmaxf(M, ml_part[(static_cast<size_t>(s) * pieces + q) * 256 + rr].x);
  constexpr int CPL = D / 32;  // columns per lane
  float acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = 0.f;
  float L = 0.f;
  for (int q = 0; q < pieces; ++q) {
    const size_t prow = (static_cast<size_t>(s) * pieces + q) * 256 + rr;
    const float2 ml = ml_part[prow];
    const float w = ml.x == -INFINITY ? 0.f : ex2(ml.x - M);
    L += w * ml.y;
    const float* op = o_part + prow * D + lane * CPL;
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[c] = fmaf(w, op[c], acc[c]);
  }
  const float inv = 1.f / L;
  uint16_t* orow = p.out + (static_cast<size_t>(bh) * p.N + dst) * D + lane * CPL;
#pragma unroll
  for (int c = 0; c < CPL; c += 2) *reinterpret_cast<uint32_t*>(orow + c) = pack_bf16(acc[c] * inv, acc[c + 1] * inv);
}

template <int D, int BN, int MODE>
static cudaError_t launch2_t(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const FlashParams& p0, int BH, cudaStream_t st) {
  using C = Attn2Cfg<D, BN, MODE>;
  auto kern = attn2_kernel<D, BN, MODE>;
  int smem = C::SMEM;
  if (smem < 116 * 1024) smem = 116 * 1024;                         // one CTA per SM (all 512 TMEM columns)
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e != cudaSuccess) return e;
  FlashParams p = p0;
  p.pairs_per_head = (p.n_rows + 255) / 256;
  p.item_base = 0;
  p.split_pieces = 0;
  const long long items = static_cast<long long>(BH) * p.pairs_per_head;
  // Whole waves as they are; the remainder split along the keys over the SMs
  // (one CTA per SM), then merged, so that no SM idles through a last wave.
  int dev = 0, nsm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const long long whole = nsm > 0 ? items / nsm * nsm : items;
  const int rem = static_cast<int>(items - whole);
  int pieces = 0;
  if (rem > 0 && p.o_part != nullptr && p.split_capacity > 0) {
    pieces = nsm / rem;
    if (pieces > p.n_kv_tiles / 4) pieces = p.n_kv_tiles / 4;
    while (pieces > 1 && pieces * rem > p.split_capacity) --pieces;
    if (pieces < 2) pieces = 0;
  }
  const long long first = pieces ? whole : items;
  if (first > 0) {
    kern<<<static_cast<unsigned>(first), C::THREADS, smem, st>>>(tmQ, tmK, tmV, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (pieces) {
    FlashParams ps = p;
    ps.item_base = static_cast<int>(whole);
    ps.split_pieces = pieces;
    kern<<<static_cast<unsigned>(rem * pieces), C::THREADS, smem, st>>>(tmQ, tmK, tmV, ps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    combine_kernel<D><<<(rem * 256 + 7) / 8, 256, 0, st>>>(p.o_part, p.ml_part, pieces, static_cast<int>(whole), rem,
                                                           p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_attn2(int D, int BN, int mode, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                         const CUtensorMap& tmV, const FlashParams& p, int BH,
                         cudaStream_t st) {
  if (p.n_rows <= 0 || BH <= 0) return cudaSuccess;
#define ISA_ATTN2_CASE(d_, bn_, m_) \
  if (D == d_ && BN == bn_ && mode == m_) return launch2_t<d_, bn_, m_>(tmQ, tmK, tmV, p, BH, st);
  ISA_ATTN2_CASE(128, 128, MODE_DENSE)
  ISA_ATTN2_CASE(128, 128, MODE_FULL)
  ISA_ATTN2_CASE(128, 64, MODE_FULL)
  ISA_ATTN2_CASE(64, 128, MODE_DENSE)
  ISA_ATTN2_CASE(64, 128, MODE_FULL)
  ISA_ATTN2_CASE(64, 64, MODE_FULL)
#undef ISA_ATTN2_CASE
  return cudaErrorInvalidValue;
}

}  // namespace isa
