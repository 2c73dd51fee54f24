// flash_pair.cu -- the two-tile attention engine of flash2.cu on a pair of
// SMs (a cluster of two CTAs, tcgen05 cta_group::2), for D = 128 and key
// tiles of 128.
//
// Each UMMA has M = 256: the even CTA's single issuing thread drives the
// tensor cores of both SMs.  CTA r of the pair holds its own 256 query rows
// (tiles 0 and 1, 128 rows each) and their S / P / O in its own tensor
// memory, but only half of every key tile: keys [64r, 64r + 64) of K (the
// N half of B in QK^T) and columns [64r, 64r + 64) of V (the N half of B in
// PV).  Against the one-SM engine this halves the UMMA instructions per
// unit of work, the shared-memory operand traffic of B and the L2 -> SM
// bytes of K and V per SM.
//
// Method ("Lightning Unified Video Editing via In-Context Sparse
// Attention", abstract): DENSE (all N keys, the in-house baseline) and FULL
// (ISA full attention for routed queries over every source block and the
// kept context blocks; gathered query rows, -1 rows are padding) exactly as
// in flash2.cu; the softmax arithmetic is the same code.
//
// Synchronisation across the pair (no TMA multicast anywhere: each CTA
// loads its own halves from global memory):
//  - the issuer's barriers live in the even CTA.  Its K / V "full" barriers
//    count its own TMA bytes and one arrival relayed by the odd CTA's warp
//    9, which waits for the odd CTA's own copies and then arrives remotely;
//    the P hand-off and (FULL) Q barriers count the softmax threads of both
//    CTAs, the odd CTA's arriving remotely;
//  - every UMMA completion (S ready, O ready, K / V slot free) is committed
//    to the barrier at the same offset in both CTAs (multicast commit);
//  - an abort (a bounded wait that gave up) is raised in both CTAs;
//  - both CTAs meet at a cluster barrier before the pair frees its tensor
//    memory (cta_group::2, one warp in each CTA) and exits.
//
// Work items: 512 query rows of one (b, h) per pair; whole waves of items
// run as one launch, the items of a partial last wave are split along the
// key tiles over all SM pairs and merged by combine_pair_kernel.
#include <cmath>

#include "isa_internal.h"
#include "tc_ptx.cuh"

namespace isa {

namespace {

template <int MODE>
struct PairCfg {
  static constexpr int D = 128, BN = 128;
  static constexpr bool kTmaQ = MODE != MODE_FULL;
  static constexpr int Q_BYTES = 128 * D * 2;     // one 128-row tile
  static constexpr int KH_BYTES = (BN / 2) * D * 2;  // this CTA's half of a K tile: 64 keys x 128 d
  static constexpr int VH_BYTES = BN * 64 * 2;       // this CTA's half of a V tile: 128 keys x 64 d
  static constexpr int STAGE_BYTES = KH_BYTES + VH_BYTES;
  static constexpr int STAGES = 4;
  static constexpr int NP = BN / 64;              // P hand-off parts
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + STAGES * STAGE_BYTES;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;  // + alignment slack
  static constexpr int THREADS = 320;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(SMEM >= 116 * 1024, "one CTA per SM (each CTA of the pair holds all 512 TMEM columns)");
};

struct PairBars {
  uint64_t q_full[2];
  uint64_t k_full[4], v_full[4];
  uint64_t k_empty[4], v_empty[4];
  uint64_t s_full[2];
  uint64_t p_part[2][2];
  uint64_t o_done[2];
  uint64_t teardown;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(PairBars) <= 512, "barrier block");

__device__ __forceinline__ void praise(PairBars* bars, const FlashParams& p) {
  *reinterpret_cast<volatile int*>(&bars->abort) = 1;
  // and in the other CTA of the pair, so that its waits end too
  st_cluster_u32(mapa_shared(smem_u32(&bars->abort), cluster_ctarank() ^ 1u), 1u);
  if (p.status != nullptr) atomicCAS(p.status, 0, 5 /* ISA_ERR_DEVICE_TIMEOUT */);
}
__device__ __forceinline__ bool pw1(uint64_t* bar, uint32_t par, PairBars* bars, const FlashParams& p) {
  const int r = mbar_wait_bounded(bar, par, reinterpret_cast<volatile int*>(&bars->abort), kWaitLimitNs);
  if (r == 2) praise(bars, p);
  return r == 0;
}
__device__ __forceinline__ bool pwarp(uint64_t* bar, uint32_t par, PairBars* bars, const FlashParams& p) {
  const bool ok = pw1(bar, par, bars, p);
  return __all_sync(0xffffffffu, ok);
}
template <int N>
__device__ __forceinline__ void pregs_after(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}
// Arrive on `bar` of the even CTA: locally there, remotely from the odd CTA.
__device__ __forceinline__ void arrive_leader(uint64_t* bar, uint32_t rank) {
  if (rank == 0) mbar_arrive(bar);
  else mbar_arrive_cluster(mapa_shared(smem_u32(bar), 0u));
}

template <int MODE>
__device__ __forceinline__ int pkv_row(const FlashParams& p, int bh, int t) {
  if constexpr (MODE == MODE_FULL) {
    const int start = (t < p.nSB) ? t * p.blk
                                  : p.N_src + __ldg(p.kept_ctx + static_cast<size_t>(bh) * p.n_keep + (t - p.nSB)) * p.blk;
    return bh * p.N + start;
  } else {
    return bh * p.N + t * 128;
  }
}
template <int MODE>
__device__ __forceinline__ int pkv_count(const FlashParams& p, int bh, int t) {
  if constexpr (MODE == MODE_FULL) {
    if (t < p.nSB) return min(p.blk, p.N_src - t * p.blk);
    const int c = __ldg(p.kept_ctx + static_cast<size_t>(bh) * p.n_keep + (t - p.nSB));
    return min(p.blk, p.N_ctx - c * p.blk);
  } else {
    return min(128, p.N - t * 128);
  }
}

}  // namespace

// tmQ: Q rows, box 64 x 128 (DENSE); tmKh: K rows, box 64 x 64 (a key
// half); tmV: V rows, box 64 x 128 (a column half).
template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKh,
                     const __grid_constant__ CUtensorMap tmV, const FlashParams p) {
  using C = PairCfg<MODE>;
  constexpr int D = C::D, BN = C::BN, ST = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  PairBars* bars = reinterpret_cast<PairBars*>(smem + C::OFF_BAR);
  const uint32_t aQ = smem_u32(smem + C::OFF_Q);
  const uint32_t aKV = smem_u32(smem + C::OFF_KV);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const bool split = p.split_pieces > 0;
  const int item = p.item_base + (split ? pair / p.split_pieces : pair);
  const int piece = split ? pair % p.split_pieces : 0;
  const int pieces = split ? p.split_pieces : 1;
  const int bh = item / p.pairs_per_head;  // items of 512 rows per head
  const int row0 = (item % p.pairs_per_head) * 512 + static_cast<int>(rank) * 256;  // this CTA's 256 rows
  const int kv0 = piece * p.n_kv_tiles / pieces;
  const int nT = (piece + 1) * p.n_kv_tiles / pieces - kv0;

  if (tid == 0) {
    const bool lead = rank == 0;
    for (int i = 0; i < 2; ++i) {
      // the even CTA's Q barrier counts both CTAs: TMA (own bytes + one relayed
      // arrival) or the gathering threads (128 here, 128 remote)
      mbar_init(&bars->q_full[i], C::kTmaQ ? (lead ? 2 : 1) : (lead ? 256 : 128));
      mbar_init(&bars->s_full[i], 1);
      for (int q = 0; q < 2; ++q) mbar_init(&bars->p_part[i][q], lead ? 256 : 128);
      mbar_init(&bars->o_done[i], 1);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bars->k_full[s], lead ? 2 : 1);
      mbar_init(&bars->v_full[s], lead ? 2 : 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->teardown, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc_pair(&bars->tmem_base, 512);
    tmem_relinquish_pair();
  }
  if (warp == 8 && lane == 0) {
    if constexpr (C::kTmaQ) tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmKh);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers (remote arrivals, commits) and TMEM in place
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 8) {
    // --------------------------------------------- TMA producer (own halves)
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
        if (t >= ST && !pw1(&bars->k_empty[st], ((t / ST) - 1) & 1, bars, p)) break;
        const int r = pkv_row<MODE>(p, bh, kv0 + t);
        uint8_t* kb = smem + C::OFF_KV + st * C::STAGE_BYTES;
        mbar_arrive_expect_tx(&bars->k_full[st], C::KH_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_2d(kb + c * (64 * 128), &tmKh, &bars->k_full[st], c * 64, r + 64 * static_cast<int>(rank));
        if (t >= ST && !pw1(&bars->v_empty[st], ((t / ST) - 1) & 1, bars, p)) break;
        mbar_arrive_expect_tx(&bars->v_full[st], C::VH_BYTES);
        tma_load_2d(kb + C::KH_BYTES, &tmV, &bars->v_full[st], 64 * static_cast<int>(rank), r);
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
  } else if (warp == 9 && rank != 0) {
    // ------------------------------------- relay of the odd CTA's copies
    // Its TMA copies complete on its own barriers; the issuer in the even
    // CTA learns of them through one remote arrival each.
    if (lane == 0) {
      bool ok = true;
      if constexpr (C::kTmaQ) {
        for (int i = 0; ok && i < 2; ++i) {
          if ((ok = pw1(&bars->q_full[i], 0, bars, p))) mbar_arrive_cluster(mapa_shared(smem_u32(&bars->q_full[i]), 0u));
        }
      }
      for (int t = 0; ok && t < nT; ++t) {
        const int st = t % ST;
        const uint32_t par = (t / ST) & 1;
        if (!(ok = pw1(&bars->k_full[st], par, bars, p))) break;
        mbar_arrive_cluster(mapa_shared(smem_u32(&bars->k_full[st]), 0u));
        if (!(ok = pw1(&bars->v_full[st], par, bars, p))) break;
        mbar_arrive_cluster(mapa_shared(smem_u32(&bars->v_full[st]), 0u));
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------- UMMA issuer (even CTA)
    if (lane == 0) {
      constexpr uint32_t IDS = idesc_bf16(256, BN, 0);
      constexpr uint32_t IDO = idesc_bf16(256, D, 1);
      bool ok = pw1(&bars->q_full[0], 0, bars, p) && pw1(&bars->q_full[1], 0, bars, p);
      tc_fence_after();
      auto issue_S = [&](int i, int t) {
        const int st = t % ST;
        const uint32_t kb = aKV + st * C::STAGE_BYTES;
        const uint32_t qa = aQ + i * C::Q_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_pair_bf16(tmem + i * BN, desc_k_sw128(qa + (kk >> 2) * (128 * 128) + (kk & 3) * 32),
                         desc_k_sw128(kb + (kk >> 2) * (64 * 128) + (kk & 3) * 32), IDS, kk > 0 ? 1u : 0u);
        umma_commit_pair(&bars->s_full[i], 3);
      };
      auto issue_PV = [&](int i, int t) -> bool {
        const int st = t % ST;
        const uint32_t vb = aKV + st * C::STAGE_BYTES + C::KH_BYTES;
        constexpr int KS = BN / 16 / C::NP;
#pragma unroll
        for (int qp = 0; qp < C::NP; ++qp) {
          if (!pw1(&bars->p_part[i][qp], t & 1, bars, p)) return false;
          tc_fence_after();
#pragma unroll
          for (int k2 = 0; k2 < KS; ++k2) {
            const int kk = qp * KS + k2;
            umma_pair_bf16_tmem_a(tmem + 2 * BN + i * D, tmem + i * BN + kk * 8,
                                  desc_mn_sw128(vb + kk * 16 * 128, 128 * 128), IDO, (t > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit_pair(&bars->o_done[i], 3);
        return true;
      };
      if (ok && nT > 0) {
        ok = pw1(&bars->k_full[0], 0, bars, p);
        if (ok) {
          tc_fence_after();
          issue_S(0, 0);
          issue_S(1, 0);
          umma_commit_pair(&bars->k_empty[0], 3);
        }
      }
      for (int t = 0; ok && t < nT; ++t) {
        const int st = t % ST;
        const bool more = t + 1 < nT;
        if (!(ok = pw1(&bars->v_full[st], (t / ST) & 1, bars, p))) break;
        // tensor-pipe order PV0(t), S0(t+1), PV1(t), S1(t+1), as in flash2.cu
        if (!(ok = issue_PV(0, t))) break;
        if (more) {
          if (!(ok = pw1(&bars->k_full[(t + 1) % ST], ((t + 1) / ST) & 1, bars, p))) break;
          tc_fence_after();
          issue_S(0, t + 1);
        }
        if (!(ok = issue_PV(1, t))) break;
        umma_commit_pair(&bars->v_empty[st], 3);
        if (more) {
          issue_S(1, t + 1);
          umma_commit_pair(&bars->k_empty[(t + 1) % ST], 3);
        }
      }
      umma_commit_pair(&bars->teardown, 1);
      mbar_wait_bounded(&bars->teardown, 0, nullptr, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------ softmax warpgroup of tile i
    const int i = warp >> 2;
    const int r = tid & 127;
    const int g = row0 + i * 128 + r;  // query row within the launch's row list
    if constexpr (!C::kTmaQ) {
      constexpr int CPR = D / 8;
      uint4 vals[CPR];
#pragma unroll
      for (int it = 0; it < CPR; ++it) {
        const int c = it * 128 + r;
        const int row = c / CPR, ch = c % CPR;
        const int gg = row0 + i * 128 + row;
        vals[it] = make_uint4(0u, 0u, 0u, 0u);
        if (gg < p.n_rows) {
          const int src = p.row_idx ? __ldg(p.row_idx + static_cast<size_t>(bh) * p.n_rows + gg) : gg;
          if (static_cast<unsigned>(src) < static_cast<unsigned>(p.N))
            vals[it] = __ldg(reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(bh) * p.N + src) * D + ch * 8));
          else if (src != -1 && p.status != nullptr)  // -1: a padding entry, skipped silently
            atomicCAS(p.status, 0, 1 /* ISA_ERR_INVALID_ARG: index out of range, row skipped */);
        }
      }
#pragma unroll
      for (int it = 0; it < CPR; ++it) {
        const int c = it * 128 + r;
        const int row = c / CPR, ch = c % CPR;
        st_shared_v4(aQ + i * C::Q_BYTES + (ch >> 3) * (128 * 128) + sw128(row, ch & 7), vals[it].x, vals[it].y,
                     vals[it].z, vals[it].w);
      }
      fence_proxy_async_smem();
      arrive_leader(&bars->q_full[i], rank);
    }

    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t sS = tmem + lane_base + i * BN;
    const uint32_t sO = tmem + lane_base + 2 * BN + i * D;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    if (p.inject != nullptr && (__ldg(p.inject) & 1)) {  // test hook: behave as if S never arrived
      praise(bars, p);
      ok = false;
    }
    int valid_next = nT > 0 ? pkv_count<MODE>(p, bh, kv0) : 0;
    for (int t = 0; ok && t < nT; ++t) {
      const int valid = valid_next;
      if (t + 1 < nT) valid_next = pkv_count<MODE>(p, bh, kv0 + t + 1);
      if (!(ok = pwarp(&bars->s_full[i], t & 1, bars, p))) break;
      tc_fence_after();
      uint32_t sreg[BN / 32][32];
      float mt = -INFINITY;
      {
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) tmem_ld32(sS + j * 32, sreg[j]);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) pregs_after(sreg[j]);
        float pm[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) pm[k] = -INFINITY;
        if (valid >= BN) {
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
      // rescale only when the running maximum grew by more than 2^32 (every
      // p stays <= 2^32; exact after the final 1/l)
      const bool need = m_new > m + 32.0f;
      const float alpha = need ? ex2(m - m_new) : 1.f;
      if (need) {
        l *= alpha;
        m = m_new;
      }
      const float mref = (m == -INFINITY) ? 0.f : m;
      float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float2 ps2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      {
        const float nm = -mref;
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(nm, nm);
#pragma unroll
        for (int qq = 0; qq < BN / 32; ++qq) {
          uint32_t w[16];
          if (valid >= BN) {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float2 a = __ffma2_rn(
                  make_float2(__uint_as_float(sreg[qq][2 * c]), __uint_as_float(sreg[qq][2 * c + 1])), sc2, nm2);
              float2 e;
              if (c % 5 == 4) {  // 3 of 16 pairs on the FMA pipe, the rest on MUFU
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
          if (qq > 0 && (qq & 1) == 0) {
            tmem_wait_st();
            tc_fence_before();
            arrive_leader(&bars->p_part[i][qq / 2 - 1], rank);
          }
          tmem_st16(sS + qq * 16, w);
          if (qq == 0 && t > 0 && __any_sync(0xffffffffu, need)) {
            // O_i rescale (PV_i(t-1) is complete, no part of PV_i(t) issued yet)
#pragma unroll 1
            for (int j = 0; j < D / 16; ++j) {
              uint32_t u[16];
              tmem_ld16(sO + j * 16, u);
              tmem_wait_ld();
              pregs_after(u);
#pragma unroll
              for (int c = 0; c < 16; ++c) u[c] = __float_as_uint(__uint_as_float(u[c]) * alpha);
              tmem_st16(sO + j * 16, u);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        arrive_leader(&bars->p_part[i][BN / 64 - 1], rank);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) ps[k] += ps2[k].x + ps2[k].y;
      l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
    }

    const bool valid_row = g < p.n_rows;
    if (ok && nT > 0 && pwarp(&bars->o_done[i], (nT - 1) & 1, bars, p)) {
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
          pregs_after(u);
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
          pregs_after(u);
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
  cluster_sync_all();  // the pair's UMMAs and remote arrivals are done in both CTAs
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Merge of key-split partials of the pair engine: row rr of split item s
// (512 rows: CTA rank rr / 256, row rr % 256 of that CTA) over its pieces;
// the pieces' partial rows are at ((s * pieces + q) * 2 + rank) * 256 + row.
// One warp per query row.  After a device error the rows are left
// unwritten (a piece that gave up wrote no partials).
template <int D>
__global__ void __launch_bounds__(256) combine_pair_kernel(const float* __restrict__ o_part,
                                                           const float2* __restrict__ ml_part, int pieces,
                                                           int item_base, int n_items, const FlashParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr_all = blockIdx.x * 8 + warp;
  if (rr_all >= n_items * 512) return;
  if (p.status != nullptr && *reinterpret_cast<const volatile int*>(p.status) != 0) return;
  const int s = rr_all / 512, rr = rr_all % 512;
  const int rk = rr / 256, within = rr % 256;
  const int item = item_base + s;
  const int bh = item / p.pairs_per_head;
  const int g = (item % p.pairs_per_head) * 512 + rr;
  if (g >= p.n_rows) return;
  int dst = p.row_idx ? __ldg(p.row_idx + static_cast<size_t>(bh) * p.n_rows + g) : g;
  if (static_cast<unsigned>(dst) >= static_cast<unsigned>(p.N)) {
    if (dst != -1 && lane == 0 && p.status != nullptr) atomicCAS(p.status, 0, 1);  // -1: padding
    return;
  }
  auto prow_of = [&](int q) { return ((static_cast<size_t>(s) * pieces + q) * 2 + rk) * 256 + within; };
  float M = -INFINITY;
  for (int q = 0; q < pieces; ++q) M = fmaxf(M, ml_part[prow_of(q)].x);
  constexpr int CPL = D / 32;
  float acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = 0.f;
  float L = 0.f;
  for (int q = 0; q < pieces; ++q) {
    const size_t prow = prow_of(q);
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

template <int MODE>
static cudaError_t launch_pair_t(const CUtensorMap& tmQ, const CUtensorMap& tmKh, const CUtensorMap& tmV,
                                 const FlashParams& p0, int BH, cudaStream_t st) {
  using C = PairCfg<MODE>;
  auto kern = attn_pair_kernel<MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  FlashParams p = p0;
  p.pairs_per_head = (p.n_rows + 511) / 512;  // 512-row pair items per head
  p.item_base = 0;
  p.split_pieces = 0;
  const long long items = static_cast<long long>(BH) * p.pairs_per_head;
  if (items * 2 > 0x7fffffffLL) return cudaErrorInvalidValue;
  int dev = 0, nsm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int npairs = nsm / 2;
  const long long whole = npairs > 0 ? items / npairs * npairs : items;
  const int rem = static_cast<int>(items - whole);
  int pieces = 0;
  // the partial buffers hold split_capacity CTAs of 256 rows: pieces * rem pairs = 2 * pieces * rem CTAs
  if (rem > 0 && p.o_part != nullptr && p.split_capacity > 0) {
    pieces = npairs / rem;
    if (pieces > p.n_kv_tiles / 4) pieces = p.n_kv_tiles / 4;
    while (pieces > 1 && 2 * pieces * rem > p.split_capacity) --pieces;
    if (pieces < 2) pieces = 0;
  }
  const long long first = pieces ? whole : items;
  if (first > 0) {
    kern<<<static_cast<unsigned>(2 * first), C::THREADS, C::SMEM, st>>>(tmQ, tmKh, tmV, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (pieces) {
    FlashParams ps = p;
    ps.item_base = static_cast<int>(whole);
    ps.split_pieces = pieces;
    kern<<<static_cast<unsigned>(2 * rem * pieces), C::THREADS, C::SMEM, st>>>(tmQ, tmKh, tmV, ps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    combine_pair_kernel<128><<<(rem * 512 + 7) / 8, 256, 0, st>>>(p.o_part, p.ml_part, pieces,
                                                                  static_cast<int>(whole), rem, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

bool attn_pair_supported(int D, int BN) { return D == 128 && BN == 128; }

cudaError_t launch_attn_pair(int mode, const CUtensorMap& tmQ, const CUtensorMap& tmKh, const CUtensorMap& tmV,
                             const FlashParams& p, int BH, cudaStream_t st) {
  if (p.n_rows <= 0 || BH <= 0) return cudaSuccess;
  if (mode == MODE_DENSE) return launch_pair_t<MODE_DENSE>(tmQ, tmKh, tmV, p, BH, st);
  if (mode == MODE_FULL) return launch_pair_t<MODE_FULL>(tmQ, tmKh, tmV, p, BH, st);
  return cudaErrorInvalidValue;
}

}  // namespace isa
