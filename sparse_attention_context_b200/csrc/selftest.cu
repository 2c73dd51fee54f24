// selftest.cu -- a one-tile check of the UMMA building blocks used by the
// attention engine: S = A B^T with both operands K-major (A written by
// threads into the 128B-swizzled layout, B loaded by TMA) and O = P V with
// V MN-major (loaded by TMA), both accumulated in TMEM and read back with
// tcgen05.ld; and O2 = P V with P written by threads into TMEM (tcgen05.st,
// two bf16 per column) and read by the UMMA as its A operand.  Also the
// exponentials of the softmax: the FMA-pipe 2^x (ex2_poly2) and the MUFU
// ex2 on given arguments, beside CUDA's exp2f.  Exported for the tests
// only (include/isa_selftest.h).
#include "isa.h"
#include "isa_internal.h"
#include "isa_selftest.h"
#include "tc_ptx.cuh"

namespace isa {

template <int D, int BN>
__global__ void __launch_bounds__(128, 1)
    umma_probe_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmV,
                      const uint16_t* A, const uint16_t* P, float* S_out, float* O_out, float* O2_out,
                      int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  constexpr int A_BYTES = 128 * D * 2, B_BYTES = BN * D * 2, P_BYTES = 128 * BN * 2;
  uint8_t* sA = smem;
  uint8_t* sB = sA + A_BYTES;
  uint8_t* sV = sB + B_BYTES;
  uint8_t* sP = sV + B_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + P_BYTES);  // [0] tma, [1] mma, [2] mma with A in TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  // columns: S [0, BN), O [BN, BN+D), P [BN+D, BN+D+BN/2), O2 [.., +D)
  constexpr int TMEM_COLS = 512;
  constexpr int PCOL = BN + D, O2COL = BN + D + BN / 2;
  const int tid = threadIdx.x, warp = tid >> 5;

  // A (128 x D) and P (128 x BN), K-major, written by threads.
  for (int c = tid; c < 128 * (D / 8); c += 128) {
    const int row = c / (D / 8), ch = c % (D / 8);
    const uint4 val = *reinterpret_cast<const uint4*>(A + row * D + ch * 8);
    st_shared_v4(smem_u32(sA) + (ch >> 3) * (128 * 128) + sw128(row, ch & 7), val.x, val.y, val.z, val.w);
  }
  for (int c = tid; c < 128 * (BN / 8); c += 128) {
    const int row = c / (BN / 8), ch = c % (BN / 8);
    const uint4 val = *reinterpret_cast<const uint4*>(P + row * BN + ch * 8);
    st_shared_v4(smem_u32(sP) + (ch >> 3) * (128 * 128) + sw128(row, ch & 7), val.x, val.y, val.z, val.w);
  }
  fence_proxy_async_smem();
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[0], 2 * B_BYTES);
    for (int c = 0; c < D / 64; ++c) tma_load_2d(sB + c * (BN * 128), &tmB, &bars[0], c * 64, 0);
    for (int c = 0; c < D / 64; ++c) tma_load_2d(sV + c * (BN * 128), &tmV, &bars[0], c * 64, 0);
    ok = mbar_wait_bounded(&bars[0], 0, nullptr, kWaitLimitNs) == 0;
    if (ok) {
      tc_fence_after();
      for (int kk = 0; kk < D / 16; ++kk)
        umma_bf16(tmem, desc_k_sw128(smem_u32(sA) + (kk >> 2) * (128 * 128) + (kk & 3) * 32),
                  desc_k_sw128(smem_u32(sB) + (kk >> 2) * (BN * 128) + (kk & 3) * 32), idesc_bf16(128, BN, 0),
                  kk > 0);
      for (int kk = 0; kk < BN / 16; ++kk)
        umma_bf16(tmem + BN, desc_k_sw128(smem_u32(sP) + (kk >> 2) * (128 * 128) + (kk & 3) * 32),
                  desc_mn_sw128(smem_u32(sV) + kk * 16 * 128, BN * 128), idesc_bf16(128, D, 1), kk > 0);
    }
    umma_commit(&bars[1]);
    if (!ok) atomicCAS(status, 0, ISA_ERR_DEVICE_TIMEOUT);
  }
  __syncwarp();
  const bool done = mbar_wait_bounded(&bars[1], 0, nullptr, kWaitLimitNs) == 0;
  ok = __all_sync(0xffffffffu, done);
  tc_fence_after();
  const int row = tid;
  const uint32_t lb = static_cast<uint32_t>(warp * 32) << 16;
  if (ok) {
    for (int j = 0; j < BN / 32; ++j) {
      uint32_t u[32];
      tmem_ld32(tmem + lb + j * 32, u);
      tmem_wait_ld();
      for (int i = 0; i < 32; ++i) S_out[row * BN + j * 32 + i] = __uint_as_float(u[i]);
    }
    for (int j = 0; j < D / 32; ++j) {
      uint32_t u[32];
      tmem_ld32(tmem + lb + BN + j * 32, u);
      tmem_wait_ld();
      for (int i = 0; i < 32; ++i) O_out[row * D + j * 32 + i] = __uint_as_float(u[i]);
    }
  } else if (tid == 0) {
    atomicCAS(status, 0, ISA_ERR_DEVICE_TIMEOUT);
  }
  // P into TMEM: lane = row, column c holds P[row][2c] (low half), P[row][2c+1].
  if (ok) {
#pragma unroll
    for (int j = 0; j < BN / 64; ++j) {
      uint32_t u[32];
#pragma unroll
      for (int i = 0; i < 32; ++i)
        u[i] = static_cast<uint32_t>(P[row * BN + j * 64 + 2 * i]) |
               (static_cast<uint32_t>(P[row * BN + j * 64 + 2 * i + 1]) << 16);
      tmem_st32(tmem + lb + PCOL + j * 32, u);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) {
    if (ok)
      for (int kk = 0; kk < BN / 16; ++kk)
        umma_bf16_tmem_a(tmem + O2COL, tmem + PCOL + kk * 8, desc_mn_sw128(smem_u32(sV) + kk * 16 * 128, BN * 128),
                         idesc_bf16(128, D, 1), kk > 0);
    umma_commit(&bars[2]);
  }
  __syncwarp();
  const bool done2 = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[2], 0, nullptr, kWaitLimitNs) == 0);
  tc_fence_after();
  if (ok && done2) {
    for (int j = 0; j < D / 32; ++j) {
      uint32_t u[32];
      tmem_ld32(tmem + lb + O2COL + j * 32, u);
      tmem_wait_ld();
      for (int i = 0; i < 32; ++i) O2_out[row * D + j * 32 + i] = __uint_as_float(u[i]);
    }
  } else if (tid == 0) {
    atomicCAS(status, 0, ISA_ERR_DEVICE_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int D, int BN>
static int run_probe(const uint16_t* A, const uint16_t* B, const uint16_t* P, const uint16_t* V, float* S, float* O,
                     float* O2, int* status, cudaStream_t st) {
  CUtensorMap tmB, tmV;
  if (!make_tmap_bf16(&tmB, B, BN, D, BN) || !make_tmap_bf16(&tmV, V, BN, D, BN)) return ISA_ERR_CUDA;
  const int smem = 128 * D * 2 + 2 * BN * D * 2 + 128 * BN * 2 + 64 + 1024 + 4096;
  auto kern = umma_probe_kernel<D, BN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return ISA_ERR_CUDA;
  kern<<<1, 128, smem, st>>>(tmB, tmV, A, P, S, O, O2, status);
  return cudaGetLastError() == cudaSuccess ? ISA_OK : ISA_ERR_CUDA;
}

// One M = 256 tile on a CTA pair (cluster of 2): S = A B^T with A rows
// [128r, 128r + 128) and B rows (keys) [64r, 64r + 64) in CTA r's shared
// memory, then O = P V with P rows [128r, 128r + 128) in CTA r's tensor
// memory and V columns [64r, 64r + 64) in its shared memory.  The even CTA
// issues both products; each CTA reads its own rows of S and O back.
// D = 128, N = 128 keys.  Operands are written into shared memory by the
// threads (no TMA), so the probe depends on nothing but the pair UMMA.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1)
    umma_pair_probe_kernel(const uint16_t* A, const uint16_t* B, const uint16_t* P, const uint16_t* V, float* S_out,
                           float* O_out, int* status) {
  constexpr int D = 128, BN = 128;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint8_t* sA = smem;                       // 128 rows x 128 d, K-major: 2 chunks of 16 KB
  uint8_t* sB = sA + 128 * D * 2;           // 64 keys x 128 d, K-major: 2 chunks of 8 KB
  uint8_t* sV = sB + 64 * D * 2;            // 128 keys x 64 d, MN-major: 16 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + 128 * 64 * 2);  // [0] S done, [1] O done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  constexpr int PCOL = 256, OCOL = 128;     // S at [0, 128), O at [128, 256), P at [256, 320)
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();

  for (int c = tid; c < 128 * (D / 8); c += 128) {
    const int row = c / (D / 8), ch = c % (D / 8);
    const uint4 val = *reinterpret_cast<const uint4*>(A + (128 * rank + row) * D + ch * 8);
    st_shared_v4(smem_u32(sA) + (ch >> 3) * (128 * 128) + sw128(row, ch & 7), val.x, val.y, val.z, val.w);
  }
  for (int c = tid; c < 64 * (D / 8); c += 128) {
    const int row = c / (D / 8), ch = c % (D / 8);
    const uint4 val = *reinterpret_cast<const uint4*>(B + (64 * rank + row) * D + ch * 8);
    st_shared_v4(smem_u32(sB) + (ch >> 3) * (64 * 128) + sw128(row, ch & 7), val.x, val.y, val.z, val.w);
  }
  for (int c = tid; c < BN * 8; c += 128) {
    const int key = c / 8, ch = c % 8;
    const uint4 val = *reinterpret_cast<const uint4*>(V + key * D + 64 * rank + ch * 8);
    st_shared_v4(smem_u32(sV) + sw128(key, ch), val.x, val.y, val.z, val.w);
  }
  fence_proxy_async_smem();
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int row = tid;
  const uint32_t lb = static_cast<uint32_t>(warp * 32) << 16;
  // P rows of this CTA into TMEM: column c holds P[row][2c] (low half), P[row][2c+1]
#pragma unroll
  for (int j = 0; j < BN / 64; ++j) {
    uint32_t u[32];
#pragma unroll
    for (int i = 0; i < 32; ++i)
      u[i] = static_cast<uint32_t>(P[(128 * rank + row) * BN + j * 64 + 2 * i]) |
             (static_cast<uint32_t>(P[(128 * rank + row) * BN + j * 64 + 2 * i + 1]) << 16);
    tmem_st32(tmem + lb + PCOL + j * 32, u);
  }
  tmem_wait_st();
  tc_fence_before();
  cluster_sync_all();  // both CTAs' operands, barriers and TMEM in place
  tc_fence_after();
  if (rank == 0 && tid == 0) {
    constexpr uint32_t IDS = idesc_bf16(256, BN, 0);
    constexpr uint32_t IDO = idesc_bf16(256, D, 1);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      umma_pair_bf16(tmem, desc_k_sw128(smem_u32(sA) + (kk >> 2) * (128 * 128) + (kk & 3) * 32),
                     desc_k_sw128(smem_u32(sB) + (kk >> 2) * (64 * 128) + (kk & 3) * 32), IDS, kk > 0 ? 1u : 0u);
    umma_commit_pair(&bars[0], 3);
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk)
      umma_pair_bf16_tmem_a(tmem + OCOL, tmem + PCOL + kk * 8, desc_mn_sw128(smem_u32(sV) + kk * 16 * 128, 128 * 128),
                            IDO, kk > 0 ? 1u : 0u);
    umma_commit_pair(&bars[1], 3);
  }
  __syncwarp();
  bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[0], 0, nullptr, kWaitLimitNs) == 0);
  ok = __all_sync(0xffffffffu, ok && mbar_wait_bounded(&bars[1], 0, nullptr, kWaitLimitNs) == 0);
  tc_fence_after();
  if (ok) {
    for (int j = 0; j < BN / 32; ++j) {
      uint32_t u[32];
      tmem_ld32(tmem + lb + j * 32, u);
      tmem_wait_ld();
      for (int i = 0; i < 32; ++i) S_out[(128 * rank + row) * BN + j * 32 + i] = __uint_as_float(u[i]);
    }
    for (int j = 0; j < D / 32; ++j) {
      uint32_t u[32];
      tmem_ld32(tmem + lb + OCOL + j * 32, u);
      tmem_wait_ld();
      for (int i = 0; i < 32; ++i) O_out[(128 * rank + row) * D + j * 32 + i] = __uint_as_float(u[i]);
    }
  } else if (tid == 0) {
    atomicCAS(status, 0, ISA_ERR_DEVICE_TIMEOUT);
  }
  tc_fence_before();
  cluster_sync_all();  // neither CTA frees TMEM or exits while the pair's UMMAs or reads run
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// y_poly = ex2_poly2(x) (two arguments per call, as the softmax uses it),
// y_mufu = ex2.approx.ftz (the MUFU path), y_ref = exp2f; one thread per pair.
__global__ void __launch_bounds__(256) ex2_probe_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                                        float* __restrict__ y_mufu, float* __restrict__ y_ref,
                                                        int n) {
  const int i = 2 * (blockIdx.x * 256 + threadIdx.x);
  if (i >= n) return;
  const bool two = i + 1 < n;
  const float2 a = make_float2(x[i], two ? x[i + 1] : 0.f);
  const float2 e = ex2_poly2(a);
  y_poly[i] = e.x;
  y_mufu[i] = ex2(a.x);
  y_ref[i] = exp2f(a.x);
  if (two) {
    y_poly[i + 1] = e.y;
    y_mufu[i + 1] = ex2(a.y);
    y_ref[i + 1] = exp2f(a.y);
  }
}

}  // namespace isa

extern "C" int isa_selftest_ex2(const float* x, float* y_poly, float* y_mufu, float* y_ref, int n, void* stream) {
  if (n < 0) return ISA_ERR_INVALID_ARG;
  if (n == 0) return ISA_OK;
  if (!x || !y_poly || !y_mufu || !y_ref) return ISA_ERR_INVALID_ARG;
  const int pairs = (n + 1) / 2;
  isa::ex2_probe_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly, y_mufu,
                                                                                            y_ref, n);
  return isa::record_cuda_status(cudaGetLastError());
}

extern "C" int isa_selftest_umma_pair(const uint16_t* A, const uint16_t* B, const uint16_t* P, const uint16_t* V,
                                      float* S, float* O, void* ws, void* stream) {
  if (!A || !B || !P || !V || !S || !O || !ws) return ISA_ERR_INVALID_ARG;
  const int smem = 128 * 128 * 2 + 64 * 128 * 2 + 128 * 64 * 2 + 64 + 1024;
  cudaError_t e = cudaFuncSetAttribute(isa::umma_pair_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       116 * 1024);  // one CTA per SM: each pair CTA holds all 512 TMEM columns
  if (e != cudaSuccess) return isa::record_cuda_status(e);
  (void)smem;
  isa::umma_pair_probe_kernel<<<2, 128, 116 * 1024, static_cast<cudaStream_t>(stream)>>>(A, B, P, V, S, O,
                                                                                         static_cast<int*>(ws));
  return isa::record_cuda_status(cudaGetLastError());
}

extern "C" int isa_selftest_umma(int d, int bn, const uint16_t* A, const uint16_t* B, const uint16_t* P,
                                 const uint16_t* V, float* S, float* O, float* O2, void* ws, void* stream) {
  if (!A || !B || !P || !V || !S || !O || !O2 || !ws) return ISA_ERR_INVALID_ARG;
  int* status = reinterpret_cast<int*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128 && bn == 128) return isa::run_probe<128, 128>(A, B, P, V, S, O, O2, status, st);
  if (d == 128 && bn == 64) return isa::run_probe<128, 64>(A, B, P, V, S, O, O2, status, st);
  if (d == 64 && bn == 128) return isa::run_probe<64, 128>(A, B, P, V, S, O, O2, status, st);
  if (d == 64 && bn == 64) return isa::run_probe<64, 64>(A, B, P, V, S, O, O2, status, st);
  return ISA_ERR_UNSUPPORTED;
}
