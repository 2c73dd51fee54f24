/*
 * isa_selftest.h -- test-only export of libisa.so (not part of the ISA method).
 *
 * isa_selftest_umma runs ONE tile of the tensor-core building blocks used by
 * the attention kernels, so that a wrong shared-memory or instruction
 * descriptor shows up as a wrong product rather than as a wrong attention
 * output.  All pointers are device pointers, row-major, 16-byte aligned:
 *   A [128, d] bf16, B [bn, d] bf16      -> S [128, bn] fp32 = A B^T
 *   P [128, bn] bf16, V [bn, d] bf16     -> O [128, d] fp32  = P V  (P from shared memory)
 *                                        -> O2 [128, d] fp32 = P V  (P from tensor memory)
 * d and bn in {64, 128}.  ws: >= 256 bytes, zeroed; its first int32 receives
 * ISA_ERR_DEVICE_TIMEOUT if a bounded wait expires.  Asynchronous on stream.
 *
 * isa_selftest_ex2 evaluates the softmax's exponentials on n given fp32
 * arguments x (device pointers, n >= 0): y_poly = the FMA-pipe 2^x of the
 * attention kernels (Cody-Waite reduction, minimax cubic; arguments taken in
 * pairs as the kernels do), y_mufu = the MUFU ex2.approx.ftz used for the
 * other exponentials, y_ref = CUDA's exp2f.  Asynchronous on stream;
 * ISA_ERR_INVALID_ARG for n < 0 or a null pointer when n > 0.
 *
 * isa_selftest_umma_pair runs one M = 256 tile on a pair of CTAs (two SMs,
 * one cluster): S [256, 128] fp32 = A B^T and O [256, 128] fp32 = P V with
 * A [256, 128], B [128, 128] (keys x d), P [256, 128], V [128, 128] bf16,
 * the even CTA issuing both products; each CTA holds 128 rows of A, half
 * the keys of B, its 128 rows of P (in tensor memory) and half the columns
 * of V.  ws as for isa_selftest_umma.
 */
#ifndef ISA_SELFTEST_H_
#define ISA_SELFTEST_H_
#include <stdint.h>
#ifdef __cplusplus
extern "C" {
#endif
int isa_selftest_umma(int d, int bn, const uint16_t* A, const uint16_t* B, const uint16_t* P, const uint16_t* V,
                      float* S, float* O, float* O2, void* ws, void* stream);
int isa_selftest_ex2(const float* x, float* y_poly, float* y_mufu, float* y_ref, int n, void* stream);
int isa_selftest_umma_pair(const uint16_t* A, const uint16_t* B, const uint16_t* P, const uint16_t* V, float* S,
                           float* O, void* ws, void* stream);
#ifdef __cplusplus
}
#endif
#endif
