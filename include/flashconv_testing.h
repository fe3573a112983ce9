/* flashconv_testing.h -- test hooks of libflashconv_b200.so (not part of the
 * convolution API).  The pages have no counterpart: these exist so the GPU
 * tests can pin the tensor-core building blocks against plain arithmetic.
 */
#ifndef FLASHCONV_B200_TESTING_H
#define FLASHCONV_B200_TESTING_H

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FC_TEST_API __attribute__((visibility("default")))
#else
#define FC_TEST_API
#endif

/* D[128 x N] (fp32, row-major, device) = A[128 x K] * B[N x K]^T, with A and
 * B row-major fp16 (bf16 = 0) or bf16 (bf16 = 1) device arrays, computed by
 * one CTA on the 5th-generation tensor cores (tcgen05.mma, accumulator in
 * tensor memory).  *err (device int, caller-zeroed) is set to 1 if the MMA
 * completion wait gave up after one second.  N, K: multiples of 16,
 * 16 <= N <= 256, 16 <= K <= 256.  Returns 0, or -1 (bad argument) / -3
 * (launch failure). */
FC_TEST_API int fc_selftest_umma(const void* A, const void* B, float* D, int* err, int N, int K, int bf16,
                                 void* stream);

/* Same product with general operand layouts: a_mn / b_mn = 1 selects an
 * MN-major operand (core matrices of 8 K-rows x 8 contiguous MN-elements),
 * 0 a K-major one; *_lbo / *_sbo are the byte offsets between core matrices
 * along K / along M or N (multiples of 16, padding allowed).  Returns -1 for
 * arguments outside those limits or a shared-memory footprint above 200 KB. */
FC_TEST_API int fc_selftest_umma2(const void* A, const void* B, float* D, int* err, int N, int K, int bf16, int a_mn,
                                  int b_mn, int a_lbo, int a_sbo, int b_lbo, int b_sbo, void* stream);

/* The same product with A held in tensor memory: each row of A (K 16-bit
 * elements) is written with tcgen05.st, two elements per 32-bit column (even
 * k in the low half), and the MMA reads A from there.  Same limits and
 * returns as fc_selftest_umma. */
FC_TEST_API int fc_selftest_umma_tmem_a(const void* A, const void* B, float* D, int* err, int N, int K, int bf16,
                                        void* stream);

/* Number of tensor-core CTAs (all tcgen05 kernels of the library, since load)
 * that gave up waiting for MMA completion after their bounded wait; each such
 * CTA skipped its remaining work and freed its tensor memory.  0 in normal
 * operation; the GPU tests assert that it stays 0. */
FC_TEST_API unsigned int fc_debug_tc_timeouts(void);

#ifdef __cplusplus
}
#endif
#endif
