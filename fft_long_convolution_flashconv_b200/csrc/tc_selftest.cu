// Self-test of the tcgen05 wrappers (test hook, not part of the convolution
// path): D[128 x N] = A[128 x K] * B[N x K]^T with fp16 or bf16 operands staged
// into the K-major no-swizzle layout, accumulated in tensor memory, read back
// with tcgen05.ld.  Used by the GPU tests to pin the descriptor and TMEM
// layouts against a plain matrix product.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/flashconv_testing.h"
#include "tc100.cuh"

namespace fc {

__global__ void __launch_bounds__(128, 1) umma_selftest_kernel(const uint16_t* __restrict__ A,
                                                               const uint16_t* __restrict__ B, float* __restrict__ D,
                                                               int* __restrict__ err, int N, int K, int bf16) {
  extern __shared__ __align__(1024) uint8_t sm[];
  __shared__ uint64_t mbar;
  __shared__ uint32_t tmem_base;
  uint8_t* sA = sm;                       // 128 x K
  uint8_t* sB = sm + (size_t)128 * K * 2; // N x K
  const int tid = threadIdx.x, warp = tid >> 5;
  // stage operands (element-wise; this is a test)
  for (int idx = tid; idx < 128 * K; idx += 128) {
    const int r = idx / K, k = idx - r * K;
    *reinterpret_cast<uint16_t*>(sA + tc::kmaj_off(r, k, K)) = A[idx];
  }
  for (int idx = tid; idx < N * K; idx += 128) {
    const int r = idx / K, k = idx - r * K;
    *reinterpret_cast<uint16_t*>(sB + tc::kmaj_off(r, k, K)) = B[idx];
  }
  uint32_t ncols = 32;
  while (ncols < (uint32_t)N) ncols <<= 1;
  if (warp == 0) tc::tmem_alloc(&tmem_base, ncols);
  if (tid == 0) {
    tc::mbar_init(&mbar, 1);
    tc::fence_mbar_init();
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = tmem_base;
  if (tid == 0) {
    const uint32_t idesc = tc::idesc_f16(128, N, bf16);
    const uint32_t a0 = tc::smem_u32(sA), b0 = tc::smem_u32(sB);
    for (int kk = 0; kk < K / 16; ++kk) {
      const uint64_t ad = tc::desc_kmajor(a0 + kk * 256, 128, (K / 8) * 128);
      const uint64_t bd = tc::desc_kmajor(b0 + kk * 256, 128, (K / 8) * 128);
      tc::mma_f16(tbase, ad, bd, idesc, kk > 0 ? 1u : 0u);
    }
    tc::mma_commit(&mbar);
  }
  const bool ok = tc::mbar_wait_bounded(&mbar, 0, 1000000000ull);
  tc::fence_after_sync();
  if (!ok) {
    if (tid == 0) atomicExch(err, 1);
  } else {
    const int row = warp * 32 + (tid & 31);
    for (int c = 0; c < N; c += 16) {
      float v[16];
      tc::tmem_ld16_wait(tbase + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
      for (int i = 0; i < 16; ++i) D[(size_t)row * N + c + i] = v[i];
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, ncols);
}

// A operand in tensor memory: each thread writes its row m of A (K 16-bit
// elements, two per 32-bit column, element k in column k / 2, even k in the low
// half) with tcgen05.st; the MMA reads A from TMEM columns [0, K/2) and B from
// shared memory; D goes to columns [128, 128 + N).
__global__ void __launch_bounds__(128, 1) umma_selftest_tmem_a_kernel(const uint16_t* __restrict__ A,
                                                                      const uint16_t* __restrict__ B,
                                                                      float* __restrict__ D, int* __restrict__ err,
                                                                      int N, int K, int bf16) {
  extern __shared__ __align__(1024) uint8_t sm[];
  __shared__ uint64_t mbar;
  __shared__ uint32_t tmem_base;
  uint8_t* sB = sm;  // N x K, K-major
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int idx = tid; idx < N * K; idx += 128) {
    const int r = idx / K, k = idx - r * K;
    *reinterpret_cast<uint16_t*>(sB + tc::kmaj_off(r, k, K)) = B[idx];
  }
  if (warp == 0) tc::tmem_alloc(&tmem_base, 512);
  if (tid == 0) {
    tc::mbar_init(&mbar, 1);
    tc::fence_mbar_init();
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = tmem_base;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const int row = warp * 32 + (tid & 31);
  for (int c = 0; c < K / 2; c += 8) {  // 8 columns = 16 elements of this row per store
    uint32_t w[8];
    for (int i = 0; i < 8; ++i)
      w[i] = (uint32_t)A[(size_t)row * K + 2 * (c + i)] | ((uint32_t)A[(size_t)row * K + 2 * (c + i) + 1] << 16);
    tc::tmem_st8(tbase + lane_off + (uint32_t)c, w);
  }
  tc::tmem_wait_st();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (tid == 0) {
    const uint32_t idesc = tc::idesc_f16(128, N, bf16);
    const uint32_t b0 = tc::smem_u32(sB);
    for (int kk = 0; kk < K / 16; ++kk)
      tc::mma_f16_tmem_a(tbase + 128, tbase + (uint32_t)(8 * kk), tc::desc_kmajor(b0 + kk * 256, 128, (K / 8) * 128),
                         idesc, kk > 0 ? 1u : 0u);
    tc::mma_commit(&mbar);
  }
  const bool ok = tc::mbar_wait_bounded(&mbar, 0, 1000000000ull);
  tc::fence_after_sync();
  if (!ok) {
    if (tid == 0) atomicExch(err, 1);
  } else {
    for (int c = 0; c < N; c += 16) {
      float v[16];
      tc::tmem_ld16_wait(tbase + lane_off + 128u + (uint32_t)c, v);
      for (int i = 0; i < 16; ++i) D[(size_t)row * N + c + i] = v[i];
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, 512);
}

// General-layout variant: A / B may be MN-major and use any core-matrix
// offsets (lbo along K, sbo along M/N), e.g. padded ones.
__global__ void __launch_bounds__(128, 1) umma_selftest2_kernel(const uint16_t* __restrict__ A,
                                                                const uint16_t* __restrict__ B,
                                                                float* __restrict__ D, int* __restrict__ err, int N,
                                                                int K, int bf16, int a_mn, int b_mn, int a_lbo,
                                                                int a_sbo, int b_lbo, int b_sbo, int a_bytes) {
  extern __shared__ __align__(1024) uint8_t sm[];
  __shared__ uint64_t mbar;
  __shared__ uint32_t tmem_base;
  uint8_t* sA = sm;
  uint8_t* sB = sm + a_bytes;
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int idx = tid; idx < 128 * K; idx += 128) {
    const int r = idx / K, k = idx - r * K;
    *reinterpret_cast<uint16_t*>(sA + tc::op_off(r, k, a_mn, a_lbo, a_sbo)) = A[idx];
  }
  for (int idx = tid; idx < N * K; idx += 128) {
    const int r = idx / K, k = idx - r * K;
    *reinterpret_cast<uint16_t*>(sB + tc::op_off(r, k, b_mn, b_lbo, b_sbo)) = B[idx];
  }
  uint32_t ncols = 32;
  while (ncols < (uint32_t)N) ncols <<= 1;
  if (warp == 0) tc::tmem_alloc(&tmem_base, ncols);
  if (tid == 0) {
    tc::mbar_init(&mbar, 1);
    tc::fence_mbar_init();
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = tmem_base;
  if (tid == 0) {
    const uint32_t idesc = tc::idesc_f16(128, N, bf16, a_mn, b_mn);
    const uint32_t a0 = tc::smem_u32(sA), b0 = tc::smem_u32(sB);
    for (int kk = 0; kk < K / 16; ++kk) {
      const uint64_t ad = tc::desc_kmajor(a0 + kk * 2 * a_lbo, a_lbo, a_sbo);
      const uint64_t bd = tc::desc_kmajor(b0 + kk * 2 * b_lbo, b_lbo, b_sbo);
      tc::mma_f16(tbase, ad, bd, idesc, kk > 0 ? 1u : 0u);
    }
    tc::mma_commit(&mbar);
  }
  const bool ok = tc::mbar_wait_bounded(&mbar, 0, 1000000000ull);
  tc::fence_after_sync();
  if (!ok) {
    if (tid == 0) atomicExch(err, 1);
  } else {
    const int row = warp * 32 + (tid & 31);
    for (int c = 0; c < N; c += 16) {
      float v[16];
      tc::tmem_ld16_wait(tbase + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
      for (int i = 0; i < 16; ++i) D[(size_t)row * N + c + i] = v[i];
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, ncols);
}

}  // namespace fc

FC_TEST_API int fc_selftest_umma_tmem_a(const void* A, const void* B, float* D, int* err, int N, int K, int bf16,
                                        void* stream) {
  if (!A || !B || !D || !err || N < 16 || N > 256 || (N % 16) || K < 16 || K > 256 || (K % 16)) return -1;
  const size_t smem = (size_t)N * K * 2;
  cudaError_t e = cudaFuncSetAttribute(fc::umma_selftest_tmem_a_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return -3;
  fc::umma_selftest_tmem_a_kernel<<<1, 128, smem, (cudaStream_t)stream>>>(
      (const uint16_t*)A, (const uint16_t*)B, D, err, N, K, bf16);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

extern "C" FC_TEST_API int fc_selftest_umma2(const void* A, const void* B, float* D, int* err, int N, int K, int bf16,
                                             int a_mn, int b_mn, int a_lbo, int a_sbo, int b_lbo, int b_sbo,
                                             void* stream) {
  if (!A || !B || !D || !err) return -1;
  if (N < 16 || N > 256 || N % 16 || K < 16 || K > 256 || K % 16 || (bf16 != 0 && bf16 != 1)) return -1;
  if (a_lbo % 16 || a_sbo % 16 || b_lbo % 16 || b_sbo % 16 || a_lbo <= 0 || b_lbo <= 0 || a_sbo <= 0 ||
      b_sbo <= 0 || a_lbo >= (1 << 18) || a_sbo >= (1 << 18) || b_lbo >= (1 << 18) || b_sbo >= (1 << 18))
    return -1;
  // footprint: furthest core matrix + 128 bytes, rounded to 1 KB
  const size_t a_bytes = ((size_t)(128 / 8 - 1) * a_sbo + (size_t)(K / 8 - 1) * a_lbo + 128 + 1023) / 1024 * 1024;
  const size_t b_bytes = (size_t)(N / 8 - 1) * b_sbo + (size_t)(K / 8 - 1) * b_lbo + 128;
  const size_t smem = a_bytes + b_bytes;
  if (smem > 200 * 1024) return -1;
  cudaError_t e = cudaFuncSetAttribute(fc::umma_selftest2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return -3;
  fc::umma_selftest2_kernel<<<1, 128, smem, (cudaStream_t)stream>>>((const uint16_t*)A, (const uint16_t*)B, D, err,
                                                                    N, K, bf16, a_mn, b_mn, a_lbo, a_sbo, b_lbo,
                                                                    b_sbo, (int)a_bytes);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

extern "C" FC_TEST_API int fc_selftest_umma(const void* A, const void* B, float* D, int* err, int N, int K, int bf16,
                                            void* stream) {
  if (!A || !B || !D || !err) return -1;
  if (N < 16 || N > 256 || N % 16 || K < 16 || K > 256 || K % 16 || (bf16 != 0 && bf16 != 1)) return -1;
  const size_t smem = (size_t)(128 + N) * K * 2;
  cudaError_t e = cudaFuncSetAttribute(fc::umma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return -3;
  fc::umma_selftest_kernel<<<1, 128, smem, (cudaStream_t)stream>>>((const uint16_t*)A, (const uint16_t*)B, D, err,
                                                                   N, K, bf16);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}
