// Diagonal-SSM filter generation (A1):
//   f[h,k] = 2 Re sum_n C[h,n] B[h,n] A[h,n]^k,  A = exp(dt * lambda)
// (H3 blog "The Convolution Connection": f = [CB, CAB, CA^2B, ...]).
//
// One CTA evaluates 2048 taps of one channel with the factored tables of
// ssm_tables.cuh (a real contraction over the modes, blocks of 64 modes).
#include "kernels.cuh"

#include "ssm_tables.cuh"

namespace fc {

constexpr int kGenTile = 2048;    // taps per CTA
constexpr int kGenThreads = 256;
constexpr int kGenMB = 64;        // modes per table block
constexpr int kGenKH = kGenTile / 64;
constexpr size_t kGenSmem = sizeof(float2) * ((size_t)kGenMB * 64 + (size_t)kGenKH * kGenMB +
                                              (size_t)kGenMB * ssm_scratch_per_mode(kGenKH));

__global__ void __launch_bounds__(kGenThreads) ssm_gen_kernel(const float* __restrict__ dt,
                                                             const float2* __restrict__ lam,
                                                             const float2* __restrict__ Bp,
                                                             const float2* __restrict__ Cp, int H, int N,
                                                             int L, float* __restrict__ f) {
  extern __shared__ float2 gsm[];
  float2* Q = gsm;                       // [m][64]
  float2* W = Q + kGenMB * 64;           // [kh][kGenMB]
  float2* X = W + kGenKH * kGenMB;       // scratch
  const int h = blockIdx.y;
  const long long k0 = (long long)blockIdx.x * kGenTile;
  const int ntap = (int)min((long long)kGenTile, (long long)L - k0);
  const int KH = (ntap + 63) >> 6;
  const int kl = threadIdx.x & 63;
  const int kg = threadIdx.x >> 6;  // 0..3
  constexpr int PER = kGenKH / (kGenThreads / 64);  // 8
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  for (int m0 = 0; m0 < N; m0 += kGenMB) {
    const int mb = min(kGenMB, N - m0);
    __syncthreads();  // previous block's readers are done
    ssm_fill_tables(dt, lam, Bp, Cp, h, N, m0, mb, kGenMB, k0, KH, Q, W, X, threadIdx.x, kGenThreads);
    for (int m = 0; m < mb; ++m) {
      const float2 q = Q[m * 64 + kl];
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int kh = kg + 4 * i;
        if (kh < KH) {
          const float2 w = W[kh * kGenMB + m];
          acc[i] = fmaf(w.x, q.x, fmaf(-w.y, q.y, acc[i]));
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int k = 64 * (kg + 4 * i) + kl;
    if (k < ntap && FC_OK_IDX(20, (long long)h * L + k0 + k, (long long)H * L)) f[(size_t)h * L + k0 + k] = acc[i];
  }
}

cudaError_t launch_ssm_gen(const float* dt, const float* lam, const float* Bp, const float* Cp, int H, int N,
                           int L, float* f, cudaStream_t st) {
  const int tiles = (L + kGenTile - 1) / kGenTile;
  cudaError_t e = cudaFuncSetAttribute(ssm_gen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGenSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(tiles, H);
  ssm_gen_kernel<<<grid, kGenThreads, kGenSmem, st>>>(dt, reinterpret_cast<const float2*>(lam),
                                                      reinterpret_cast<const float2*>(Bp),
                                                      reinterpret_cast<const float2*>(Cp), H, N, L, f);
  return cudaGetLastError();
}

}  // namespace fc

FC_CHECK_READER(fc_check_ssm_gen)
