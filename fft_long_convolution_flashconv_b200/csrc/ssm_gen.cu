// Diagonal-SSM filter generation (A1):
//   f[h,k] = 2 Re sum_n C[h,n] B[h,n] A[h,n]^k,  A = exp(dt * lambda)
// (H3 blog "The Convolution Connection": f = [CB, CAB, CA^2B, ...]).
//
// One CTA evaluates 1024 taps of one channel with the factored tables of
// ssm_tables.cuh (a real contraction over the modes, blocks of 64 modes).
#include "kernels.cuh"

#include "ssm_tables.cuh"

namespace fc {

constexpr int kGenTile = 1024;    // taps per CTA
constexpr int kGenThreads = 128;
constexpr int kGenMB = 64;        // modes per table block
constexpr int kGenKH = kGenTile / 64;  // 16
constexpr size_t kGenSmem = sizeof(float2) * ((size_t)kGenMB * 64 + (size_t)kGenKH * kGenMB +
                                              (size_t)kGenMB * ssm_scratch_per_mode(kGenKH));

// Thread t owns taps e in {2(t%32), 2(t%32)+1} x kh in {4(t/32) .. 4(t/32)+3}:
// per mode one 16-byte Q load (two consecutive e) and four broadcast 8-byte W
// loads (the warp shares its kh group) feed 16 FMAs.
__global__ void __launch_bounds__(kGenThreads) ssm_gen_kernel(const float* __restrict__ dt,
                                                             const float2* __restrict__ lam,
                                                             const float2* __restrict__ Bp,
                                                             const float2* __restrict__ Cp, int H, int N,
                                                             int L, float* __restrict__ f) {
  extern __shared__ __align__(16) float2 gsm[];
  float2* Q = gsm;                       // [m][64]
  float2* Wt = Q + kGenMB * 64;          // [kh][kGenMB] as written by ssm_fill_tables
  float2* X = Wt + kGenKH * kGenMB;      // scratch
  const int h = blockIdx.y;
  const long long k0 = (long long)blockIdx.x * kGenTile;
  const int ntap = (int)min((long long)kGenTile, (long long)L - k0);
  const int KH = (ntap + 63) >> 6;
  const int lane = threadIdx.x & 31;
  const int g = threadIdx.x >> 5;  // kh group 0..3
  float acc[2][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
  for (int m0 = 0; m0 < N; m0 += kGenMB) {
    const int mb = min(kGenMB, N - m0);
    __syncthreads();  // previous block's readers are done
    ssm_fill_tables(dt, lam, Bp, Cp, h, N, m0, mb, kGenMB, k0, KH, Q, Wt, X, threadIdx.x, kGenThreads);
    for (int m = 0; m < mb; ++m) {
      const float4 q = *reinterpret_cast<const float4*>(Q + m * 64 + 2 * lane);
      float2 w[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int kh = 4 * g + c;
        w[c] = kh < KH ? Wt[kh * kGenMB + m] : make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[0][c] = fmaf(w[c].x, q.x, fmaf(-w[c].y, q.y, acc[0][c]));
        acc[1][c] = fmaf(w[c].x, q.z, fmaf(-w[c].y, q.w, acc[1][c]));
      }
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int k = 64 * (4 * g + c) + 2 * lane + a;
      if (k < ntap && FC_OK_IDX(20, (long long)h * L + k0 + k, (long long)H * L)) f[(size_t)h * L + k0 + k] = acc[a][c];
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
