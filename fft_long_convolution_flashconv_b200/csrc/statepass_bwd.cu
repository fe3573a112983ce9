// Backward pass of state passing (the long-sequence SSM): gradients with
// respect to u and the initial state, given dy and the gradient G of the
// final state.
//
// H3 summary, section 4 "Long-sequence computation" and appendix C.1
// "Backward Pass".  With lambda_t = dL/dx_t (complex: d/dRe + i d/dIm),
//   lambda_{L-1} = 2 conj(C) dy_{L-1} + G,
//   lambda_t     = 2 conj(C) dy_t + conj(A) lambda_{t+1},
//   du_t         = D dy_t + Re sum_n conj(lambda_t,n) B_n,
//   dstate_in    = conj(A) lambda_0.
// In reversed time tau = L-1-t this is the forward SSM
//   x'_tau = A' x'_{tau-1} + B' dy[L-1-tau],  y'_tau = 2 Re(C' x'_tau) + D dy[L-1-tau]
// with A' = conj(A) (lambda' = conj(lambda)), B' = 2 conj(C), C' = conj(B) / 2
// and x'_{-1} = G / conj(A), so du = reverse(y') and lambda_0 = x'_{L-1}: the
// same state-passing pipeline (chunk convolutions, end states, carry,
// initial-state term) runs on the reversed dy with these parameters.
#include "kernels.cuh"

namespace fc {

// lambda' = conj(lambda), B' = 2 conj(C), C' = conj(B) / 2 (H x N); x0' = G / conj(A) (B x H x N) when G is given.
__global__ void sp_adjoint_params_kernel(const float* __restrict__ dt, const float2* __restrict__ lam,
                                         const float2* __restrict__ Bp, const float2* __restrict__ Cp,
                                         const float2* __restrict__ G, float2* __restrict__ lam_a,
                                         float2* __restrict__ B_a, float2* __restrict__ C_a,
                                         float2* __restrict__ x0_a, int B, int H, int N) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long hn = (long long)H * N;
  if (i < hn) {
    const float2 l = lam[i], b = Bp[i], c = Cp[i];
    lam_a[i] = make_float2(l.x, -l.y);
    B_a[i] = make_float2(2.f * c.x, -2.f * c.y);
    C_a[i] = make_float2(0.5f * b.x, -0.5f * b.y);
  }
  if (G != nullptr && i < (long long)B * hn) {
    const long long r = i % hn;
    const int h = (int)(r / N);
    const float2 l = lam[r];
    const float2 a = ssm_pow(dt[h], l.x, -l.y, 1.0);  // conj(A)
    const float2 g = G[i];
    const float den = a.x * a.x + a.y * a.y;
    // g / a = g conj(a) / |a|^2
    x0_a[i] = make_float2((g.x * a.x + g.y * a.y) / den, (g.y * a.x - g.x * a.y) / den);
  }
}

// out[row][t] = in[row][L-1-t] for rows of L 16-bit or 32-bit elements (L a multiple of 16).
template <typename T>
__global__ void reverse_rows_kernel(const T* __restrict__ in, T* __restrict__ out, long long rows, int L) {
  constexpr int V = 16 / sizeof(T);  // elements per 16-byte vector
  const long long nv = (long long)L / V;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * nv) return;
  const long long r = i / nv, c = i - r * nv;
  const T* src = in + r * L + c * V;
  T* dst = out + r * L + (nv - 1 - c) * V;
  alignas(16) T v[V], w[V];
  *reinterpret_cast<uint4*>(v) = *reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int e = 0; e < V; ++e) w[e] = v[V - 1 - e];
  *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(w);
}

// dstate_in = conj(A) lambda_0 (lambda_0 = the adjoint run's final state).
__global__ void sp_adjoint_state_kernel(const float* __restrict__ dt, const float2* __restrict__ lam,
                                        const float2* __restrict__ lam0, float2* __restrict__ dsin, int B, int H,
                                        int N) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long hn = (long long)H * N;
  if (i >= (long long)B * hn) return;
  const long long r = i % hn;
  const int h = (int)(r / N);
  const float2 l = lam[r];
  dsin[i] = cmul(ssm_pow(dt[h], l.x, -l.y, 1.0), lam0[i]);
}

cudaError_t launch_sp_adjoint_params(const float* dt, const float* lam, const float* Bp, const float* Cp,
                                     const float* G, float* lam_a, float* B_a, float* C_a, float* x0_a, int B, int H,
                                     int N, cudaStream_t st) {
  const long long n = (long long)B * H * N;
  sp_adjoint_params_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
      dt, (const float2*)lam, (const float2*)Bp, (const float2*)Cp, (const float2*)G, (float2*)lam_a,
      (float2*)B_a, (float2*)C_a, (float2*)x0_a, B, H, N);
  return cudaGetLastError();
}

cudaError_t launch_reverse_rows(const void* in, void* out, long long rows, int L, int dtype, cudaStream_t st) {
  const long long n = rows * (long long)L / (dtype == 0 ? 4 : 8);
  const unsigned grid = (unsigned)((n + 255) / 256);
  if (dtype == 0)
    reverse_rows_kernel<float><<<grid, 256, 0, st>>>((const float*)in, (float*)out, rows, L);
  else
    reverse_rows_kernel<uint16_t><<<grid, 256, 0, st>>>((const uint16_t*)in, (uint16_t*)out, rows, L);
  return cudaGetLastError();
}

cudaError_t launch_sp_adjoint_state(const float* dt, const float* lam, const float* lam0, float* dsin, int B, int H,
                                    int N, cudaStream_t st) {
  const long long n = (long long)B * H * N;
  sp_adjoint_state_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(dt, (const float2*)lam,
                                                                      (const float2*)lam0, (float2*)dsin, B, H, N);
  return cudaGetLastError();
}

}  // namespace fc
