// State passing beyond one fused chunk (A7-A9), after the chunk convolutions
// (A6, done by the fused FFT-conv kernel with chunk-length rows).
//
// H3 summary section 4 "Long-sequence computation": each chunk is an FFT
// convolution and an end-state carried between chunks initialises the next;
// appendix C "State Passing": the chunk-input -> end-state map M_ux has the
// columns A^(T-1) B ... A B, B.  With x_t = A x_{t-1} + B u_t and
// y_t = 2 Re(C x_t) + D u_t:
//   local end-state   s_c[n]  = B_n sum_{i<T} A_n^(T-1-i) u_c[i]          (A7)
//   carry             x_c     = A^T x_{c-1} + s_c,  x_{-1} = state_in       (A8)
//   correction        y_c[t] += 2 Re sum_n C_n A_n^(t+1) x_{c-1,n}          (A9)
//
// Both contractions are evaluated in factored form with blocks of BL = 64
// positions (BL = T when T < 64), so that the inner loops are small real
// matrix products against tables of exactly phase-reduced powers:
//   A7:  Z[ih][n]  = sum_{il<BL} u[BL ih + il] A_n^(BL-1-il)
//        s[n]      = B_n sum_ih A_n^(T - BL (ih+1)) Z[ih][n]
//   A9:  e = t + 1 = BL eh + el,
//        y[e-1]   += sum_n Re( G[eh][n] Q[n][el] ),
//        G[eh][n]  = 2 C_n x_n A_n^(BL eh),  Q[n][el] = A_n^el
// One CTA owns one (b, h) row and walks its chunks; modes are processed in
// blocks of 64.  These CUDA-core kernels serve fp32 I/O, chunks other than
// 2048/4096/8192 and N > 64; the other cases run the same contractions as
// tcgen05 GEMMs (statepass_tc.cu) with this file's carry kernel.
#include "kernels.cuh"

namespace fc {

constexpr int kSpThr = 256;
constexpr int kSpNB = 64;   // modes per block
constexpr int kSpBL = 64;   // positions per block (when T >= 64)
constexpr int kSpMaxT = 8192;
constexpr int kSpMaxNH = kSpMaxT / kSpBL;               // 128
constexpr int kSpAcc = (kSpMaxNH + 1 + 3) / 4;          // 33 accumulators / thread

// ---------------------------------------------------------------- A7: local end-states
// grid (H, B).  smem: us[T] floats | Ap[BL][NB] float2 (A^(BL-1-il), [il][n]) | red[4][NB] float2
template <typename T>
__global__ void __launch_bounds__(kSpThr) sp_state_kernel(const T* __restrict__ u, const float* __restrict__ dt,
                                                           const float2* __restrict__ lam,
                                                           const float2* __restrict__ Bp, int H, int L, int N,
                                                           int Tc, float2* __restrict__ s_ws) {
  extern __shared__ __align__(16) float sp_sm[];
  const int h = blockIdx.x, b = blockIdx.y;
  const int C = L / Tc;
  const int BL = Tc < kSpBL ? Tc : kSpBL;
  const int NH = Tc / BL;
  float* us = sp_sm;                                             // Tc floats
  float2* Ap = reinterpret_cast<float2*>(sp_sm + kSpMaxT);       // BL x NB
  float2* red = Ap + kSpBL * kSpNB;                              // 4 x NB
  const int tid = threadIdx.x;
  const int nl = tid & (kSpNB - 1);
  const int ig = tid >> 6;  // 0..3
  const float d = dt[h];
  const size_t rowoff = ((size_t)b * H + h) * (size_t)L;
  const long long ulim = (long long)gridDim.y * H * L;

  for (int n0 = 0; n0 < N; n0 += kSpNB) {
    const int nb = min(kSpNB, N - n0);
    __syncthreads();
    for (int idx = tid; idx < BL * kSpNB; idx += kSpThr) {
      const int il = idx / kSpNB, n = idx - il * kSpNB;
      float2 v = make_float2(0.f, 0.f);
      if (n < nb) {
        const float2 lm = lam[(size_t)h * N + n0 + n];
        v = ssm_pow(d, lm.x, lm.y, (double)(BL - 1 - il));
      }
      if (FC_OK_IDX(30, idx, kSpBL * kSpNB)) Ap[idx] = v;
    }
    // per-thread walking factor A^(4 BL) and the start power for its last block
    const bool nv = nl < nb;
    float2 step = make_float2(1.f, 0.f), p0 = make_float2(0.f, 0.f);
    int ihmax = -1;
    if (nv) {
      const float2 lm = lam[(size_t)h * N + n0 + nl];
      step = ssm_pow(d, lm.x, lm.y, 4.0 * BL);
      for (int ih = ig; ih < NH; ih += 4) ihmax = ih;
      if (ihmax >= 0) p0 = ssm_pow(d, lm.x, lm.y, (double)(Tc - BL * (ihmax + 1)));
    }
    for (int c = 0; c < C; ++c) {
      __syncthreads();
      for (int i = tid; i < Tc; i += kSpThr) {
        const long long gi = (long long)rowoff + (long long)c * Tc + i;
        us[i] = FC_OK_IDX(31, gi, ulim) ? IO<T>::ld(u + gi) : 0.f;
      }
      __syncthreads();
      float2 acc = make_float2(0.f, 0.f);
      if (nv) {
        float2 p = p0;
        for (int ih = ihmax; ih >= 0; ih -= 4) {
          float zr = 0.f, zi = 0.f;
          const float* ub = us + ih * BL;
          for (int il = 0; il < BL; ++il) {
            const float uv = FC_OK_IDX(32, ih * BL + il, Tc) ? ub[il] : 0.f;
            const float2 a = Ap[il * kSpNB + nl];
            zr = fmaf(uv, a.x, zr);
            zi = fmaf(uv, a.y, zi);
          }
          acc = cadd(acc, cmul(p, make_float2(zr, zi)));
          p = cmul(p, step);
        }
      }
      if (FC_OK_IDX(33, ig * kSpNB + nl, 4 * kSpNB)) red[ig * kSpNB + nl] = acc;
      __syncthreads();
      if (tid < nb) {
        float2 s = red[tid];
        for (int g = 1; g < 4; ++g) s = cadd(s, red[g * kSpNB + tid]);
        const size_t si = (((size_t)b * H + h) * C + c) * N + n0 + tid;
        if (FC_OK_IDX(34, si, (long long)gridDim.y * H * C * N)) s_ws[si] = cmul(s, Bp[(size_t)h * N + n0 + tid]);
      }
    }
  }
}

// ---------------------------------------------------------------- A8: carry
// One thread per (b, h, n): x_ws[(row c) N + n] = state entering chunk c.
__global__ void sp_carry_kernel(const float* __restrict__ dt, const float2* __restrict__ lam,
                                const float2* __restrict__ s_ws, const float2* __restrict__ state_in,
                                float2* __restrict__ state_out, float2* __restrict__ x_ws, int B, int H, int N, int C,
                                int Tc) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)B * H * N;
  if (idx >= total) return;
  const int n = (int)(idx % N);
  const long long bh = idx / N;
  const int h = (int)(bh % H);
  const float2 lm = lam[(size_t)h * N + n];
  const float2 aT = ssm_pow(dt[h], lm.x, lm.y, (double)Tc);
  float2 x = make_float2(0.f, 0.f);
  if (state_in != nullptr) x = state_in[idx];
  for (int c = 0; c < C; ++c) {
    const long long si = (bh * C + c) * N + n;
    if (!FC_OK_IDX(40, si, total * C)) break;
    x_ws[si] = x;
    x = cadd(cmul(aT, x), s_ws[si]);
  }
  if (state_out != nullptr) state_out[idx] = x;
}

// ---------------------------------------------------------------- A9: correction
// grid (H, B).  smem: Q[NB][BL] (A^el, [n][el]) | AH[NH+1][NB] (A^(BL eh)) | G[NH+1][NB]
template <typename T>
__global__ void __launch_bounds__(kSpThr) sp_corr_kernel(T* __restrict__ y, const float* __restrict__ dt,
                                                          const float2* __restrict__ lam,
                                                          const float2* __restrict__ Cp,
                                                          const float2* __restrict__ x_ws, int H, int L, int N,
                                                          int Tc) {
  extern __shared__ __align__(16) float2 spc_sm[];
  const int h = blockIdx.x, b = blockIdx.y;
  const int C = L / Tc;
  const int BL = Tc < kSpBL ? Tc : kSpBL;
  const int NH = Tc / BL;
  float2* Q = spc_sm;                                  // kSpNB x kSpBL
  float2* AH = Q + kSpNB * kSpBL;                      // (kSpMaxNH+1) x kSpNB
  float2* G = AH + (kSpMaxNH + 1) * kSpNB;             // (kSpMaxNH+1) x kSpNB
  const int tid = threadIdx.x;
  const int el = tid & 63;
  const int eg = tid >> 6;
  const float d = dt[h];
  const size_t rowoff = ((size_t)b * H + h) * (size_t)L;
  const long long ylim = (long long)gridDim.y * H * L;
  const int QN = kSpNB * kSpBL, GN = (kSpMaxNH + 1) * kSpNB;

  for (int c = 0; c < C; ++c) {
    float acc[kSpAcc];
#pragma unroll
    for (int k = 0; k < kSpAcc; ++k) acc[k] = 0.f;
    for (int n0 = 0; n0 < N; n0 += kSpNB) {
      const int nb = min(kSpNB, N - n0);
      __syncthreads();
      if (c == 0 || N > kSpNB) {  // tables depend on the mode block only
        for (int idx = tid; idx < kSpNB * BL; idx += kSpThr) {
          const int n = idx / BL, e = idx - n * BL;
          float2 v = make_float2(0.f, 0.f);
          if (n < nb) {
            const float2 lm = lam[(size_t)h * N + n0 + n];
            v = ssm_pow(d, lm.x, lm.y, (double)e);
          }
          if (FC_OK_IDX(50, n * kSpBL + e, QN)) Q[n * kSpBL + e] = v;
        }
        for (int idx = tid; idx < (NH + 1) * kSpNB; idx += kSpThr) {
          const int eh = idx / kSpNB, n = idx - eh * kSpNB;
          float2 v = make_float2(0.f, 0.f);
          if (n < nb) {
            const float2 lm = lam[(size_t)h * N + n0 + n];
            v = ssm_pow(d, lm.x, lm.y, (double)BL * eh);
          }
          if (FC_OK_IDX(51, idx, GN)) AH[idx] = v;
        }
        __syncthreads();
      }
      const size_t xrow = (((size_t)b * H + h) * C + c) * N + n0;
      for (int idx = tid; idx < (NH + 1) * kSpNB; idx += kSpThr) {
        const int eh = idx / kSpNB, n = idx - eh * kSpNB;
        float2 v = make_float2(0.f, 0.f);
        if (n < nb && FC_OK_IDX(52, xrow + n, (long long)gridDim.y * H * C * N)) {
          const float2 w = cmul(Cp[(size_t)h * N + n0 + n], x_ws[xrow + n]);
          v = cmul(make_float2(2.f * w.x, 2.f * w.y), AH[idx]);
        }
        if (FC_OK_IDX(53, idx, GN)) G[idx] = v;
      }
      __syncthreads();
      if (el < BL) {
        for (int n = 0; n < nb; ++n) {
          const float2 q = Q[n * kSpBL + el];
#pragma unroll
          for (int k = 0; k < kSpAcc; ++k) {
            const int eh = eg + 4 * k;
            if (eh <= NH) {
              const float2 g = G[eh * kSpNB + n];
              acc[k] = fmaf(g.x, q.x, fmaf(-g.y, q.y, acc[k]));
            }
          }
        }
      }
    }
    // y[c T + e - 1] += acc, for 1 <= e = BL eh + el <= T
    if (el < BL) {
#pragma unroll
      for (int k = 0; k < kSpAcc; ++k) {
        const int eh = eg + 4 * k;
        const int e = BL * eh + el;
        if (eh <= NH && e >= 1 && e <= Tc) {
          const long long yi = (long long)rowoff + (long long)c * Tc + e - 1;
          if (FC_OK_IDX(54, yi, ylim)) IO<T>::st(y + yi, IO<T>::ldplain(y + yi) + acc[k]);
        }
      }
    }
  }
}

template <typename T>
static cudaError_t sp_tail(const void* u, const float* dt, const float* lam, const float* Bp, const float* Cp,
                           void* y, int B, int H, int L, int N, int Tc, const float* state_in, float* state_out,
                           float* s_ws, float* x_ws, cudaStream_t st) {
  if (Tc > kSpMaxT || Tc < 1) return cudaErrorInvalidValue;
  const int C = L / Tc;
  const size_t smem1 = sizeof(float) * kSpMaxT + sizeof(float2) * (kSpBL * kSpNB + 4 * kSpNB);
  cudaError_t e = smem_optin<sp_state_kernel<T>>(smem1);
  if (e != cudaSuccess) return e;
  sp_state_kernel<T><<<dim3(H, B), kSpThr, smem1, st>>>((const T*)u, dt, (const float2*)lam, (const float2*)Bp, H,
                                                         L, N, Tc, (float2*)s_ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long nst = (long long)B * H * N;
  sp_carry_kernel<<<(unsigned)((nst + 255) / 256), 256, 0, st>>>(dt, (const float2*)lam, (const float2*)s_ws,
                                                                 (const float2*)state_in, (float2*)state_out,
                                                                 (float2*)x_ws, B, H, N, C, Tc);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem3 = sizeof(float2) * ((size_t)kSpNB * kSpBL + 2 * (size_t)(kSpMaxNH + 1) * kSpNB);
  e = smem_optin<sp_corr_kernel<T>>(smem3);
  if (e != cudaSuccess) return e;
  sp_corr_kernel<T><<<dim3(H, B), kSpThr, smem3, st>>>((T*)y, dt, (const float2*)lam, (const float2*)Cp,
                                                        (const float2*)x_ws, H, L, N, Tc);
  return cudaGetLastError();
}

// Tensor-core tail: end states and corrections as tcgen05 GEMMs, the carry as above.
static cudaError_t sp_tail_tc(const void* u, const float* dt, const float* lam, const float* Bp, const float* Cp,
                              void* y, int B, int H, int L, int N, int Tc, const float* state_in, float* state_out,
                              float* s_ws, float* x_ws, int dtype, cudaStream_t st) {
  const int C = L / Tc;
  cudaError_t e = launch_sp_state_tc(u, dt, lam, Bp, B, H, L, N, Tc, s_ws, dtype, st);
  if (e != cudaSuccess) return e;
  const long long nst = (long long)B * H * N;
  sp_carry_kernel<<<(unsigned)((nst + 255) / 256), 256, 0, st>>>(dt, (const float2*)lam, (const float2*)s_ws,
                                                                 (const float2*)state_in, (float2*)state_out,
                                                                 (float2*)x_ws, B, H, N, C, Tc);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // with no initial state the first chunk needs no correction
  return launch_sp_corr_tc(y, dt, lam, Cp, x_ws, B, H, L, N, Tc, state_in != nullptr ? 0 : 1, dtype, st);
}

cudaError_t launch_statepass_tail(const void* u, const float* dt, const float* lam, const float* Bp,
                                  const float* Cp, void* y, int B, int H, int L, int N, int T_,
                                  const float* state_in, float* state_out, float* s_ws, float* x_ws, int dtype,
                                  cudaStream_t st) {
  if (statepass_tc_supported(T_, N, dtype))
    return sp_tail_tc(u, dt, lam, Bp, Cp, y, B, H, L, N, T_, state_in, state_out, s_ws, x_ws, dtype, st);
  switch (dtype) {
    case 0: return sp_tail<float>(u, dt, lam, Bp, Cp, y, B, H, L, N, T_, state_in, state_out, s_ws, x_ws, st);
    case 1: return sp_tail<__half>(u, dt, lam, Bp, Cp, y, B, H, L, N, T_, state_in, state_out, s_ws, x_ws, st);
    case 2:
      return sp_tail<__nv_bfloat16>(u, dt, lam, Bp, Cp, y, B, H, L, N, T_, state_in, state_out, s_ws, x_ws, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fc

FC_CHECK_READER(fc_check_statepass)
