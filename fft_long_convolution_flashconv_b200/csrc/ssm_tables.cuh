// Factored evaluation of the diagonal-SSM filter (H3 blog "The Convolution
// Connection": f = [CB, CAB, CA^2B, ...], 2 Re for the conjugate pairs):
//   f[k0 + 64 kh + e] = sum_m Re( W[kh][m] * Q[m][e] ),
//   Q[m][e]  = A_m^e                       (e < 64)
//   W[kh][m] = 2 C_m B_m A_m^(k0 + 64 kh)  (kh < KH)
// so the N-sum becomes a small real contraction.  Per mode only five
// exactly phase-reduced powers are evaluated (fc::ssm_pow): A, A^8, A^64,
// A^512 and A^k0.  The tables A^b, A^(8b), A^(64b) (b < 8) and A^(512 a)
// (a < ceil(KH/8)) follow by at most 15 successive products, and every table
// entry is a product of at most four of them, so the relative error stays at
// a few 1e-7 whatever k is (no growth along the filter).
#pragma once

#include "common.cuh"

namespace fc {

__host__ __device__ constexpr int ssm_scratch_per_mode(int KH) { return 29 + (KH + 7) / 8; }

// Fill the tables for modes m0 .. m0+mb-1 of channel h.  Q: [m][64] (stride
// 64), W: [kh][MBS] (stride MBS >= mb), X: scratch of mb * ssm_scratch_per_mode(KH).
// All threads of the block (nthr) take part; ends with a __syncthreads().
// X per mode: [0..4] exact A, A^8, A^64, A^512, A^k0 | [5..12] A^b | [13..20] A^(8b)
//             | [21..28] A^(64b) | [29..] A^(512 a)
__device__ __forceinline__ void ssm_fill_tables(const float* __restrict__ dt, const float2* __restrict__ lam,
                                                const float2* __restrict__ Bp, const float2* __restrict__ Cp,
                                                int h, int N, int m0, int mb, int MBS, long long k0, int KH,
                                                float2* Q, float2* W, float2* X, int tid, int nthr) {
  const int KH8 = (KH + 7) / 8;
  const int XS = ssm_scratch_per_mode(KH);
  const float d = dt[h];
  for (int idx = tid; idx < mb * 5; idx += nthr) {
    const int m = idx / 5, s = idx - m * 5;
    const float2 lm = lam[(size_t)h * N + m0 + m];
    const double k = s == 0 ? 1.0 : s == 1 ? 8.0 : s == 2 ? 64.0 : s == 3 ? 512.0 : (double)k0;
    X[m * XS + s] = ssm_pow(d, lm.x, lm.y, k);
  }
  __syncthreads();
  for (int idx = tid; idx < mb * 4; idx += nthr) {  // four power chains per mode
    const int m = idx >> 2, c = idx & 3;
    float2* xm = X + m * XS;
    const float2 base = xm[c];
    const int len = c < 3 ? 8 : KH8;
    float2* out = xm + 5 + 8 * c;
    float2 p = make_float2(1.f, 0.f);
    for (int i = 0; i < len; ++i) {
      out[i] = p;
      p = cmul(p, base);
    }
  }
  __syncthreads();
  for (int idx = tid; idx < mb * 64; idx += nthr) {
    const int m = idx >> 6, e = idx & 63;
    Q[m * 64 + e] = cmul(X[m * XS + 13 + (e >> 3)], X[m * XS + 5 + (e & 7)]);
  }
  for (int idx = tid; idx < KH * mb; idx += nthr) {
    const int kh = idx / mb, m = idx - kh * mb;
    const size_t pm = (size_t)h * N + m0 + m;
    const float2 c = cmul(Cp[pm], Bp[pm]);
    const float2* xm = X + m * XS;
    const float2 p = cmul(cmul(xm[4], xm[29 + (kh >> 3)]), xm[21 + (kh & 7)]);
    const float2 w = cmul(c, p);
    W[kh * MBS + m] = make_float2(2.f * w.x, 2.f * w.y);
  }
  __syncthreads();
}

}  // namespace fc
