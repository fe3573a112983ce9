// H3 mixer forward (A10-A11), CUDA-core version.
//
// H3 blog "The Solution, Part 1": O = Q (.) SSM_diag(SSM_shift(K) (.) V);
// H3 summary appendix D.2 "H3 Complexity" (heads, head dimension O(1)).
// Per head, with k~ the shift-SSM output, the diagonal-SSM convolution of the
// kv outer product contracted with q rearranges exactly into a causal,
// Toeplitz-weighted product (no 64x64-channel intermediate is ever formed):
//   o_j[t] = sum_{s<=t} (f_h[t-s] + D_h [s==t]) (q_t . k~_s) v_s[j]
// One CTA owns a 64-row tile of t for one (batch, head) and sweeps the s
// tiles s <= t: S = Q K~^T (64x64, K = head_dim), P = S (.) Toeplitz(f),
// O += P V.  The shift SSM (k~[s,c] = sum_j Cshift[c,j] k[s-j,c]) is applied
// while the K tile is loaded.
#include "kernels.cuh"

namespace fc {

constexpr int kMixHD = 64;   // head_dim (only size built)
constexpr int kMixT = 64;    // tile rows (t and s)
constexpr int kMixLd = 68;   // padded leading dimension (floats), rows 16-byte aligned
constexpr int kMixThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kMixThreads) h3_mixer_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                                const T* __restrict__ v,
                                                                const float* __restrict__ Cshift,
                                                                const float* __restrict__ fdiag,
                                                                const float* __restrict__ D, T* __restrict__ o,
                                                                int L, int heads, int S) {
  extern __shared__ __align__(16) float msm[];
  float* Qt = msm;                       // [i][t]
  float* Kt = Qt + kMixHD * kMixLd;      // [i][s]
  float* Vs = Kt + kMixHD * kMixLd;      // [s][j]
  float* Ps = Vs + kMixT * kMixLd;       // [t][s]
  float* fs = Ps + kMixT * kMixLd;       // 128 filter taps around the diagonal
  const int tt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int dm = heads * kMixHD;
  const int t0 = tt * kMixT;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const size_t bbase = (size_t)b * L * dm + (size_t)h * kMixHD;

  for (int idx = tid; idx < kMixT * kMixHD; idx += kMixThreads) {
    const int r = idx >> 6, i = idx & 63;
    const int t = t0 + r;
    Qt[i * kMixLd + r] = t < L ? IO<T>::ld(q + bbase + (size_t)t * dm + i) : 0.f;
  }
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
  const float dh = D[h];
  const float* fh = fdiag + (size_t)h * L;

  for (int st = 0; st <= tt; ++st) {
    const int s0 = st * kMixT;
    __syncthreads();  // previous tile's readers are done
    for (int idx = tid; idx < kMixT * kMixHD; idx += kMixThreads) {
      const int r = idx >> 6, i = idx & 63;
      const int s = s0 + r;
      const int c = h * kMixHD + i;
      float kt = 0.f, vv = 0.f;
      if (s < L) {
        for (int j = 0; j < S && j <= s; ++j)
          kt = fmaf(Cshift[(size_t)c * S + j], IO<T>::ld(k + bbase + (size_t)(s - j) * dm + i), kt);
        vv = IO<T>::ld(v + bbase + (size_t)s * dm + i);
      }
      Kt[i * kMixLd + r] = kt;
      Vs[r * kMixLd + i] = vv;
    }
    if (tid < 2 * kMixT) {
      // fs[x] = weight for t - s = x - 63 + (t0 - s0)
      const int d = tid - (kMixT - 1) + (t0 - s0);
      float w = (d >= 0 && d < L) ? fh[d] : 0.f;
      if (d == 0) w += dh;
      fs[tid] = w;
    }
    __syncthreads();
    // S = Q K~^T  (rows t = ty*4+a, cols s = tx*4+c)
    float sacc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) sacc[a][c] = 0.f;
#pragma unroll 8
    for (int i = 0; i < kMixHD; ++i) {
      const float4 qa = *reinterpret_cast<const float4*>(Qt + i * kMixLd + ty * 4);
      const float4 kb = *reinterpret_cast<const float4*>(Kt + i * kMixLd + tx * 4);
      const float qv[4] = {qa.x, qa.y, qa.z, qa.w};
      const float kv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) sacc[a][c] = fmaf(qv[a], kv[c], sacc[a][c]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      float4 pw;
      float* pp = &pw.x;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int dl = (ty * 4 + a) - (tx * 4 + c);  // local t - s in [-63, 63]
        pp[c] = sacc[a][c] * fs[dl + kMixT - 1];
      }
      *reinterpret_cast<float4*>(Ps + (ty * 4 + a) * kMixLd + tx * 4) = pw;
    }
    __syncthreads();
    // O += P V  (rows t = ty*4+a, cols j = tx*4+c)
#pragma unroll 8
    for (int s = 0; s < kMixT; ++s) {
      const float4 vb = *reinterpret_cast<const float4*>(Vs + s * kMixLd + tx * 4);
      const float vv[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float p = Ps[(ty * 4 + a) * kMixLd + s];
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(p, vv[c], acc[a][c]);
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int t = t0 + ty * 4 + a;
    if (t < L) {
#pragma unroll
      for (int c = 0; c < 4; ++c) IO<T>::st(o + bbase + (size_t)t * dm + tx * 4 + c, acc[a][c]);
    }
  }
}

template <typename T>
static cudaError_t mixer_t(const void* q, const void* k, const void* v, const float* Cs, const float* f,
                           const float* D, void* o, int B, int L, int heads, int S, cudaStream_t st) {
  const size_t smem = sizeof(float) * ((size_t)2 * kMixHD * kMixLd + (size_t)2 * kMixT * kMixLd + 2 * kMixT);
  auto kern = h3_mixer_kernel<T>;
  cudaError_t e = smem_optin<h3_mixer_kernel<T>>(smem);
  if (e != cudaSuccess) return e;
  dim3 grid((L + kMixT - 1) / kMixT, heads, B);
  kern<<<grid, kMixThreads, smem, st>>>((const T*)q, (const T*)k, (const T*)v, Cs, f, D, (T*)o, L, heads, S);
  return cudaGetLastError();
}

cudaError_t launch_h3_mixer(const void* q, const void* k, const void* v, const float* Cshift, const float* fdiag,
                            const float* D, void* o, int B, int L, int heads, int shift_len, int dtype,
                            cudaStream_t st) {
  switch (dtype) {
    case 0: return mixer_t<float>(q, k, v, Cshift, fdiag, D, o, B, L, heads, shift_len, st);
    case 1: return mixer_t<__half>(q, k, v, Cshift, fdiag, D, o, B, L, heads, shift_len, st);
    case 2: return mixer_t<__nv_bfloat16>(q, k, v, Cshift, fdiag, D, o, B, L, heads, shift_len, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fc
