// Recurrent (token-by-token) evaluation for generation.
//
// H3 summary, section 2 "Recurrent view": an SSM computes each output from
// the current state, x_t = A x_{t-1} + B u_t, y_t = C x_t + D u_t, so the
// next token needs O(N) work and no history (2 Re for the conjugate pairs of
// the complex diagonal SSM); section 5: this is where H3's faster generation
// comes from.  The H3 layer in recurrent form (H3 blog, "The Solution,
// Part 1") keeps two states per head: the shift SSM's last S-1 keys (a ring
// buffer) and the diagonal SSM's state over the head's hd x hd key-value
// channels, N complex modes each.
//
//   ssm_decode_kernel   one (b, h) row per group of 32*W threads; T steps in
//                       order with the state in registers
//   h3_decode_kernel    one block per (b, head, output channel j)
//
// Both are memory-bound on the state; A = exp(dt lambda) is recomputed per
// mode with the exactly phase-reduced power (no scratch).
#include "kernels.cuh"

namespace fc {

// T steps of x <- A x + B u_t, y_t = 2 Re(C . x) + D u_t for one (b, h) row
// per 32*W threads (W warps), MPL modes per thread (n = tid_in_row + 32 W m).
template <typename T, int MPL, int W>
__global__ void __launch_bounds__(128) ssm_decode_kernel(const T* __restrict__ u, float2* __restrict__ x,
                                                         const float* __restrict__ dt, const float2* __restrict__ lam,
                                                         const float2* __restrict__ Bp, const float2* __restrict__ Cp,
                                                         const float* __restrict__ D, T* __restrict__ y, int B, int H,
                                                         int N, int Tn) {
  constexpr int RPB = 4 / W;  // rows per block
  __shared__ float red[4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rloc = warp / W, wr = warp % W;
  const long long row = (long long)blockIdx.x * RPB + rloc;
  const bool rv = row < (long long)B * H;
  const int h = rv ? (int)(row % H) : 0;
  const int t0 = wr * 32 + lane;
  float2 a[MPL], bb[MPL], cc[MPL], xs[MPL];
  const float d = dt[h];
#pragma unroll
  for (int m = 0; m < MPL; ++m) {
    const int n = t0 + 32 * W * m;
    a[m] = bb[m] = cc[m] = xs[m] = make_float2(0.f, 0.f);
    if (rv && n < N) {
      const float2 l = lam[(size_t)h * N + n];
      a[m] = ssm_pow(d, l.x, l.y, 1.0);
      bb[m] = Bp[(size_t)h * N + n];
      cc[m] = Cp[(size_t)h * N + n];
      xs[m] = x[(size_t)row * N + n];
    }
  }
  const float dh = rv ? D[h] : 0.f;
  for (int t = 0; t < Tn; ++t) {
    const float ut = rv ? IO<T>::ldplain(u + (size_t)row * Tn + t) : 0.f;
    float acc = 0.f;
#pragma unroll
    for (int m = 0; m < MPL; ++m) {
      const float2 ax = cmul(a[m], xs[m]);
      xs[m] = make_float2(fmaf(bb[m].x, ut, ax.x), fmaf(bb[m].y, ut, ax.y));
      acc = fmaf(cc[m].x, xs[m].x, fmaf(-cc[m].y, xs[m].y, acc));  // Re(C x)
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if constexpr (W > 1) {
      if (lane == 0) red[warp] = acc;
      __syncthreads();
      acc = 0.f;
#pragma unroll
      for (int w = 0; w < W; ++w) acc += red[rloc * W + w];
      __syncthreads();
    }
    if (rv && wr == 0 && lane == 0) IO<T>::st(y + (size_t)row * Tn + t, fmaf(dh, ut, 2.f * acc));
  }
#pragma unroll
  for (int m = 0; m < MPL; ++m) {
    const int n = t0 + 32 * W * m;
    if (rv && n < N) x[(size_t)row * N + n] = xs[m];
  }
}

template <typename T, int MPL, int W>
static cudaError_t decode_t(const void* u, float* x, const float* dt, const float* lam, const float* Bp,
                            const float* Cp, const float* D, void* y, int B, int H, int N, int Tn, cudaStream_t st) {
  constexpr int RPB = 4 / W;
  const long long rows = (long long)B * H;
  const unsigned grid = (unsigned)((rows + RPB - 1) / RPB);
  ssm_decode_kernel<T, MPL, W><<<grid, 128, 0, st>>>((const T*)u, (float2*)x, dt, (const float2*)lam,
                                                      (const float2*)Bp, (const float2*)Cp, D, (T*)y, B, H, N, Tn);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t decode_dispatch(const void* u, float* x, const float* dt, const float* lam, const float* Bp,
                                   const float* Cp, const float* D, void* y, int B, int H, int N, int Tn,
                                   cudaStream_t st) {
  if (N <= 32) return decode_t<T, 1, 1>(u, x, dt, lam, Bp, Cp, D, y, B, H, N, Tn, st);
  if (N <= 64) return decode_t<T, 2, 1>(u, x, dt, lam, Bp, Cp, D, y, B, H, N, Tn, st);
  if (N <= 128) return decode_t<T, 4, 1>(u, x, dt, lam, Bp, Cp, D, y, B, H, N, Tn, st);
  if (N <= 256) return decode_t<T, 8, 1>(u, x, dt, lam, Bp, Cp, D, y, B, H, N, Tn, st);
  if (N <= 512) return decode_t<T, 8, 2>(u, x, dt, lam, Bp, Cp, D, y, B, H, N, Tn, st);
  return decode_t<T, 8, 4>(u, x, dt, lam, Bp, Cp, D, y, B, H, N, Tn, st);  // N <= 1024
}

cudaError_t launch_ssm_decode(const void* u, float* x, const float* dt, const float* lam, const float* Bp,
                              const float* Cp, const float* D, void* y, int B, int H, int N, int Tn, int dtype,
                              cudaStream_t st) {
  switch (dtype) {
    case 0: return decode_dispatch<float>(u, x, dt, lam, Bp, Cp, D, y, B, H, N, Tn, st);
    case 1: return decode_dispatch<__half>(u, x, dt, lam, Bp, Cp, D, y, B, H, N, Tn, st);
    case 2: return decode_dispatch<__nv_bfloat16>(u, x, dt, lam, Bp, Cp, D, y, B, H, N, Tn, st);
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------- H3 mixer, one token
// Block (j, head, b), 256 threads = 8 warps; warp w takes key channels
// i = w, w + 8, ... < hd; lane over modes n.  state: B x heads x hd x hd x N
// complex ([b][head][i][j][n]); kring: B x (S-1) x dm keys of earlier tokens
// (slot p % (S-1) holds the key of position p).
template <typename T>
__global__ void __launch_bounds__(256) h3_decode_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                        const T* __restrict__ v, T* __restrict__ kring,
                                                        float2* __restrict__ state, const float* __restrict__ Cs,
                                                        const float* __restrict__ dt, const float2* __restrict__ lam,
                                                        const float2* __restrict__ Bp, const float2* __restrict__ Cp,
                                                        const float* __restrict__ D, T* __restrict__ o, int heads,
                                                        int hd, int N, int S, long long pos) {
  __shared__ float kt[64], qs[64], part[8];
  extern __shared__ float2 abc[];  // A, B, C of the head's modes: 3 x N complex
  const int j = blockIdx.x, head = blockIdx.y, b = blockIdx.z;
  const int dm = heads * hd;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t tok = (size_t)b * dm + (size_t)head * hd;
  // shift SSM on the head's keys: k~_i = sum_{s<S, s<=pos} Cs[c][s] k_{pos-s}[c]
  if (threadIdx.x < hd) {
    const int c = head * hd + threadIdx.x;
    float acc = Cs[(size_t)c * S] * IO<T>::ldplain(k + tok + threadIdx.x);
    for (int s = 1; s < S; ++s) {
      if ((long long)s > pos) break;
      const long long p = pos - s;
      acc = fmaf(Cs[(size_t)c * S + s], IO<T>::ldplain(kring + ((size_t)b * (S - 1) + (size_t)(p % (S - 1))) * dm + c),
                 acc);
    }
    kt[threadIdx.x] = acc;
    qs[threadIdx.x] = IO<T>::ldplain(q + tok + threadIdx.x);
  }
  const float d = dt[head];
  for (int n = threadIdx.x; n < N; n += blockDim.x) {
    const float2 l = lam[(size_t)head * N + n];
    abc[n] = ssm_pow(d, l.x, l.y, 1.0);
    abc[N + n] = Bp[(size_t)head * N + n];
    abc[2 * N + n] = Cp[(size_t)head * N + n];
  }
  __syncthreads();
  const float vj = IO<T>::ldplain(v + tok + j);
  const float dh = D[head];
  float contrib = 0.f;
  for (int i = warp; i < hd; i += 8) {
    const float kv = kt[i] * vj;
    float2* X = state + ((((size_t)b * heads + head) * hd + i) * hd + j) * (size_t)N;
    float acc = 0.f;
    for (int n = lane; n < N; n += 32) {
      const float2 a = abc[n], bn = abc[N + n], cn = abc[2 * N + n];
      const float2 ax = cmul(a, X[n]);
      const float2 xn = make_float2(fmaf(bn.x, kv, ax.x), fmaf(bn.y, kv, ax.y));
      X[n] = xn;
      acc = fmaf(cn.x, xn.x, fmaf(-cn.y, xn.y, acc));
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    contrib = fmaf(qs[i], fmaf(dh, kv, 2.f * acc), contrib);  // q_i y_ij
  }
  if (lane == 0) part[warp] = contrib;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += part[w];
    IO<T>::st(o + tok + j, s);
  }
}

// After every block of the token has read the ring, store this token's keys.
template <typename T>
__global__ void h3_ring_store_kernel(const T* __restrict__ k, T* __restrict__ kring, int Bn, int dm, int S,
                                     long long pos) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)Bn * dm) return;
  const long long b = idx / dm, c = idx - b * dm;
  kring[((size_t)b * (S - 1) + (size_t)(pos % (S - 1))) * dm + c] = k[idx];
}

template <typename T>
static cudaError_t h3_decode_t(const void* q, const void* k, const void* v, void* kring, float* state,
                               const float* Cs, const float* dt, const float* lam, const float* Bp, const float* Cp,
                               const float* D, void* o, int B, int heads, int hd, int N, int S, long long pos,
                               cudaStream_t st) {
  const size_t smem = sizeof(float2) * 3 * (size_t)N;
  if (smem > 48 * 1024) {
    cudaError_t e = smem_optin<h3_decode_kernel<T>>(smem);
    if (e != cudaSuccess) return e;
  }
  h3_decode_kernel<T><<<dim3(hd, heads, B), 256, smem, st>>>(
      (const T*)q, (const T*)k, (const T*)v, (T*)kring, (float2*)state, Cs, dt, (const float2*)lam,
      (const float2*)Bp, (const float2*)Cp, D, (T*)o, heads, hd, N, S, pos);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || S < 2) return e;
  const long long n = (long long)B * heads * hd;
  h3_ring_store_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>((const T*)k, (T*)kring, B, heads * hd, S, pos);
  return cudaGetLastError();
}

cudaError_t launch_h3_decode(const void* q, const void* k, const void* v, void* kring, float* state, const float* Cs,
                             const float* dt, const float* lam, const float* Bp, const float* Cp, const float* D,
                             void* o, int B, int heads, int hd, int N, int S, long long pos, int dtype,
                             cudaStream_t st) {
  switch (dtype) {
    case 0: return h3_decode_t<float>(q, k, v, kring, state, Cs, dt, lam, Bp, Cp, D, o, B, heads, hd, N, S, pos, st);
    case 1: return h3_decode_t<__half>(q, k, v, kring, state, Cs, dt, lam, Bp, Cp, D, o, B, heads, hd, N, S, pos, st);
    case 2:
      return h3_decode_t<__nv_bfloat16>(q, k, v, kring, state, Cs, dt, lam, Bp, Cp, D, o, B, heads, hd, N, S, pos, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fc
