// Gradient of the causal FFT convolution with respect to the filter and D
// (the weight half of the backward pass; the input gradient is the forward
// kernel run with the conjugate filter spectrum).
//
// H3 summary, appendix C.1 "Backward Pass": the backward of the FFT
// convolution is again computed with FFTs, with conjugate transforms.  For
// y = f * u + D u and an upstream gradient dy:
//   df[h,k] = sum_b sum_{t>=k} dy[b,h,t] u[b,h,t-k]      (k < L)
//   dD[h]   = sum_b sum_t dy[b,h,t] u[b,h,t]
// With both sequences zero-padded to M = 2L, df is the circular correlation
//   df = IFFT( sum_b DY_b . conj(U_b) )  cropped to k < L
// (a lag k >= 0 never wraps for t, t - k in [0, L)).  Rows shorter than the
// transform half-length (L < M/2, any L) are read with zeros past L.
//
// One group of TG threads owns a channel and walks its B rows.  Each row's u
// and dy are packed as one complex sequence z = u + i dy, so one FFT gives
// both spectra: with Zc[m] = conj(Z[M - m]),  U = (Z + Zc) / 2 and
// DY = (Z - Zc) / (2i).  The product spectrum P = sum_b DY conj(U) is
// Hermitian, so each thread accumulates only the bins of its lower half
// (r <= RL/2 in the last-stage layout) and the rest is filled in from the
// mirror bins before the one inverse FFT per channel.  dD is summed in the
// time domain while the rows are loaded.
#include "fftconv_impl.cuh"

namespace fc {

template <typename T, int LOGM>
__global__ void __launch_bounds__(ConvGeom<LOGM>::THREADS, ConvGeom<LOGM>::MINB)
    fftconv_df_kernel(const T* __restrict__ dy, const T* __restrict__ u, float* __restrict__ df,
                      float* __restrict__ dD, int B, int H, int Lv) {
  using P = FftPlan<LOGM>;
  using Gm = ConvGeom<LOGM>;
  constexpr int M = P::M, TG = P::TG, RM = P::RMAX, R0 = P::R0, RL = P::RLAST;
  constexpr int L = M / 2;
  constexpr int PER0 = RM / R0, PERL = RM / RL;
  constexpr int HALF = RL / 2 + 1;  // accumulated bins per last-stage DFT (r <= RL/2)
  constexpr int SH = Gm::SH;
  extern __shared__ float2 smem[];
  const int g = threadIdx.x / TG;
  const int tid = threadIdx.x - g * TG;
  float2* buf = smem + (size_t)g * (Gm::BUF + Gm::FH);
  float2* tw = smem + (size_t)Gm::G * (Gm::BUF + Gm::FH);
  for (int j = threadIdx.x; j < P::TWN; j += Gm::THREADS) {
    float sn, cs;
    sincospif(-2.0f * (float)j / (float)M, &sn, &cs);
    tw[j] = make_float2(cs, sn);
  }
  const int h = blockIdx.x * Gm::G + g;
  const bool gv = h < H;
  __syncthreads();

  float2 acc[PERL * HALF];
#pragma unroll
  for (int k = 0; k < PERL * HALF; ++k) acc[k] = make_float2(0.f, 0.f);
  float dsum = 0.f;
  float2 v[RM];
  for (int b = 0; b < B; ++b) {  // every group runs B rows: the barriers stay uniform
    const size_t row = ((size_t)b * H + (gv ? h : 0)) * (size_t)Lv;
#pragma unroll
    for (int i = 0; i < PER0; ++i) {
      const int j = tid + i * TG;
#pragma unroll
      for (int r = 0; r < R0; ++r) {
        const int n = j + r * (M / R0);
        float2 z = make_float2(0.f, 0.f);
        if (r < R0 / 2 && gv && n < Lv) {
          z = make_float2(IO<T>::ld(u + row + n), IO<T>::ld(dy + row + n));
          dsum = fmaf(z.x, z.y, dsum);
        }
        v[i * R0 + r] = z;
      }
    }
    fft_fwd<LOGM>(v, buf, tid, tw);
    __syncthreads();  // the transform's last reads of buf are done
#pragma unroll
    for (int i = 0; i < PERL; ++i) {
      const int j = tid + i * TG;
#pragma unroll
      for (int r = 0; r < RL; ++r) buf[padix<SH>(j + r * (M / RL))] = v[i * RL + r];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < PERL; ++i) {
      const int j = tid + i * TG;
#pragma unroll
      for (int r = 0; r < HALF; ++r) {
        const int m = j + r * (M / RL);
        const float2 Z = v[i * RL + r];
        const float2 Zc = cconj(buf[padix<SH>((M - m) & (M - 1))]);
        const float2 Uf = make_float2(0.5f * (Z.x + Zc.x), 0.5f * (Z.y + Zc.y));
        // (Z - Zc) / (2i) = (Im(Z - Zc) - i Re(Z - Zc)) / 2
        const float2 Df = make_float2(0.5f * (Z.y - Zc.y), -0.5f * (Z.x - Zc.x));
        acc[i * HALF + r] = cadd(acc[i * HALF + r], cmul(Df, cconj(Uf)));
      }
    }
    __syncthreads();  // mirror reads done before the next row's transform writes buf
  }
  // full Hermitian spectrum (scaled by 1/M) in the last-stage layout, then one inverse FFT
  constexpr float inv_m = 1.0f / (float)M;
#pragma unroll
  for (int i = 0; i < PERL; ++i) {
    const int j = tid + i * TG;
#pragma unroll
    for (int r = 0; r < HALF; ++r) buf[padix<SH>(j + r * (M / RL))] = acc[i * HALF + r];
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < PERL; ++i) {
    const int j = tid + i * TG;
#pragma unroll
    for (int r = 0; r < RL; ++r) {
      const int m = j + r * (M / RL);
      const float2 p = r < HALF ? acc[i * HALF + (r < HALF ? r : 0)] : cconj(buf[padix<SH>((M - m) & (M - 1))]);
      v[i * RL + r] = make_float2(p.x * inv_m, p.y * inv_m);
    }
  }
  __syncthreads();
  fft_inv<LOGM>(v, buf, tid, tw);
  if (gv) {
    float* dfh = df + (size_t)h * Lv;
#pragma unroll
    for (int i = 0; i < PER0; ++i) {
      const int j = tid + i * TG;
#pragma unroll
      for (int r = 0; r < R0 / 2; ++r)
        if (j + r * (M / R0) < Lv) dfh[j + r * (M / R0)] = v[i * R0 + r].x;
    }
  }
  // dD: reduce dsum over the group's TG threads
  constexpr int W = TG < 32 ? TG : 32;
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o, W);
  if constexpr (TG > 32) {
    __syncthreads();
    float* red = reinterpret_cast<float*>(buf);
    if ((tid & 31) == 0) red[tid >> 5] = dsum;
    __syncthreads();
    if (tid == 0) {
      float s = 0.f;
      for (int w = 0; w < TG / 32; ++w) s += red[w];
      if (gv) dD[h] = s;
    }
  } else {
    if (tid == 0 && gv) dD[h] = dsum;
  }
}

template <typename T, int LOGM>
static cudaError_t launch_df_t(const void* dy, const void* u, float* df, float* dD, int B, int H, int Lv,
                               cudaStream_t st) {
  using Gm = ConvGeom<LOGM>;
  const size_t smem = Gm::smem_bytes;
  if (smem > 48 * 1024) {
    cudaError_t e = smem_optin<fftconv_df_kernel<T, LOGM>>(smem);
    if (e != cudaSuccess) return e;
  }
  const unsigned grid = (unsigned)((H + Gm::G - 1) / Gm::G);
  fftconv_df_kernel<T, LOGM><<<grid, Gm::THREADS, smem, st>>>((const T*)dy, (const T*)u, df, dD, B, H, Lv);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_df_dispatch(const void* dy, const void* u, float* df, float* dD, int B, int H, int L,
                                      cudaStream_t st) {
  int Lc = 16;
  while (Lc < L) Lc <<= 1;
  switch (Lc) {
    case 16: return launch_df_t<T, 5>(dy, u, df, dD, B, H, L, st);
    case 32: return launch_df_t<T, 6>(dy, u, df, dD, B, H, L, st);
    case 64: return launch_df_t<T, 7>(dy, u, df, dD, B, H, L, st);
    case 128: return launch_df_t<T, 8>(dy, u, df, dD, B, H, L, st);
    case 256: return launch_df_t<T, 9>(dy, u, df, dD, B, H, L, st);
    case 512: return launch_df_t<T, 10>(dy, u, df, dD, B, H, L, st);
    case 1024: return launch_df_t<T, 11>(dy, u, df, dD, B, H, L, st);
    case 2048: return launch_df_t<T, 12>(dy, u, df, dD, B, H, L, st);
    case 4096: return launch_df_t<T, 13>(dy, u, df, dD, B, H, L, st);
    case 8192: return launch_df_t<T, 14>(dy, u, df, dD, B, H, L, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fftconv_dfilter(const void* dy, const void* u, float* df, float* dD, int B, int H, int L,
                                   int dtype, cudaStream_t st) {
  switch (dtype) {
    case 0: return launch_df_dispatch<float>(dy, u, df, dD, B, H, L, st);
    case 1: return launch_df_dispatch<__half>(dy, u, df, dD, B, H, L, st);
    case 2: return launch_df_dispatch<__nv_bfloat16>(dy, u, df, dD, B, H, L, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fc
