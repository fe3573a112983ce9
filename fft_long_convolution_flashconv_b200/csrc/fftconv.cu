// Fused FFT causal convolution (A2-A4): one kernel does zero-pad -> FFT ->
// multiply by the filter spectrum -> inverse FFT -> crop -> + D u, with the
// whole 2L-point sequence kept on chip (H3 summary section 4 "Short-sequence
// computation": FFT, pointwise multiply and inverse FFT fused in one kernel
// so the sequence does not round-trip through HBM).
//
// Layout of the work:
//  * A group of TG threads owns one channel h.  It first transforms the
//    filter f[h] and keeps the Hermitian half of its spectrum (scaled by
//    1/M) in shared memory, then walks over the channel's rows two at a
//    time: rows q0 and q1 are packed as one complex sequence
//    z = u[q0] + i u[q1].  Because f is real, conv(z, f) = conv(u0, f) +
//    i conv(u1, f), so one complex 2L-point FFT convolution yields both
//    rows (no real-FFT post-processing pass is needed).
//  * u is read straight from global memory into the first radix stage's
//    registers (the zero-padded half is never loaded); y is written straight
//    from the last inverse stage's registers (the discarded half is never
//    computed into memory).
//  * The same kernel serves the chunk convolutions of state passing: a
//    "row" is then a chunk of length T of a longer sequence.
#include "fft_stockham.cuh"
#include "kernels.cuh"

namespace fc {

template <int LOGM>
struct ConvGeom {
  using P = FftPlan<LOGM>;
  static constexpr int M = P::M;
  static constexpr int TG = P::TG;
  static constexpr int G = TG >= 128 ? 1 : 128 / TG;  // channel groups per CTA
  static constexpr int SH = ILog2<P::R0>::v;
  static constexpr int BUF = M + (M >> SH);
  static constexpr int FH = M / 2 + 1;
  static constexpr size_t smem_bytes = sizeof(float2) * ((size_t)G * (BUF + FH) + P::TWN);
  static constexpr int THREADS = G * TG;
  // blocks per SM the register budget must allow (<= 128 registers a thread)
  static constexpr int MINB = THREADS >= 512 ? 1 : 512 / THREADS;
};

// Forward FFT; v holds the stage-0 inputs on entry and the spectrum (last-stage
// layout: DFT j holds bins j + r*M/RLAST) on exit.
template <int LOGM>
__device__ __forceinline__ void fft_fwd(float2* v, float2* buf, int tid, const float2* tw) {
  using P = FftPlan<LOGM>;
  using Gm = ConvGeom<LOGM>;
  constexpr int M = P::M, TG = P::TG, RM = P::RMAX, SH = Gm::SH;
  using S0 = Stage<M, P::R0, 1, TG, RM, SH>;
  using S1 = Stage<M, P::R1, P::R0, TG, RM, SH>;
  S0::template compute<-1>(v, tid, tw);
  __syncthreads();
  S0::store(buf, v, tid);
  __syncthreads();
  S1::load(buf, v, tid);
  S1::template compute<-1>(v, tid, tw);
  if constexpr (P::NST == 3) {
    using S2 = Stage<M, P::R2, P::R0 * P::R1, TG, RM, SH>;
    __syncthreads();
    S1::store(buf, v, tid);
    __syncthreads();
    S2::load(buf, v, tid);
    S2::template compute<-1>(v, tid, tw);
  }
}

// Inverse FFT (stages in reverse radix order); v holds the product spectrum in
// the forward last-stage layout on entry, and on exit DFT j holds outputs
// j + r*M/R0 (the positions the forward stage 0 loaded).
template <int LOGM>
__device__ __forceinline__ void fft_inv(float2* v, float2* buf, int tid, const float2* tw) {
  using P = FftPlan<LOGM>;
  using Gm = ConvGeom<LOGM>;
  constexpr int M = P::M, TG = P::TG, RM = P::RMAX, SH = Gm::SH;
  if constexpr (P::NST == 3) {
    using I0 = Stage<M, P::R2, 1, TG, RM, SH>;
    using I1 = Stage<M, P::R1, P::R2, TG, RM, SH>;
    using I2 = Stage<M, P::R0, P::R2 * P::R1, TG, RM, SH>;
    I0::template compute<+1>(v, tid, tw);
    __syncthreads();
    I0::store(buf, v, tid);
    __syncthreads();
    I1::load(buf, v, tid);
    I1::template compute<+1>(v, tid, tw);
    __syncthreads();
    I1::store(buf, v, tid);
    __syncthreads();
    I2::load(buf, v, tid);
    I2::template compute<+1>(v, tid, tw);
  } else {
    using I0 = Stage<M, P::R1, 1, TG, RM, SH>;
    using I1 = Stage<M, P::R0, P::R1, TG, RM, SH>;
    I0::template compute<+1>(v, tid, tw);
    __syncthreads();
    I0::store(buf, v, tid);
    __syncthreads();
    I1::load(buf, v, tid);
    I1::template compute<+1>(v, tid, tw);
  }
}

// u, y: rows of a B x H x Lrow array; each row holds C chunks of length
// Lc = M/2 (C = 1 for a plain convolution).  Sub-row q in [0, B*C) of
// channel h starts at ((q / C) * H + h) * Lrow + (q % C) * Lc.
// f: filter of channel h at f + h * fstride (Lc taps used).
template <typename T, int LOGM>
__global__ void __launch_bounds__(ConvGeom<LOGM>::THREADS, ConvGeom<LOGM>::MINB)
    fftconv_kernel(const T* __restrict__ u, const float* __restrict__ f, int fstride,
                   const float* __restrict__ D, T* __restrict__ y, int B, int H, long long Lrow, int C) {
  using P = FftPlan<LOGM>;
  using Gm = ConvGeom<LOGM>;
  constexpr int M = P::M, TG = P::TG, RM = P::RMAX, R0 = P::R0, RL = P::RLAST;
  constexpr int Lc = M / 2;
  constexpr int PER0 = RM / R0, PERL = RM / RL;
  extern __shared__ float2 smem[];
  const int g = threadIdx.x / TG;
  const int tid = threadIdx.x - g * TG;
  float2* buf = smem + (size_t)g * (Gm::BUF + Gm::FH);
  float2* fh = buf + Gm::BUF;
  float2* tw = smem + (size_t)Gm::G * (Gm::BUF + Gm::FH);
  for (int j = threadIdx.x; j < P::TWN; j += Gm::THREADS) {
    float sn, cs;
    sincospif(-2.0f * (float)j / (float)M, &sn, &cs);
    tw[j] = make_float2(cs, sn);
  }
  __syncthreads();
  const int h = blockIdx.x * Gm::G + g;
  const bool hv = h < H;
  float2 v[RM];

  // ---- spectrum of the zero-padded filter (once per channel)
  {
    const float* fr = f + (size_t)(hv ? h : 0) * fstride;
#pragma unroll
    for (int i = 0; i < PER0; ++i) {
      const int j = tid + i * TG;
#pragma unroll
      for (int r = 0; r < R0; ++r)
        v[i * R0 + r] = (r < R0 / 2 && hv && FC_OK_IDX(10, (long long)h * fstride + j + r * (M / R0), (long long)H * fstride))
                            ? make_float2(__ldg(fr + j + r * (M / R0)), 0.f)
                            : make_float2(0.f, 0.f);
    }
    fft_fwd<LOGM>(v, buf, tid, tw);
    constexpr float inv_m = 1.0f / (float)M;
#pragma unroll
    for (int i = 0; i < PERL; ++i) {
      const int j = tid + i * TG;
#pragma unroll
      for (int r = 0; r < RL; ++r) {
        const int m = j + r * (M / RL);
        if (m <= M / 2) fh[m] = make_float2(v[i * RL + r].x * inv_m, v[i * RL + r].y * inv_m);
      }
    }
  }
  const float dh = hv ? D[h] : 0.f;
  const int Q = B * C;
  for (int p = 0; p < (Q + 1) / 2; ++p) {
    const int q0 = 2 * p, q1 = 2 * p + 1;
    const bool has1 = q1 < Q;
    const size_t o0 = ((size_t)(q0 / C) * H + (hv ? h : 0)) * (size_t)Lrow + (size_t)(q0 % C) * Lc;
    const size_t o1 = has1 ? ((size_t)(q1 / C) * H + (hv ? h : 0)) * (size_t)Lrow + (size_t)(q1 % C) * Lc : o0;
    const T* u0 = u + o0;
    const T* u1 = u + o1;
#pragma unroll
    for (int i = 0; i < PER0; ++i) {
      const int j = tid + i * TG;
#pragma unroll
      for (int r = 0; r < R0; ++r) {
        const int n = j + r * (M / R0);
        float2 z = make_float2(0.f, 0.f);
        if (r < R0 / 2 && hv && FC_OK_IDX(11, o0 + n, (long long)B * H * Lrow) &&
            FC_OK_IDX(12, o1 + n, (long long)B * H * Lrow)) {
          z.x = IO<T>::ld(u0 + n);
          z.y = has1 ? IO<T>::ld(u1 + n) : 0.f;
        }
        v[i * R0 + r] = z;
      }
    }
    fft_fwd<LOGM>(v, buf, tid, tw);
    // pointwise product with the filter spectrum (Hermitian: F[M-m] = conj F[m])
#pragma unroll
    for (int i = 0; i < PERL; ++i) {
      const int j = tid + i * TG;
#pragma unroll
      for (int r = 0; r < RL; ++r) {
        const int m = j + r * (M / RL);
        const float2 F = (m <= M / 2) ? fh[m] : cconj(fh[M - m]);
        v[i * RL + r] = cmul(v[i * RL + r], F);
      }
    }
    fft_inv<LOGM>(v, buf, tid, tw);
    if (hv) {
      T* y0 = y + o0;
      T* y1 = y + o1;
#pragma unroll
      for (int i = 0; i < PER0; ++i) {
        const int j = tid + i * TG;
#pragma unroll
        for (int r = 0; r < R0 / 2; ++r) {
          const int n = j + r * (M / R0);
          if (!FC_OK_IDX(13, o0 + n, (long long)B * H * Lrow) || !FC_OK_IDX(14, o1 + n, (long long)B * H * Lrow))
            continue;
          IO<T>::st(y0 + n, fmaf(dh, IO<T>::ld(u0 + n), v[i * R0 + r].x));
          if (has1) IO<T>::st(y1 + n, fmaf(dh, IO<T>::ld(u1 + n), v[i * R0 + r].y));
        }
      }
    }
  }
}

template <typename T, int LOGM>
static cudaError_t launch_fftconv_t(const T* u, const float* f, int fstride, const float* D, T* y, int B, int H,
                                    long long Lrow, int C, cudaStream_t st) {
  using Gm = ConvGeom<LOGM>;
  auto kern = fftconv_kernel<T, LOGM>;
  const size_t smem = Gm::smem_bytes;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int grid = (H + Gm::G - 1) / Gm::G;
  kern<<<grid, Gm::G * FftPlan<LOGM>::TG, smem, st>>>(u, f, fstride, D, y, B, H, Lrow, C);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_fftconv_dispatch(const T* u, const float* f, int fstride, const float* D, T* y, int B,
                                           int H, long long Lrow, int Lc, int C, cudaStream_t st) {
  switch (Lc) {
    case 16: return launch_fftconv_t<T, 5>(u, f, fstride, D, y, B, H, Lrow, C, st);
    case 32: return launch_fftconv_t<T, 6>(u, f, fstride, D, y, B, H, Lrow, C, st);
    case 64: return launch_fftconv_t<T, 7>(u, f, fstride, D, y, B, H, Lrow, C, st);
    case 128: return launch_fftconv_t<T, 8>(u, f, fstride, D, y, B, H, Lrow, C, st);
    case 256: return launch_fftconv_t<T, 9>(u, f, fstride, D, y, B, H, Lrow, C, st);
    case 512: return launch_fftconv_t<T, 10>(u, f, fstride, D, y, B, H, Lrow, C, st);
    case 1024: return launch_fftconv_t<T, 11>(u, f, fstride, D, y, B, H, Lrow, C, st);
    case 2048: return launch_fftconv_t<T, 12>(u, f, fstride, D, y, B, H, Lrow, C, st);
    case 4096: return launch_fftconv_t<T, 13>(u, f, fstride, D, y, B, H, Lrow, C, st);
    case 8192: return launch_fftconv_t<T, 14>(u, f, fstride, D, y, B, H, Lrow, C, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fftconv(const void* u, const float* f, int fstride, const float* D, void* y, int B, int H,
                           long long Lrow, int Lc, int C, int dtype, cudaStream_t st) {
  switch (dtype) {
    case 0:
      return launch_fftconv_dispatch<float>((const float*)u, f, fstride, D, (float*)y, B, H, Lrow, Lc, C, st);
    case 1:
      return launch_fftconv_dispatch<__half>((const __half*)u, f, fstride, D, (__half*)y, B, H, Lrow, Lc, C, st);
    case 2:
      return launch_fftconv_dispatch<__nv_bfloat16>((const __nv_bfloat16*)u, f, fstride, D, (__nv_bfloat16*)y, B,
                                                    H, Lrow, Lc, C, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fc

FC_CHECK_READER(fc_check_fftconv)
