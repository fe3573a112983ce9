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
#pragma once

#include <algorithm>

#include "common.cuh"
#include "fft_stockham.cuh"
#include "ssm_tables.cuh"

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

// Two rows' inputs at one stage-0 position, kept in registers from the load
// (prefetch) until the D*u term of the output.
template <typename T> struct UPair;
template <> struct UPair<float> {
  float2 v;
  __device__ __forceinline__ void load(const float* a, const float* b, bool hb) {
    v.x = __ldg(a);
    v.y = hb ? __ldg(b) : 0.f;
  }
  __device__ __forceinline__ float2 get() const { return v; }
  __device__ __forceinline__ void zero() { v = make_float2(0.f, 0.f); }
};
template <> struct UPair<__half> {
  __half2 v;
  __device__ __forceinline__ void load(const __half* a, const __half* b, bool hb) {
    v = __halves2half2(__ldg(a), hb ? __ldg(b) : __float2half_rn(0.f));
  }
  __device__ __forceinline__ float2 get() const { return __half22float2(v); }
  __device__ __forceinline__ void zero() { v = __float2half2_rn(0.f); }
};
template <> struct UPair<__nv_bfloat16> {
  __nv_bfloat162 v;
  __device__ __forceinline__ void load(const __nv_bfloat16* a, const __nv_bfloat16* b, bool hb) {
    v = __halves2bfloat162(__ldg(a), hb ? __ldg(b) : __float2bfloat16_rn(0.f));
  }
  __device__ __forceinline__ float2 get() const { return __bfloat1622float2(v); }
  __device__ __forceinline__ void zero() { v = __float2bfloat162_rn(0.f); }
};

// Mode-block size for the fused filter generation: the tables must fit in the
// FFT buffer (BUF entries) of the channel group.
template <int LOGM>
struct GenGeom {
  static constexpr int L = (1 << LOGM) / 2;
  static constexpr int KH = L >= 64 ? L / 64 : 1;
  static constexpr int per = 64 + KH + ssm_scratch_per_mode(KH);
  static constexpr int BUF = ConvGeom<LOGM>::BUF;
  static constexpr int MB = (64 * per <= BUF) ? 64 : (32 * per <= BUF) ? 32 : (16 * per <= BUF) ? 16 : 8;
  static constexpr bool ok = (L >= 1024) && (MB * per <= BUF);
};

// Flattened work: item = (channel h, pair p) with pairs p = 0 .. NP-1 of the
// channel's Q = B*C rows.  With one group per CTA (long transforms) each CTA
// takes a contiguous range of items, so the load is balanced to one item and
// the filter spectrum is recomputed only when the channel changes.  With
// several groups per CTA (short transforms) each group owns one channel.
//
// u, y: rows of a B x H x Lrow array; each row holds C chunks of length
// Lc = M/2 (C = 1 for a plain convolution).  Sub-row q in [0, B*C) of channel
// h starts at ((q / C) * H + h) * Lrow + (q % C) * Lc.  Filter: f + h*fstride
// (Lc taps), or generated from the SSM parameters when GEN.  With C = 1 a row
// may be shorter than Lc (any L <= Lc): the transform runs at Lc with the
// positions t >= L read as zeros and never stored.  The causal outputs t < L
// depend only on u and f at positions <= t, so they are exact.
template <typename T, int LOGM, bool GEN>
__global__ void __launch_bounds__(ConvGeom<LOGM>::THREADS, ConvGeom<LOGM>::MINB)
    fftconv_kernel(const T* __restrict__ u, const float* __restrict__ f, int fstride, SsmArgs sp,
                   const float* __restrict__ D, T* __restrict__ y, int B, int H, long long Lrow, int C,
                   int conj_filter) {
  using P = FftPlan<LOGM>;
  using Gm = ConvGeom<LOGM>;
  constexpr int M = P::M, TG = P::TG, RM = P::RMAX, R0 = P::R0, RL = P::RLAST;
  constexpr int Lc = M / 2;
  constexpr int PER0 = RM / R0, PERL = RM / RL;
  constexpr int NU = PER0 * (R0 / 2);  // stage-0 positions per thread holding input
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
  const int Q = B * C;
  const int NP = (Q + 1) / 2;
  long long it0, it1;
  bool gv = true;  // group owns real work
  if constexpr (Gm::G == 1) {
    const long long total = (long long)H * NP;
    it0 = (long long)blockIdx.x * total / gridDim.x;
    it1 = (long long)(blockIdx.x + 1) * total / gridDim.x;
  } else {
    const int hg = blockIdx.x * Gm::G + g;
    gv = hg < H;
    it0 = (long long)(gv ? hg : 0) * NP;
    it1 = it0 + NP;  // every group runs the same number of items (barriers stay uniform)
  }
  auto row_off = [&](int h, int q) -> size_t {
    return ((size_t)(q / C) * H + h) * (size_t)Lrow + (size_t)(q % C) * Lc;
  };
  const int Lv = (C == 1 && Lrow < Lc) ? (int)Lrow : Lc;  // valid positions of a sub-row
  auto prefetch = [&](long long it, UPair<T>* dst) {
    const int h = (int)(it / NP), p = (int)(it - (long long)h * NP);
    const int q0 = 2 * p, q1 = 2 * p + 1;
    const bool has1 = q1 < Q;
    const T* u0 = u + row_off(h, q0);
    const T* u1 = u + row_off(h, has1 ? q1 : q0);
#pragma unroll
    for (int i = 0; i < PER0; ++i) {
      const int j = tid + i * TG;
#pragma unroll
      for (int r = 0; r < R0 / 2; ++r) {
        const int n = j + r * (M / R0);
        if (gv && n < Lv && FC_OK_IDX(11, (long long)row_off(h, q0) + n, (long long)B * H * Lrow))
          dst[i * (R0 / 2) + r].load(u0 + n, u1 + n, has1);
        else
          dst[i * (R0 / 2) + r].zero();
      }
    }
  };
  __syncthreads();

  UPair<T> ucur[NU], unxt[NU];
  if (it0 < it1) prefetch(it0, ucur);
  int hcur = -1;
  float dh = 0.f;
  float2 v[RM];
  for (long long it = it0; it < it1; ++it) {
    const int h = (int)(it / NP), p = (int)(it - (long long)h * NP);
    if (it + 1 < it1) prefetch(it + 1, unxt);
    if (h != hcur) {
      // ---- spectrum of the zero-padded filter of channel h
      if constexpr (GEN) {
        using Gg = GenGeom<LOGM>;
        static_assert(Gg::ok, "fused filter generation needs L >= 1024");
        float2* Qt = buf;
        float2* Wt = Qt + Gg::MB * 64;
        float2* Xs = Wt + Gg::KH * Gg::MB;
        float acc[NU];
#pragma unroll
        for (int k = 0; k < NU; ++k) acc[k] = 0.f;
        for (int m0 = 0; m0 < sp.N; m0 += Gg::MB) {
          const int mb = min(Gg::MB, sp.N - m0);
          __syncthreads();  // buf readers (previous item / previous block) are done
          ssm_fill_tables(sp.dt, sp.lam, sp.Bp, sp.Cp, h, sp.N, m0, mb, Gg::MB, 0, Gg::KH, Qt, Wt, Xs,
                          threadIdx.x, Gm::THREADS);
          for (int m = 0; m < mb; ++m) {
#pragma unroll
            for (int i = 0; i < PER0; ++i) {
              const int j = tid + i * TG;
#pragma unroll
              for (int r = 0; r < R0 / 2; ++r) {
                const int n = j + r * (M / R0);
                const float2 q = Qt[m * 64 + (n & 63)];
                const float2 w = Wt[(n >> 6) * Gg::MB + m];
                acc[i * (R0 / 2) + r] = fmaf(w.x, q.x, fmaf(-w.y, q.y, acc[i * (R0 / 2) + r]));
              }
            }
          }
        }
#pragma unroll
        for (int i = 0; i < PER0; ++i)
#pragma unroll
          for (int r = 0; r < R0; ++r)
            v[i * R0 + r] = make_float2(r < R0 / 2 ? acc[i * (R0 / 2) + (r < R0 / 2 ? r : 0)] : 0.f, 0.f);
      } else {
        const float* fr = f + (size_t)(gv ? h : 0) * fstride;
#pragma unroll
        for (int i = 0; i < PER0; ++i) {
          const int j = tid + i * TG;
#pragma unroll
          for (int r = 0; r < R0; ++r)
            v[i * R0 + r] = (r < R0 / 2 && gv && j + r * (M / R0) < Lv &&
                             FC_OK_IDX(10, (long long)h * fstride + j + r * (M / R0), (long long)H * fstride))
                                ? make_float2(__ldg(fr + j + r * (M / R0)), 0.f)
                                : make_float2(0.f, 0.f);
        }
      }
      fft_fwd<LOGM>(v, buf, tid, tw);
      constexpr float inv_m = 1.0f / (float)M;
      // conj_filter: multiply by conj(F^) instead, i.e. correlate with f (the
      // input gradient of the convolution)
      const float im_sign = conj_filter ? -inv_m : inv_m;
#pragma unroll
      for (int i = 0; i < PERL; ++i) {
        const int j = tid + i * TG;
#pragma unroll
        for (int r = 0; r < RL; ++r) {
          const int m = j + r * (M / RL);
          if (m <= M / 2) fh[m] = make_float2(v[i * RL + r].x * inv_m, v[i * RL + r].y * im_sign);
        }
      }
      hcur = h;
      dh = gv ? D[h] : 0.f;
    }
    const int q0 = 2 * p, q1 = 2 * p + 1;
    const bool has1 = q1 < Q;
#pragma unroll
    for (int i = 0; i < PER0; ++i)
#pragma unroll
      for (int r = 0; r < R0; ++r)
        v[i * R0 + r] = r < R0 / 2 ? ucur[i * (R0 / 2) + (r < R0 / 2 ? r : 0)].get() : make_float2(0.f, 0.f);
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
    if (gv) {
      T* y0 = y + row_off(h, q0);
      T* y1 = y + row_off(h, has1 ? q1 : q0);
#pragma unroll
      for (int i = 0; i < PER0; ++i) {
        const int j = tid + i * TG;
#pragma unroll
        for (int r = 0; r < R0 / 2; ++r) {
          const int n = j + r * (M / R0);
          if (n >= Lv || !FC_OK_IDX(13, (long long)row_off(h, q0) + n, (long long)B * H * Lrow)) continue;
          const float2 uu = ucur[i * (R0 / 2) + r].get();
          IO<T>::st(y0 + n, fmaf(dh, uu.x, v[i * R0 + r].x));
          if (has1) IO<T>::st(y1 + n, fmaf(dh, uu.y, v[i * R0 + r].y));
        }
      }
    }
#pragma unroll
    for (int k = 0; k < NU; ++k) ucur[k] = unxt[k];
  }
}

// Fused-generation variants (L >= 1024), instantiated in their own translation unit.
template <typename T>
cudaError_t launch_fftconv_gen(const T* u, const float* f, int fstride, SsmArgs sp, const float* D, T* y, int B,
                               int H, long long Lrow, int Lc, int C, cudaStream_t st);

template <typename T, int LOGM, bool GEN>
static cudaError_t launch_fftconv_t(const T* u, const float* f, int fstride, SsmArgs sp, const float* D, T* y,
                                    int B, int H, long long Lrow, int C, int conj_filter, cudaStream_t st) {
  using Gm = ConvGeom<LOGM>;
  auto kern = fftconv_kernel<T, LOGM, GEN>;
  const size_t smem = Gm::smem_bytes;
  static std::atomic<int> blocks_per_sm{0};  // per instantiation; the same on every B200
  if (smem > 48 * 1024) {
    cudaError_t e = smem_optin<fftconv_kernel<T, LOGM, GEN>>(smem);
    if (e != cudaSuccess) return e;
  }
  if (blocks_per_sm.load(std::memory_order_relaxed) == 0) {
    int b = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, Gm::THREADS, smem);
    if (e != cudaSuccess) return e;
    blocks_per_sm.store(b < 1 ? 1 : b, std::memory_order_relaxed);
  }
  long long grid;
  if constexpr (Gm::G == 1) {
    const long long items = (long long)H * ((B * C + 1) / 2);
    grid = std::min<long long>(items, (long long)blocks_per_sm.load(std::memory_order_relaxed) * num_sms());
  } else {
    grid = (H + Gm::G - 1) / Gm::G;
  }
  kern<<<(unsigned)grid, Gm::THREADS, smem, st>>>(u, f, fstride, sp, D, y, B, H, Lrow, C, conj_filter);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_fftconv_dispatch(const T* u, const float* f, int fstride, SsmArgs sp, const float* D,
                                           T* y, int B, int H, long long Lrow, int Lc, int C, int conj_filter,
                                           cudaStream_t st) {
  if (sp.dt != nullptr) return launch_fftconv_gen<T>(u, f, fstride, sp, D, y, B, H, Lrow, Lc, C, st);
  
  switch (Lc) {
    case 16: return launch_fftconv_t<T, 5, false>(u, f, fstride, sp, D, y, B, H, Lrow, C, conj_filter, st);
    case 32: return launch_fftconv_t<T, 6, false>(u, f, fstride, sp, D, y, B, H, Lrow, C, conj_filter, st);
    case 64: return launch_fftconv_t<T, 7, false>(u, f, fstride, sp, D, y, B, H, Lrow, C, conj_filter, st);
    case 128: return launch_fftconv_t<T, 8, false>(u, f, fstride, sp, D, y, B, H, Lrow, C, conj_filter, st);
    case 256: return launch_fftconv_t<T, 9, false>(u, f, fstride, sp, D, y, B, H, Lrow, C, conj_filter, st);
    case 512: return launch_fftconv_t<T, 10, false>(u, f, fstride, sp, D, y, B, H, Lrow, C, conj_filter, st);
    case 1024: return launch_fftconv_t<T, 11, false>(u, f, fstride, sp, D, y, B, H, Lrow, C, conj_filter, st);
    case 2048: return launch_fftconv_t<T, 12, false>(u, f, fstride, sp, D, y, B, H, Lrow, C, conj_filter, st);
    case 4096: return launch_fftconv_t<T, 13, false>(u, f, fstride, sp, D, y, B, H, Lrow, C, conj_filter, st);
    case 8192: return launch_fftconv_t<T, 14, false>(u, f, fstride, sp, D, y, B, H, Lrow, C, conj_filter, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fc

