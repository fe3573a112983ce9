// Register DFTs and Stockham radix-R stages for the fused FFT convolution.
//
// A length-M complex FFT (M = 2L) is factored into 2 or 3 radix stages
// R0 * R1 [* R2] = M (Stockham autosort, so results come out in natural
// order without a bit-reversal pass).  Each thread owns RMAX points per
// stage: it loads them, applies the inter-stage twiddles, runs an in-register
// R-point DFT (fully unrolled, compile-time twiddles), and writes them back.
// Stages exchange data through one padded shared-memory buffer.  The last
// forward stage, the pointwise product with the filter spectrum and the first
// inverse stage all run on the same registers (same radix, same thread
// mapping), so the spectrum never goes back to shared memory.
//
// Twiddle constants are cos/sin(2 pi m / 64), m = 0..16, computed from the
// definition (they are the exact values rounded to double).
#pragma once

#include "common.cuh"

namespace fc {

__host__ __device__ constexpr double cos64_base(int i) {  // cos(2 pi i / 64), 0 <= i <= 16
  return i == 0    ? 1.0
         : i == 1  ? 0.9951847266721969
         : i == 2  ? 0.9807852804032304
         : i == 3  ? 0.9569403357322088
         : i == 4  ? 0.9238795325112867
         : i == 5  ? 0.881921264348355
         : i == 6  ? 0.8314696123025452
         : i == 7  ? 0.773010453362737
         : i == 8  ? 0.7071067811865476
         : i == 9  ? 0.6343932841636455
         : i == 10 ? 0.5555702330196023
         : i == 11 ? 0.4713967368259978
         : i == 12 ? 0.38268343236508984
         : i == 13 ? 0.29028467725446233
         : i == 14 ? 0.19509032201612833
         : i == 15 ? 0.09801714032956077
                   : 0.0;
}
__host__ __device__ constexpr double cos64(int m) {  // cos(2 pi m / 64), any m
  m = ((m % 64) + 64) % 64;
  return m <= 16 ? cos64_base(m) : m <= 32 ? -cos64_base(32 - m) : m <= 48 ? -cos64_base(m - 32) : cos64_base(64 - m);
}
__host__ __device__ constexpr double sin64(int m) { return cos64(m - 16); }

// a * exp(DIR * 2 pi i k / n).  k and n are compile-time constants once the
// loops below are unrolled, so every branch folds away; multiplications by
// 1, +-i and (1 +- i)/sqrt(2) use no general complex multiply.
template <int DIR>
__device__ __forceinline__ float2 twmul(float2 a, int k, int n) {
  constexpr float h = 0.70710678118654752440f;
  if (k == 0) return a;
  if (4 * k == n) return DIR < 0 ? make_float2(a.y, -a.x) : make_float2(-a.y, a.x);
  if (8 * k == n)
    return DIR < 0 ? make_float2((a.x + a.y) * h, (a.y - a.x) * h) : make_float2((a.x - a.y) * h, (a.x + a.y) * h);
  if (8 * k == 3 * n)
    return DIR < 0 ? make_float2((a.y - a.x) * h, -(a.x + a.y) * h) : make_float2(-(a.x + a.y) * h, (a.x - a.y) * h);
  const int m = k * (64 / n);
  const float c = (float)cos64(m);
  const float s = (float)(DIR * sin64(m));
  return make_float2(fmaf(a.x, c, -a.y * s), fmaf(a.x, s, a.y * c));
}

template <int X> struct ILog2 { static constexpr int v = 1 + ILog2<X / 2>::v; };
template <> struct ILog2<1> { static constexpr int v = 0; };

__host__ __device__ constexpr int bitrev(int x, int bits) {
  int r = 0;
  for (int i = 0; i < bits; ++i) r |= ((x >> i) & 1) << (bits - 1 - i);
  return r;
}

// In-place R-point DFT of v[0..R-1] (natural order in and out):
//   v[k] <- sum_r v[r] exp(DIR * 2 pi i r k / R).
// Radix-2 decimation in frequency over compile-time indices, followed by a
// bit-reversal that is only a renaming of registers.
template <int R, int DIR>
__device__ __forceinline__ void dft(float2* v) {
  constexpr int LG = ILog2<R>::v;
#pragma unroll
  for (int lev = 0; lev < LG; ++lev) {
    const int span = R >> (lev + 1);
#pragma unroll
    for (int start = 0; start < R; start += 2 * span) {
#pragma unroll
      for (int k = 0; k < span; ++k) {
        const float2 a = v[start + k], b = v[start + k + span];
        v[start + k] = cadd(a, b);
        v[start + k + span] = twmul<DIR>(csub(a, b), k, 2 * span);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int j = bitrev(i, LG);
    if (j > i) {
      const float2 t = v[i];
      v[i] = v[j];
      v[j] = t;
    }
  }
}

// Padded shared-memory index: one spare slot every 2^SH entries.
template <int SH>
__device__ __forceinline__ int padix(int a) { return a + (a >> SH); }

// Multiply v[r] by w^r, r = 1..R-1 (w = this DFT's base twiddle).
template <int R>
__device__ __forceinline__ void apply_twiddle(float2* v, float2 w) {
  float2 wr = w;
#pragma unroll
  for (int r = 1; r < R; ++r) {
    v[r] = cmul(v[r], wr);
    if (r + 1 < R) wr = cmul(wr, w);
  }
}

// Stockham stage geometry.  Stage radix R, NS = product of earlier radices.
// DFT j (0 <= j < M/R) reads x[j + r*M/R] and writes out[(j/NS)*NS*R + j%NS + r*NS].
template <int M, int R, int NS, int TG, int RMAX, int SH>
struct Stage {
  static constexpr int NDFT = M / R;
  static constexpr int PER = RMAX / R;
  static_assert(PER * TG == NDFT, "plan: each thread owns RMAX points per stage");

  static __device__ __forceinline__ void load(const float2* buf, float2* v, int tid) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int j = tid + i * TG;
#pragma unroll
      for (int r = 0; r < R; ++r) v[i * R + r] = buf[padix<SH>(j + r * NDFT)];
    }
  }
  // tw[j] = exp(-2 pi i j / M) for j < M / RMIN (forward sign; the inverse uses
  // the conjugate).  Stage base twiddle for DFT j: exp(DIR 2 pi i k / (NS R)),
  // k = j mod NS, i.e. table index k * M / (NS * R).
  template <int DIR>
  static __device__ __forceinline__ void compute(float2* v, int tid, const float2* tw) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int j = tid + i * TG;
      if constexpr (NS > 1) {
        const float2 w = tw[(j & (NS - 1)) * (M / (NS * R))];
        apply_twiddle<R>(v + i * R, DIR < 0 ? w : cconj(w));
      }
      dft<R, DIR>(v + i * R);
    }
  }
  static __device__ __forceinline__ void store(float2* buf, const float2* v, int tid) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int j = tid + i * TG;
      const int k = j & (NS - 1);
      const int base = (j - k) * R + k;
#pragma unroll
      for (int r = 0; r < R; ++r) buf[padix<SH>(base + r * NS)] = v[i * R + r];
    }
  }
};

// Factorisations of M = 2L.  TG threads per sequence, RMAX points per thread.
template <int LOGM> struct FftPlan;
#define FC_PLAN(LOGM_, R0_, R1_, R2_)                                          \
  template <> struct FftPlan<LOGM_> {                                          \
    static constexpr int M = 1 << LOGM_;                                       \
    static constexpr int R0 = R0_, R1 = R1_, R2 = R2_;                         \
    static constexpr int NST = (R2_ > 1) ? 3 : 2;                              \
    static constexpr int RMAX = (R0 > R1 ? (R0 > R2 ? R0 : R2) : (R1 > R2 ? R1 : R2)); \
    static constexpr int TG = M / RMAX;                                        \
    static constexpr int RLAST = (R2_ > 1) ? R2_ : R1_;                        \
    static constexpr int RMIN = (R2_ > 1) ? (R0 < R1 ? (R0 < R2 ? R0 : R2) : (R1 < R2 ? R1 : R2)) \
                                          : (R0 < R1 ? R0 : R1);               \
    static constexpr int TWN = M / RMIN;                                       \
  };
FC_PLAN(5, 4, 8, 1)
FC_PLAN(6, 8, 8, 1)
FC_PLAN(7, 16, 8, 1)
FC_PLAN(8, 16, 16, 1)
FC_PLAN(9, 16, 32, 1)
FC_PLAN(10, 32, 32, 1)
FC_PLAN(11, 16, 16, 8)
FC_PLAN(12, 16, 16, 16)
FC_PLAN(13, 32, 16, 16)
FC_PLAN(14, 32, 32, 16)
#undef FC_PLAN

}  // namespace fc
