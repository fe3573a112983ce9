// Causal convolution with an arbitrary real filter as long as the input
// (8192 < L <= 65536, any length), as one zero-padded FFT convolution per row.
//
// H3 summary, appendix F "Raw speech and EEG": long convolutions over
// 12,000-step EEG clips; §2 "Convolutional view": y = f * u + D u with the
// causal crop of the zero-padded (linear) convolution.  The transform length
// M = 2^ceil(log2(2L - 1)) (32768 .. 131072) does not fit one SM's shared
// memory in fp32, so it is split four-step: M = M1 x M2 with M2 = 256 and
// M1 = M / 256, n = n1 + M1 n2, k = M2 k1 + k2 (n1, k1 < M1; n2, k2 < M2),
//   X[M2 k1 + k2] = sum_n1 w_M1^(n1 k1) [ w_M^(n1 k2) sum_n2 w_M2^(n2 k2) x[n1 + M1 n2] ].
// Three passes per pair of rows (two real rows packed as u0 + i u1; f is
// real, so the real and imaginary outputs are the two convolutions), with
// the spectrum in fp32 global memory between them:
//   pass 1  per n1: the M2-point DFT over n2, then the twiddle w_M^(n1 k2)
//   pass 2  per k2: the M1-point DFT over n1, the product with F^ / M, the
//           inverse M1-point DFT and the conjugate twiddle
//   pass 3  per n1: the inverse M2-point DFT, the crop to n < L, + D u
// F^ comes from passes 1 and 2 run on the filter once per channel: pass 1
// takes the H filters and the row pairs in one launch, and pass 2 (one CTA per
// block of k2 and channel, looping over the channel's pairs) first transforms
// its slice of the filter's pass-1 output and keeps it in registers (for
// M1 = 512 the slice does not fit, and lc_spectrum writes F^ to the workspace
// first).  Every DFT is the register/shared-memory Stockham FFT of
// fft_stockham.cuh, one group of TG threads per sequence; each pass stages its
// tile through shared memory (the same region as the FFT buffers) so that
// global reads and writes run along the contiguous index.
#include "fftconv_impl.cuh"
#include "kernels.cuh"

namespace fc {

namespace {
constexpr int kLM2 = 8, kM2 = 1 << kLM2;  // inner DFT length
constexpr int kThr = 256;
constexpr int kNB = 16;                   // n1 values per CTA in passes 1 and 3 (one per thread group)

template <typename T> __device__ __forceinline__ float ld_io(const T* p) { return (float)*p; }
template <> __device__ __forceinline__ float ld_io<__half>(const __half* p) { return __half2float(*p); }
template <> __device__ __forceinline__ float ld_io<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }
template <typename T> __device__ __forceinline__ T st_io(float v) { return (T)v; }
template <> __device__ __forceinline__ __half st_io<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 st_io<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// The four-step twiddle w_M^(n1 k2) (n1 < M1, k2 < 256, so n1 k2 < M needs no
// reduction) as the product of two table entries: with t = 256 a + b,
// w_M^t = w_M1^a w_M^b.  hi[a] = w_M1^a (M1 entries), lo[b] = w_M^b (256).
template <int LOGM1>
__device__ __forceinline__ void fill_step_twiddles(float2* hi, float2* lo, int tid) {
  constexpr int M1 = 1 << LOGM1, M = M1 * kM2;
  for (int j = tid; j < M1 + kM2; j += kThr) {
    float sn, cs;
    if (j < M1) {
      sincospif(-2.0f * (float)j / (float)M1, &sn, &cs);
      hi[j] = make_float2(cs, sn);
    } else {
      sincospif(-2.0f * (float)(j - M1) / (float)M, &sn, &cs);
      lo[j - M1] = make_float2(cs, sn);
    }
  }
}
__device__ __forceinline__ float2 step_twiddle(const float2* hi, const float2* lo, int n1, int k2) {
  const int t = n1 * k2;
  return cmul(hi[t >> kLM2], lo[t & (kM2 - 1)]);
}

template <int LOGN>
struct Grp {  // one length-N sequence per group of TG threads
  using P = FftPlan<LOGN>;
  static constexpr int N = P::M, TG = P::TG, R0 = P::R0, RL = P::RLAST, RM = P::RMAX;
  static constexpr int G = kThr / TG;                       // sequences per CTA
  static constexpr int SH = ILog2<R0>::v;
  static constexpr int BUF = N + (N >> SH);
  static constexpr int PER0 = RM / R0, PER_L = RM / RL;
  // row stride (in float2) of a [position][G] staging tile: with G + 2 the 32
  // lanes of a warp (32 / TG sequences x TG positions, TG = 8 or 16) hit every
  // 8-byte bank pair exactly twice, and rows stay 16-byte aligned
  static constexpr int TS = G + 2;
  static_assert(TG == 8 || TG == 16, "stride chosen for 8 or 16 threads per sequence");
  // a staging tile of `rows` positions and the group FFT buffers share one
  // region: the tile is read into registers before the first buffer store
  // (after a CTA barrier inside the transform) and written only after a
  // barrier that follows the last buffer load
  static constexpr size_t region(int rows) {
    return (size_t)rows * TS > (size_t)G * BUF ? (size_t)rows * TS : (size_t)G * BUF;
  }
};

template <int LOGN>
__device__ __forceinline__ void fill_twiddles(float2* tw, int tid) {
  using P = FftPlan<LOGN>;
  for (int j = tid; j < P::TWN; j += kThr) {
    float sn, cs;
    sincospif(-2.0f * (float)j / (float)P::M, &sn, &cs);
    tw[j] = make_float2(cs, sn);
  }
}

// Row q of channel h in a B x H x L array.
__device__ __forceinline__ size_t row_of(int b, int h, int H, int L) { return ((size_t)b * H + h) * (size_t)L; }

}  // namespace

// ---------------------------------------------------------------- pass 1
// grid (M1 / kNB, rows): CTA = 16 consecutive n1 of one item q = q0 +
// blockIdx.y: the filter of channel q for q < nfr (into Yf), else row pair
// q - nfr (into Y).  Out[item][n1][k2] = w_M^(n1 k2) DFT_M2(x[n1 + M1 n2]).
template <typename T, int LOGM1>
__global__ void __launch_bounds__(kThr) lc_pass1(const T* __restrict__ u, const float* __restrict__ f,
                                                 float2* __restrict__ Y, float2* __restrict__ Yf, int B, int H,
                                                 int L, int q0, int nfr) {
  using G2 = Grp<kLM2>;
  static_assert(G2::G == kNB, "one thread group per n1 of the CTA");
  constexpr int M1 = 1 << LOGM1;
  extern __shared__ float2 lsm[];
  float2* tile = lsm;                        // [n2][TS]
  float2* gbuf = lsm;                        // per group FFT buffers (same region)
  float2* tw = lsm + G2::region(kM2);
  float2* thi = tw + FftPlan<kLM2>::TWN;     // four-step twiddle tables
  float2* tlo = thi + M1;
  const int tid = threadIdx.x, g = tid / G2::TG, tg = tid - g * G2::TG;
  const int n10 = blockIdx.x * kNB, q = q0 + (int)blockIdx.y;
  const bool filt = q < nfr;
  const int p = filt ? q : q - nfr;
  fill_twiddles<kLM2>(tw, tid);
  fill_step_twiddles<LOGM1>(thi, tlo, tid);
  // the two real rows of the pair (channel h, batches 2 bp and 2 bp + 1), or the filter
  const float* fr = nullptr;
  const T* u0 = nullptr;
  const T* u1 = nullptr;
  if (filt) {
    fr = f + (size_t)p * L;
  } else {
    const int nbp = (B + 1) / 2, h = p / nbp, bp = p - h * nbp;
    u0 = u + row_of(2 * bp, h, H, L);
    if (2 * bp + 1 < B) u1 = u + row_of(2 * bp + 1, h, H, L);
  }
  for (int idx = tid; idx < kM2 * kNB; idx += kThr) {
    const int n2 = idx / kNB, c = idx - n2 * kNB;
    const long long n = (long long)(n10 + c) + (long long)M1 * n2;
    float2 v = make_float2(0.f, 0.f);
    if (n < L) {
      if (fr) {
        v.x = fr[n];
      } else {
        v.x = ld_io(u0 + n);
        if (u1) v.y = ld_io(u1 + n);
      }
    }
    tile[n2 * G2::TS + c] = v;
  }
  __syncthreads();
  float2 v[G2::RM];
#pragma unroll
  for (int i = 0; i < G2::PER0; ++i)
#pragma unroll
    for (int r = 0; r < G2::R0; ++r) v[i * G2::R0 + r] = tile[(tg + i * G2::TG + r * (kM2 / G2::R0)) * G2::TS + g];
  fft_fwd<kLM2>(v, gbuf + g * G2::BUF, tg, tw);
  // v[i RL + r] = bin k2 = j + r M2 / RL, j = tg + i TG; twiddle and store row n1 of Y
  const int n1 = n10 + g;
  float2* yrow = (filt ? Yf : Y) + ((size_t)p * M1 + n1) * kM2;
#pragma unroll
  for (int i = 0; i < G2::PER_L; ++i)
#pragma unroll
    for (int r = 0; r < G2::RL; ++r) {
      const int k2 = tg + i * G2::TG + r * (kM2 / G2::RL);
      yrow[k2] = cmul(v[i * G2::RL + r], step_twiddle(thi, tlo, n1, k2));
    }
}

// ---------------------------------------------------------------- pass 2
// 16-byte asynchronous global -> shared copies (two float2 at a time)
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Filter spectra: grid (M2 / G1, channels), CTA = G1 consecutive k2 of one
// filter.  The forward M1-point DFT of the filter's pass-1 output, written as
// Fs[h][k2][k1] = X[M2 k1 + k2] / M.
template <int LOGM1>
__global__ void __launch_bounds__(kThr) lc_spectrum(const float2* __restrict__ Y, float2* __restrict__ Fs, int h0) {
  using G1 = Grp<LOGM1>;
  constexpr int M1 = 1 << LOGM1, M = M1 * kM2, GK = G1::G;
  extern __shared__ float2 lsm[];
  float2* tile = lsm;                        // [n1][TS]
  float2* gbuf = lsm;                        // (same region)
  float2* tw = lsm + G1::region(M1);
  const int tid = threadIdx.x, g = tid / G1::TG, tg = tid - g * G1::TG;
  const int k20 = blockIdx.x * GK, h = h0 + (int)blockIdx.y;
  fill_twiddles<LOGM1>(tw, tid);
  const float2* yp = Y + (size_t)h * M1 * kM2;
  for (int idx = tid; idx < M1 * GK; idx += kThr) {
    const int n1 = idx / GK, c = idx - n1 * GK;
    tile[n1 * G1::TS + c] = yp[(size_t)n1 * kM2 + k20 + c];
  }
  __syncthreads();
  float2 v[G1::RM];
#pragma unroll
  for (int i = 0; i < G1::PER0; ++i)
#pragma unroll
    for (int r = 0; r < G1::R0; ++r) v[i * G1::R0 + r] = tile[(tg + i * G1::TG + r * (M1 / G1::R0)) * G1::TS + g];
  fft_fwd<LOGM1>(v, gbuf + g * G1::BUF, tg, tw);
  // v[i RL + r] = X[M2 k1 + k2], k1 = j + r M1 / RL
  const int k2 = k20 + g;
  float2* fs = Fs + ((size_t)h * kM2 + k2) * M1;
  constexpr float inv_m = 1.0f / (float)M;
#pragma unroll
  for (int i = 0; i < G1::PER_L; ++i)
#pragma unroll
    for (int r = 0; r < G1::RL; ++r) {
      const int k1 = tg + i * G1::TG + r * (M1 / G1::RL);
      fs[k1] = make_float2(v[i * G1::RL + r].x * inv_m, v[i * G1::RL + r].y * inv_m);
    }
}

// grid (M2 / G1, channels): CTA = G1 consecutive k2 of every row pair of one
// channel h (pairs p = h ceil(B / 2) + bp).  Per pair: the forward M1-point
// DFT over n1, the product with the filter spectrum F^, the inverse DFT, the
// conjugate twiddle, back into Y.  The next item's columns are copied into
// the second staging tile while this one is transformed.  Where the
// spectrum slice fits in registers (M1 <= 256), the CTA computes it itself
// first, from the filter's pass-1 output Yf[h] (F^ = forward DFT / M); past
// that it reads F^ from Fs[h][k2][k1], written by lc_spectrum.
template <int LOGM1>
__global__ void __launch_bounds__(kThr, LOGM1 == 9 ? 1 : 3) lc_pass2(float2* __restrict__ Y, const float2* __restrict__ Fsrc, int B,
                                                 int h0, int conj_filter) {
  using G1 = Grp<LOGM1>;
  constexpr int M1 = 1 << LOGM1, M = M1 * kM2, GK = G1::G;
  constexpr bool kFreg = G1::RM <= 16;
  constexpr int kReg = (int)G1::region(M1);
  constexpr int q0 = kFreg ? 0 : 1;          // item 0 is the filter, items 1.. the pairs
  extern __shared__ float2 lsm[];
  float2* tw = lsm + 2 * kReg;               // [tile 0][tile 1][FFT twiddles][four-step tables]
  float2* thi = tw + FftPlan<LOGM1>::TWN;
  float2* tlo = thi + M1;
  const int tid = threadIdx.x, g = tid / G1::TG, tg = tid - g * G1::TG;
  const int k20 = blockIdx.x * GK, h = h0 + (int)blockIdx.y, k2 = k20 + g;
  const int nbp = (B + 1) / 2;
  fill_twiddles<LOGM1>(tw, tid);
  fill_step_twiddles<LOGM1>(thi, tlo, tid);
  auto prefetch = [&](int q) {  // columns k20 .. k20 + GK of item q into tile q % 2
    float2* tile = lsm + (q & 1) * kReg;
    const float2* yp = (q == 0 ? Fsrc + (size_t)h * M1 * kM2 : Y + ((size_t)h * nbp + (q - 1)) * M1 * kM2) + k20;
    for (int idx = 2 * tid; idx < M1 * GK; idx += 2 * kThr) {
      const int n1 = idx / GK, c = idx - n1 * GK;
      cp_async16(tile + n1 * G1::TS + c, yp + (size_t)n1 * kM2 + c);
    }
    cp_async_commit();
  };
  prefetch(q0);
  const float2* fs = Fsrc + ((size_t)h * kM2 + k2) * M1;  // Fs layout (kFreg false)
  const float sgn = conj_filter ? -1.f : 1.f;
  float2 F[kFreg ? G1::RM : 1];
  for (int q = q0; q <= nbp; ++q) {
    float2* tile = lsm + (q & 1) * kReg;
    float2* gbuf = tile;                     // the FFT buffers share the current tile's region
    if (q < nbp) {
      prefetch(q + 1);  // tile (q + 1) % 2 was released by the barrier that ended item q - 1
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    float2 v[G1::RM];
#pragma unroll
    for (int i = 0; i < G1::PER0; ++i)
#pragma unroll
      for (int r = 0; r < G1::R0; ++r) v[i * G1::R0 + r] = tile[(tg + i * G1::TG + r * (M1 / G1::R0)) * G1::TS + g];
    fft_fwd<LOGM1>(v, gbuf + g * G1::BUF, tg, tw);
    if (q == 0) {  // the filter: v[i RL + r] = X[M2 k1 + k2], k1 = j + r M1 / RL
      if constexpr (kFreg) {
        constexpr float inv_m = 1.0f / (float)M;
#pragma unroll
        for (int k = 0; k < G1::RM; ++k) F[k] = make_float2(v[k].x * inv_m, sgn * v[k].y * inv_m);
      }
      __syncthreads();  // tile 0 is free for the prefetch of item 2
      continue;
    }
#pragma unroll
    for (int i = 0; i < G1::PER_L; ++i)
#pragma unroll
      for (int r = 0; r < G1::RL; ++r) {
        float2 f;
        if constexpr (kFreg) {
          f = F[i * G1::RL + r];
        } else {
          f = fs[tg + i * G1::TG + r * (M1 / G1::RL)];
          f.y *= sgn;
        }
        v[i * G1::RL + r] = cmul(v[i * G1::RL + r], f);
      }
    __syncthreads();  // every group is past its forward transform (buffer reuse in the inverse)
    fft_inv<LOGM1>(v, gbuf + g * G1::BUF, tg, tw);
    __syncthreads();  // every group is done with its buffer (the tile's region)
    // v[i R0 + r] = n1 = j + r M1 / R0: conjugate twiddle, then back through the tile
#pragma unroll
    for (int i = 0; i < G1::PER0; ++i)
#pragma unroll
      for (int r = 0; r < G1::R0; ++r) {
        const int n1 = tg + i * G1::TG + r * (M1 / G1::R0);
        tile[n1 * G1::TS + g] = cmul(v[i * G1::R0 + r], cconj(step_twiddle(thi, tlo, n1, k2)));
      }
    __syncthreads();
    float2* yp = Y + ((size_t)h * nbp + (q - 1)) * M1 * kM2 + k20;
    for (int idx = tid; idx < M1 * GK; idx += kThr) {
      const int n1 = idx / GK, c = idx - n1 * GK;
      yp[(size_t)n1 * kM2 + c] = tile[n1 * G1::TS + c];
    }
    __syncthreads();  // tile q % 2 is free for the prefetch of item q + 2
  }
}

// ---------------------------------------------------------------- pass 3
// grid (M1 / kNB, pairs): CTA = 16 consecutive n1 of one row pair.  The
// inverse M2-point DFT of Y'[n1][.] gives x[n1 + M1 n2]; rows n < L are
// stored with + D u.
template <typename T, int LOGM1>
__global__ void __launch_bounds__(kThr) lc_pass3(const float2* __restrict__ Y, const T* __restrict__ u,
                                                 const float* __restrict__ D, T* __restrict__ y, int B, int H,
                                                 int L, int p0) {
  using G2 = Grp<kLM2>;
  constexpr int M1 = 1 << LOGM1;
  extern __shared__ float2 lsm[];
  float2* tile = lsm;                        // [n2][TS]
  float2* gbuf = lsm;                        // (same region)
  float2* tw = lsm + G2::region(kM2);
  const int tid = threadIdx.x, g = tid / G2::TG, tg = tid - g * G2::TG;
  const int n10 = blockIdx.x * kNB, p = p0 + (int)blockIdx.y;
  fill_twiddles<kLM2>(tw, tid);
  // u for the D u term, loaded first so that its latency hides under the transform
  const int nbp = (B + 1) / 2, h = p / nbp, bp = p - h * nbp;
  const size_t r0 = row_of(2 * bp, h, H, L);
  const bool has1 = 2 * bp + 1 < B;
  const size_t r1 = has1 ? row_of(2 * bp + 1, h, H, L) : r0;
  const float dh = D[h];
  constexpr int kPer = kM2 * kNB / kThr;
  float du0[kPer], du1[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int idx = tid + k * kThr, n2 = idx / kNB, c = idx - n2 * kNB;
    const long long n = (long long)(n10 + c) + (long long)M1 * n2;
    du0[k] = n < L ? dh * ld_io(u + r0 + n) : 0.f;
    du1[k] = (has1 && n < L) ? dh * ld_io(u + r1 + n) : 0.f;
  }
  __syncthreads();
  const int n1 = n10 + g;
  const float2* yrow = Y + ((size_t)p * M1 + n1) * kM2;
  float2 v[G2::RM];
  // input in the forward's last-stage layout: v[i RL + r] = k2 = j + r M2 / RL
#pragma unroll
  for (int i = 0; i < G2::PER_L; ++i)
#pragma unroll
    for (int r = 0; r < G2::RL; ++r) v[i * G2::RL + r] = yrow[tg + i * G2::TG + r * (kM2 / G2::RL)];
  fft_inv<kLM2>(v, gbuf + g * G2::BUF, tg, tw);
  __syncthreads();  // every group is done with its buffer (the tile's region)
#pragma unroll
  for (int i = 0; i < G2::PER0; ++i)
#pragma unroll
    for (int r = 0; r < G2::R0; ++r) tile[(tg + i * G2::TG + r * (kM2 / G2::R0)) * G2::TS + g] = v[i * G2::R0 + r];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int idx = tid + k * kThr, n2 = idx / kNB, c = idx - n2 * kNB;
    const long long n = (long long)(n10 + c) + (long long)M1 * n2;
    if (n < L) {
      const float2 z = tile[n2 * G2::TS + c];
      y[r0 + n] = st_io<T>(z.x + du0[k]);
      if (has1) y[r1 + n] = st_io<T>(z.y + du1[k]);
    }
  }
}

namespace {
template <int LOGN>
constexpr size_t pass_smem(int tile_rows, int step_tw) {
  return sizeof(float2) * (Grp<LOGN>::region(tile_rows) + (size_t)FftPlan<LOGN>::TWN + (size_t)step_tw);
}

size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

int log2_transform(int L) {  // M = 2^m >= 2L - 1
  int m = 0;
  while ((1LL << m) < 2LL * L - 1) ++m;
  return m;
}

template <typename T, int LOGM1>
cudaError_t long_conv_t(const void* u, const float* f, const float* D, void* y, int B, int H, int L, char* ws,
                        cudaStream_t st) {
  constexpr int M1 = 1 << LOGM1, M = M1 * kM2;
  const long long pairs = (long long)H * ((B + 1) / 2);
  float2* Y = reinterpret_cast<float2*>(ws);
  float2* Fs = reinterpret_cast<float2*>(ws + round256((size_t)pairs * M * sizeof(float2)));
  constexpr size_t s13 = pass_smem<kLM2>(kM2, M1 + kM2);
  constexpr size_t ssp = pass_smem<LOGM1>(M1, 0);
  constexpr size_t s2 = sizeof(float2) * (2 * Grp<LOGM1>::region(M1) + FftPlan<LOGM1>::TWN + M1 + kM2);
  cudaError_t e;
  if ((e = smem_optin<lc_pass1<T, LOGM1>>(s13)) != cudaSuccess) return e;
  if ((e = smem_optin<lc_spectrum<LOGM1>>(ssp)) != cudaSuccess) return e;
  if ((e = smem_optin<lc_pass2<LOGM1>>(s2)) != cudaSuccess) return e;
  if ((e = smem_optin<lc_pass3<T, LOGM1>>(s13)) != cudaSuccess) return e;
  const unsigned g13 = M1 / kNB, g2 = kM2 / Grp<LOGM1>::G;
  // pass 1 on the H filter rows and the row pairs; where pass 2 takes the
  // spectra from the filters' pass-1 output (M1 <= 256) in one launch, the
  // filters' output in the Fs area; otherwise the filters first, through the
  // Y area into lc_spectrum.  Then pass 2 per channel and pass 3 per row pair.
  constexpr bool fused_spectrum = Grp<LOGM1>::RM <= 16;
  const long long q_first = fused_spectrum ? 0 : H;
  if (!fused_spectrum) {
    for (long long c0 = 0; c0 < H; c0 += 65535) {
      const unsigned n = (unsigned)std::min<long long>(65535, H - c0);
      lc_pass1<T, LOGM1><<<dim3(g13, n), kThr, s13, st>>>((const T*)u, f, Y, Y, B, H, L, (int)c0, H);
      lc_spectrum<LOGM1><<<dim3(g2, n), kThr, ssp, st>>>(Y, Fs, (int)c0);
    }
  }
  for (long long c0 = q_first; c0 < H + pairs; c0 += 65535) {
    const unsigned n = (unsigned)std::min<long long>(65535, H + pairs - c0);
    lc_pass1<T, LOGM1><<<dim3(g13, n), kThr, s13, st>>>((const T*)u, f, Y, Fs, B, H, L, (int)c0, H);
  }
  for (long long c0 = 0; c0 < H; c0 += 65535) {
    const unsigned n = (unsigned)std::min<long long>(65535, H - c0);
    lc_pass2<LOGM1><<<dim3(g2, n), kThr, s2, st>>>(Y, Fs, B, (int)c0, 0);
  }
  for (long long c0 = 0; c0 < pairs; c0 += 65535) {
    const unsigned n = (unsigned)std::min<long long>(65535, pairs - c0);
    lc_pass3<T, LOGM1><<<dim3(g13, n), kThr, s13, st>>>(Y, (const T*)u, D, (T*)y, B, H, L, (int)c0);
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t long_conv_m(const void* u, const float* f, const float* D, void* y, int B, int H, int L, char* ws,
                        cudaStream_t st) {
  switch (log2_transform(L) - kLM2) {
    case 7: return long_conv_t<T, 7>(u, f, D, y, B, H, L, ws, st);
    case 8: return long_conv_t<T, 8>(u, f, D, y, B, H, L, ws, st);
    case 9: return long_conv_t<T, 9>(u, f, D, y, B, H, L, ws, st);
    default: return cudaErrorInvalidValue;
  }
}
}  // namespace

// [Y: pairs x M complex][Fs: H x M complex], 256-aligned; 0 for L outside (8192, 65536]
size_t fftconv_long_workspace_bytes(int B, int H, int L) {
  if (B < 1 || H < 1 || L <= 8192 || L > 65536) return 0;
  const size_t M = (size_t)1 << log2_transform(L);
  const size_t pairs = (size_t)H * (size_t)((B + 1) / 2);
  return round256(pairs * M * sizeof(float2)) + round256((size_t)H * M * sizeof(float2));
}

cudaError_t launch_fftconv_long(const void* u, const float* f, const float* D, void* y, int B, int H, int L,
                                void* workspace, int dtype, cudaStream_t st) {
  char* ws = (char*)workspace;
  switch (dtype) {
    case 0: return long_conv_m<float>(u, f, D, y, B, H, L, ws, st);
    case 1: return long_conv_m<__half>(u, f, D, y, B, H, L, ws, st);
    default: return long_conv_m<__nv_bfloat16>(u, f, D, y, B, H, L, ws, st);
  }
}

}  // namespace fc
