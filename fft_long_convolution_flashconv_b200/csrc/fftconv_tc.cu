// Fused FFT convolution with block-FFT stages on the 5th-generation tensor
// cores (fp16 / bf16 I/O, L = 1024, i.e. M = 2L = 2048 = 128 x 16).
//
// H3 summary section 4 "Short-sequence computation": FFT, pointwise multiply
// and inverse FFT fused in one kernel, with the block FFT written partly as
// matrix multiplies so that it runs on the tensor cores (H3 blog, "Fused Block
// FFTConv").  Index split n = 16 n1 + n2, k = k1 + 128 k2 (n1, k1 < 128,
// n2, k2 < 16), w_K = exp(-2 pi i / K):
//   stage A   (GEMM)  Y[k1,n2]  = sum_{n1<64} w_128^(n1 k1) x[16 n1 + n2]   (n1 >= 64: zero padding)
//   registers         X^[k1,k2] = sum_n2 w_16^(n2 k2) w_2048^(k1 n2) Y[k1,n2]  (the 2048-point transform at k1 + 128 k2)
//                     V         = X^ . F^ / M
//                     Z[k1,n2]  = w_2048^(-k1 n2) sum_k2 w_16^(-n2 k2) V[k1,k2]
//   stage A'  (GEMM)  y[16 n1 + n2] = sum_{k1} w_128^(-n1 k1) Z[k1, n2],      n1 < 64
// (F^ is the filter's transform, computed by the same steps as one more
// sequence.)  The length-128 DFTs are the dense contractions and run on the
// tensor cores with fp32 accumulation in TMEM; everything between them (both
// twiddle multiplies, the two radix-4 x 4 DFT-16s and the filter product) is
// one pass in fp32 registers: the thread that owns TMEM lane k1 holds all 16
// values n2 of a sequence.  Two constant 128x128 matrices hold the real
// DFT-128 blocks,
//   CA[k1][j] = j<64 ?  cos(2 pi k1 j/128) : sin(2 pi k1 (j-64)/128)
//   CB[k1][j] = j<64 ? -sin(2 pi k1 j/128) : cos(2 pi k1 (j-64)/128)
// read K-major by stage A and (the DFT matrix being symmetric) MN-major by
// stage A':
//   stage A : Yr = CA[:, :64] Xr + CA[:, 64:] Xi,   Yi = CA[:, :64] Xi + CB[:, :64] Xr
//   stage A': rows j<64 give Re y[n1=j], rows j>=64 give Im y[n1=j-64]:
//             y = CA^T Zr + CB^T Zi
// Both GEMMs take their operands in the I/O type.  The constant blocks and
// the twiddles come from tables built with the library (tc_tables.inc) and are
// copied into shared memory once per CTA.
//
// Stage A runs as D = C [Xr | Xi] + S [Xi | -Xr] = [Yr | Yi] with C = CA[:, :64],
// S = CA[:, 64:] held in tensor memory (A operand) and the operand written as
// three planes [Xr | Xi | -Xr], so 8 MMAs of N = 2 NC cover both parts.
//
// Work: a tuple is one row pair of one channel (two real rows packed as one
// complex sequence u0 + i u1; f is real, so the real and imaginary outputs
// are the two convolutions); a round is 3 consecutive tuples (channel-major),
// spanning at most 2 channels when every channel has >= 2 pairs (B >= 3).
// Stage-A columns of a round: its filters, then its pairs (NC = 16 x (nf +
// np) <= 80).  CTA b takes the rounds b + G i (G = grid size).  One CTA per
// SM, warp-specialised:
//   warps 0..11  register pass: three threads per frequency row, one tuple each
//                (its filter's F^ and its pair), then the previous round's
//                outputs of the same tuple (epilogue) from the other stage-A'
//                accumulator;
//   warps 12..14 bulk copies of the rows and filters two rounds ahead (two
//                staging buffers; one lane per warp, each with its own byte
//                count on the buffer's copy barrier) and the stage-A operand
//                from the staged rows (two operand buffers, so the operand of
//                round j + 1 is written while stage A of round j reads);
//   warp 15      issues every MMA: stage A of round j + 1 as soon as its operand
//                is written, stage A' of round j once the register pass is done.
// Tensor memory: C, S; two stage-A accumulators and two stage-A' accumulators,
// so stage A of the next round and stage A' of this one run under the
// register pass.  The stage-A' operand Z has one buffer: the register pass of
// round j writes it once stage A' of round j - 1 has completed (which the
// epilogue of round j - 1 waits for anyway).  All waits are on mbarriers with a time bound; a wait that
// runs out marks the CTA aborted and counts it in a device counter, after
// which the issuing threads complete every phase by plain arrivals (no more
// copies or MMAs), nothing is written to y, and the CTA drains its MMAs and
// copies and frees its TMEM.
#include "kernels.cuh"
#include "tc100.cuh"

#define FC_TABLES_DFT128
#define FC_TABLES_1K
#include "tc_tables.inc"

namespace fc {

static __device__ unsigned int g_fftconv_tc_timeouts;

namespace {
constexpr int kN1 = 128, kN2 = 16, kM = kN1 * kN2, kL = kM / 2;
constexpr int kThr = 512;
constexpr int kCompWarps = 12;                              // three threads per frequency row
constexpr int kFillWarps = 3;                               // then three operand warps and one MMA warp
constexpr int kSlots = 3;                                   // (channel, row pair) tuples per round
constexpr int kMaxF = 2;                                    // distinct channels per round (needs >= 2 pairs per channel)
constexpr int kMaxNC = kN2 * (kMaxF + kSlots);              // stage-A columns per part
// tensor memory columns: the DFT-128 blocks C, S (A operand of stage A), two
// stage-A accumulators (re | im), two stage-A' accumulators
constexpr uint32_t kTConst = 0, kTA0 = 64, kTA1 = kTA0 + 2 * kMaxNC, kTB0 = kTA1 + 2 * kMaxNC,
                   kTB1 = kTB0 + kN2 * kSlots;
static_assert(kTB1 + kN2 * kSlots <= 512, "TMEM budget");
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kCLbo = 128, kCSbo = (kN1 / 8) * 128;   // CA / CB K-major: 128 rows x 128 K
constexpr uint32_t kCBytes = kN1 * kN1 * 2;
constexpr uint32_t kTwBytes = kN1 * kN2 * 8;                // fp32 twiddles, [n2 / 2][k1][n2 % 2]
constexpr uint32_t kRowBytes = kL * 2;                      // one 16-bit input row
constexpr uint32_t kFBytes = kL * 4;                        // one fp32 filter
constexpr uint32_t kXBytes = 64 * 3 * kMaxNC * 2;           // stage-A operand [Xr | Xi | -Xr], 64 K-rows
constexpr uint32_t kZBytes = 2 * kN1 * kN2 * kSlots * 2;    // stage-A' operand, 256 K-rows (re | im)
// shared memory layout (bytes)
constexpr uint32_t kOCa = 0, kOCb = kCBytes, kOTw = 2 * kCBytes;
constexpr uint32_t kSUBytes = 2 * kSlots * kRowBytes;      // one round's staged input rows (2 per tuple)
constexpr uint32_t kSFBytes = kMaxF * kFBytes;              // one round's staged filters
constexpr uint32_t kOSU = kOTw + kTwBytes;                  // two staging buffers: round j in buffer j % 2
constexpr uint32_t kOSF = kOSU + 2 * kSUBytes;
constexpr uint32_t kOX = kOSF + 2 * kSFBytes;               // two stage-A operand buffers: round j in j % 2
constexpr uint32_t kOZ = kOX + 2 * kXBytes;                 // one stage-A' operand buffer
// mbarriers: tables, copies[0], A[2], A'[2], drain, Z[2], copies[1]
constexpr uint32_t kOBar = kOZ + kZBytes;
constexpr uint32_t kOMisc = kOBar + 8 * 10;                 // TMEM base, abort flag
constexpr uint32_t kSmem = kOMisc + 16;
static_assert(kSmem <= 232448, "shared memory budget");

template <typename T> struct Op;
template <> struct Op<__half> {
  static constexpr int bf16 = 0;
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ const uint16_t* ca() { return g_ca_f16; }
  static __device__ __forceinline__ const uint16_t* cb() { return g_cb_f16; }
};
template <> struct Op<__nv_bfloat16> {
  static constexpr int bf16 = 1;
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ const uint16_t* ca() { return g_ca_bf16; }
  static __device__ __forceinline__ const uint16_t* cb() { return g_cb_bf16; }
};

// named barrier 1: the four support warps
__device__ __forceinline__ void nbar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// cos, sin of 2 pi m / 16
constexpr float kCos16[10] = {1.0f, 0.92387953251128674f, 0.70710678118654752f, 0.38268343236508977f, 0.0f,
                              -0.38268343236508977f, -0.70710678118654752f, -0.92387953251128674f, -1.0f,
                              -0.92387953251128674f};
constexpr float kSin16[10] = {0.0f, 0.38268343236508977f, 0.70710678118654752f, 0.92387953251128674f, 1.0f,
                              0.92387953251128674f, 0.70710678118654752f, 0.38268343236508977f, 0.0f,
                              -0.38268343236508977f};

// (r + i im) *= w_16^m (forward) or w_16^-m (INV)
template <int m, bool INV>
__host__ __device__ __forceinline__ void rot16(float& r, float& im) {
  if constexpr (m == 0) {
  } else if constexpr (m == 4) {
    const float t = r;
    if constexpr (!INV) { r = im; im = -t; } else { r = -im; im = t; }
  } else {
    constexpr float c = kCos16[m], s = INV ? kSin16[m] : -kSin16[m];
    const float t = r;
    r = t * c - im * s;
    im = t * s + im * c;
  }
}

// in-place 4-point DFT of (a, b, c, d), forward (w_4 = -i) or inverse (w_4 = +i), unnormalised
template <bool INV>
__host__ __device__ __forceinline__ void dft4(float& ar, float& ai, float& br, float& bi, float& cr, float& ci,
                                              float& dr, float& di) {
  const float s0r = ar + cr, s0i = ai + ci, d0r = ar - cr, d0i = ai - ci;
  const float s1r = br + dr, s1i = bi + di, d1r = br - dr, d1i = bi - di;
  ar = s0r + s1r; ai = s0i + s1i;
  cr = s0r - s1r; ci = s0i - s1i;
  if constexpr (!INV) { br = d0r + d1i; bi = d0i - d1r; dr = d0r - d1i; di = d0i + d1r; }
  else                { br = d0r - d1i; bi = d0i + d1r; dr = d0r + d1i; di = d0i - d1r; }
}

// twiddles w_16^(p q) at position 4 p + q (p, q < 4) between the two radix-4 steps
template <bool INV>
__host__ __device__ __forceinline__ void rot16_grid(float* re, float* im) {
  rot16<1, INV>(re[5], im[5]);   rot16<2, INV>(re[6], im[6]);   rot16<3, INV>(re[7], im[7]);
  rot16<2, INV>(re[9], im[9]);   rot16<4, INV>(re[10], im[10]); rot16<6, INV>(re[11], im[11]);
  rot16<3, INV>(re[13], im[13]); rot16<6, INV>(re[14], im[14]); rot16<9, INV>(re[15], im[15]);
}

// 16-point DFT, radix 4 x 4, n = 4 a + b, k = c + 4 d.
// Forward: natural-order input, output X[c + 4 d] at position 4 c + d.
// Inverse: input V[c + 4 d] at position 4 c + d (the forward's order), output
// W[n] at position n.  Unnormalised.
template <bool INV>
__host__ __device__ __forceinline__ void dft16(float* re, float* im) {
  if constexpr (!INV) {
#pragma unroll
    for (int b = 0; b < 4; ++b)  // over a: positions b + 4 a -> T_b[c] at 4 c + b
      dft4<false>(re[b], im[b], re[b + 4], im[b + 4], re[b + 8], im[b + 8], re[b + 12], im[b + 12]);
    rot16_grid<false>(re, im);   // w_16^(b c)
#pragma unroll
    for (int c = 0; c < 4; ++c)  // over b: positions 4 c + b -> X[c + 4 d] at 4 c + d
      dft4<false>(re[4 * c], im[4 * c], re[4 * c + 1], im[4 * c + 1], re[4 * c + 2], im[4 * c + 2], re[4 * c + 3],
                  im[4 * c + 3]);
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c)  // over d: positions 4 c + d -> S_c[e] at 4 c + e
      dft4<true>(re[4 * c], im[4 * c], re[4 * c + 1], im[4 * c + 1], re[4 * c + 2], im[4 * c + 2], re[4 * c + 3],
                 im[4 * c + 3]);
    rot16_grid<true>(re, im);    // w_16^(-c e)
#pragma unroll
    for (int e = 0; e < 4; ++e)  // over c: positions e + 4 c -> W[e + 4 f] at e + 4 f
      dft4<true>(re[e], im[e], re[e + 4], im[e + 4], re[e + 8], im[e + 8], re[e + 12], im[e + 12]);
  }
}

// (re, im)[n2] *= w_2048^(+-k1 n2) for this thread's row k1 (tw points at its first pair of factors)
template <bool CONJ>
__device__ __forceinline__ void twiddle(float* re, float* im, const float4* tw) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 w = tw[j * kN1];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int n = 2 * j + q;
      if (n == 0) continue;  // w = 1
      const float wr = q ? w.z : w.x, wi = CONJ ? -(q ? w.w : w.y) : (q ? w.w : w.y);
      const float r = re[n];
      re[n] = r * wr - im[n] * wi;
      im[n] = r * wi + im[n] * wr;
    }
  }
}

// The tuples of one round: tuple t = 3 r + t' is (channel h, row pair p)
// with h = t / npairs, p = t % npairs; filters are listed once per distinct
// channel (channels are non-decreasing within a round).
struct Round {
  int np, nf, NC;   // valid tuples, distinct channels, stage-A columns per part
  int h0, h1, h2, p0, p1, p2, f1, f2;  // channels, pairs, filter index of tuples 1, 2 (tuple 0: filter 0)
  __host__ __device__ __forceinline__ int h(int t) const { return t == 0 ? h0 : (t == 1 ? h1 : h2); }
  __host__ __device__ __forceinline__ int p(int t) const { return t == 0 ? p0 : (t == 1 ? p1 : p2); }
  __host__ __device__ __forceinline__ int fidx(int t) const { return t == 0 ? 0 : (t == 1 ? f1 : f2); }
  __host__ __device__ __forceinline__ int ch(int f) const {  // channel of filter f
    return f == 0 ? h0 : (f1 == 1 ? h1 : h2);
  }
};
// Walks one CTA's rounds r = r0 + G i without dividing per round: the first
// tuple 3 r as (channel, pair), advanced by 3 G tuples at a time.
struct RoundCursor {
  long long t0, step, total;
  int h0, p0, dh, dp, npairs;
  __host__ __device__ __forceinline__ void init(long long r0, long long G, long long total_, int npairs_) {
    total = total_;
    npairs = npairs_;
    t0 = 3 * r0;
    step = 3 * G;
    h0 = (int)(t0 / npairs);
    p0 = (int)(t0 - (long long)h0 * npairs);
    dh = (int)(step / npairs);
    dp = (int)(step - (long long)dh * npairs);
  }
  __host__ __device__ __forceinline__ void advance() {
    t0 += step;
    h0 += dh;
    p0 += dp;
    if (p0 >= npairs) {
      p0 -= npairs;
      ++h0;
    }
  }
  __host__ __device__ __forceinline__ Round get() const {
    Round R;
    R.np = (int)min(3LL, total - t0);
    int h1 = h0, p1 = p0 + 1;
    if (p1 >= npairs) { p1 = 0; ++h1; }
    int h2 = h1, p2 = p1 + 1;
    if (p2 >= npairs) { p2 = 0; ++h2; }
    if (R.np < 2) { h1 = h0; p1 = p0; }  // invalid tuples repeat the last valid one
    if (R.np < 3) { h2 = h1; p2 = p1; }
    R.h0 = h0; R.p0 = p0; R.h1 = h1; R.p1 = p1; R.h2 = h2; R.p2 = p2;
    R.f1 = (h1 != h0) ? 1 : 0;
    R.f2 = R.f1 + ((h2 != h1) ? 1 : 0);
    R.nf = 1 + (R.np > 1 ? R.f1 : 0) + (R.np > 2 ? R.f2 - R.f1 : 0);
    R.NC = kN2 * (R.nf + R.np);
    return R;
  }
};
}  // namespace

// u, y: B x H x 1024 (T); f: H x 1024 fp32 filters; D: H.  B >= 3 (every channel
// has >= 2 row pairs, so a round of 3 tuples spans <= 2 channels).
template <typename T>
__global__ void __launch_bounds__(kThr, 1) fftconv_tc_kernel(const T* __restrict__ u, const float* __restrict__ f,
                                                             const float* __restrict__ D, T* __restrict__ y, int B,
                                                             int H, int conj_filter) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool compute = warp < kCompWarps;
  const bool filler = warp >= kCompWarps && warp < kCompWarps + kFillWarps;
  const bool mma_warp = warp == kCompWarps + kFillWarps;
  const int slot = warp >> 2;                       // compute: tuple of this thread within a round
  const int row = tid & (kN1 - 1);                  // TMEM lane: frequency row k1 / output lane j
  const int ft = tid - kCompWarps * 32;             // operand thread 0..95
  const int lq = warp - kCompWarps;                 // operand warp 0..2: copies tuple lq's rows and filter lq
  const bool loader = filler && lane == 0;
  const bool issuer = mma_warp && lane == 0;        // issues every MMA
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint16_t* ub = reinterpret_cast<const uint16_t*>(u);
  uint16_t* yb = reinterpret_cast<uint16_t*>(y);
  uint64_t* const bars = reinterpret_cast<uint64_t*>(sm + kOBar);
  uint64_t* const mbar_tab = bars + 0;
  uint64_t* const mbar_ld0 = bars + 1;  // copies into staging buffer 0 / 1: one arrival per loader
  uint64_t* const mbar_ld1 = bars + 9;
  uint64_t* const mbar_a = bars + 2;   // [2] stage A of a round done
  uint64_t* const mbar_b = bars + 4;   // [2] stage A' of a round done
  uint64_t* const mbar_fin = bars + 6;
  uint64_t* const mbar_z = bars + 7;   // [2] register pass of a round done: one arrival per compute warp
  uint32_t* const tmem_p = reinterpret_cast<uint32_t*>(sm + kOMisc);
  unsigned int* const abort_p = reinterpret_cast<unsigned int*>(sm + kOMisc + 4);
  const uint32_t s0 = tc::smem_u32(sm);
  const uint32_t ca = s0 + kOCa, cb = s0 + kOCb;
  const float4* const twp = reinterpret_cast<const float4*>(sm + kOTw) + row;

  const int npairs = (B + 1) / 2;
  const long long total = (long long)H * npairs;
  const long long nrounds = (total + kSlots - 1) / kSlots;
  const long long G = gridDim.x;
  const int nloc = (int)((nrounds - blockIdx.x + G - 1) / G);  // rounds of this CTA: blockIdx.x + G i
  RoundCursor cur0;  // this CTA's first round
  cur0.init(blockIdx.x, G, total, npairs);

  if (warp == 0) tc::tmem_alloc(tmem_p, 512);
  if (tid == 0) {
    for (int i = 0; i < 7; ++i) tc::mbar_init(bars + i, i == 1 ? kFillWarps : 1);
    tc::mbar_init(mbar_z, kCompWarps);
    tc::mbar_init(mbar_z + 1, kCompWarps);
    tc::mbar_init(mbar_ld1, kFillWarps);
    *abort_p = 0u;
    tc::fence_mbar_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  // Bounded wait.  A wait that runs out marks the CTA aborted (and counts it
  // once); from then on the issuing threads complete every later phase by a
  // plain arrival instead of issuing copies or MMAs, so all threads keep the
  // same sequence of waits and barriers, nothing is written to y, and the
  // kernel ends.
  auto wait_bar = [&](uint64_t* mb, uint32_t parity) {
    if (!tc::mbar_wait_bounded(mb, parity, kWaitNs) && atomicCAS(abort_p, 0u, 1u) == 0u)
      atomicAdd(&g_fftconv_tc_timeouts, 1u);
  };
  auto aborted = [&]() { return *reinterpret_cast<volatile unsigned int*>(abort_p) != 0u; };

  // ---- copies of a round's inputs into staging buffer sb (round j uses buffer j % 2): loader
  // lq copies tuple lq's rows and filter lq with its own byte count on the buffer's copy
  // barrier, so the copies issue from three schedulers at once
  uint32_t ld_out = 0u, ld_par = 0u;  // bit sb: a copy phase into buffer sb is in flight, its parity (loaders)
  auto issue_u = [&](const Round& R, int sb, bool& live) {
    uint64_t* const mb = sb ? mbar_ld1 : mbar_ld0;
    live = !aborted();
    const bool row0 = lq < R.np, row1 = row0 && 2 * R.p(lq) + 1 < B, filt = lq < R.nf;
    const uint32_t bytes = live ? (row0 ? kRowBytes : 0u) + (row1 ? kRowBytes : 0u) + (filt ? kFBytes : 0u) : 0u;
    tc::mbar_expect_tx(mb, bytes);
    if (live && row0) {
      const uint16_t* src = ub + ((size_t)(2 * R.p(lq)) * H + R.h(lq)) * kL;
      const uint32_t dst = s0 + kOSU + (uint32_t)sb * kSUBytes + (uint32_t)(2 * lq) * kRowBytes;
      tc::bulk_g2s(dst, src, kRowBytes, mb);
      if (row1) tc::bulk_g2s(dst + kRowBytes, src + (size_t)H * kL, kRowBytes, mb);
    }
  };
  auto issue_f = [&](const Round& R, int sb, bool live) {  // after issue_u of the same round
    if (live && lq < R.nf)
      tc::bulk_g2s(s0 + kOSF + (uint32_t)sb * kSFBytes + (uint32_t)lq * kFBytes, f + (size_t)R.ch(lq) * kL, kFBytes,
                   sb ? mbar_ld1 : mbar_ld0);
  };
  auto mark_out = [&](int sb, int jr) {  // round jr's copies are in flight in buffer sb
    ld_out |= 1u << sb;
    ld_par = (ld_par & ~(1u << sb)) | ((uint32_t)((jr >> 1) & 1) << sb);
  };
  // ---- staged inputs -> stage-A operand (operand threads): MN-major, 64 K-rows (n1) x 3 NC
  // columns [Xr | Xi | -Xr]; column blocks of each part: the filters, then the pairs.
  // Thread ft owns the 16-byte chunks ft and ft + 96 of every staged row (8 values n2 = 8 hf ..
  // of row n1 = chunk / 2).
  auto fill_x = [&](const Round& R, int sb, float d0, float d1) {
    const uint32_t lbo = (uint32_t)(3 * R.NC / 8) * 128;  // next 8 K-rows
    uint8_t* const X = sm + kOX + (uint32_t)sb * kXBytes;
    const uint8_t* const su = sm + kOSU + (uint32_t)sb * kSUBytes;
    const uint8_t* const sf = sm + kOSF + (uint32_t)sb * kSFBytes;
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      const int chunk = ft + 96 * pass;
      if (chunk < 128) {
        const int n1 = chunk >> 1, hf = chunk & 1;
        const uint32_t kofs = (uint32_t)(n1 >> 3) * lbo + (uint32_t)(n1 & 7) * 16;
        uint4 v[2 * kSlots];
#pragma unroll
        for (int k = 0; k < 2 * kSlots; ++k) {  // staged row k = 2 t + c
          v[k] = make_uint4(0, 0, 0, 0);
          if ((k >> 1) < R.np && 2 * R.p(k >> 1) + (k & 1) < B)
            v[k] = *reinterpret_cast<const uint4*>(su + (uint32_t)k * kRowBytes + (uint32_t)chunk * 16);
        }
        float4 fa[kMaxF], fb[kMaxF];
#pragma unroll
        for (int q = 0; q < kMaxF; ++q) {
          if (q < R.nf) {
            const uint8_t* src = sf + (uint32_t)q * kFBytes + (uint32_t)chunk * 32;  // taps 8 chunk ..
            fa[q] = *reinterpret_cast<const float4*>(src);
            fb[q] = *reinterpret_cast<const float4*>(src + 16);
          }
        }
#pragma unroll
        for (int t = 0; t < kSlots; ++t) {
          if (t < R.np) {
            const int n = (R.nf + t) * kN2 + hf * 8;
            const uint4 a = v[2 * t], b = v[2 * t + 1];
            *reinterpret_cast<uint4*>(X + (uint32_t)(n >> 3) * 128 + kofs) = a;
            *reinterpret_cast<uint4*>(X + (uint32_t)((R.NC + n) >> 3) * 128 + kofs) = b;
            *reinterpret_cast<uint4*>(X + (uint32_t)((2 * R.NC + n) >> 3) * 128 + kofs) =
                make_uint4(a.x ^ 0x80008000u, a.y ^ 0x80008000u, a.z ^ 0x80008000u, a.w ^ 0x80008000u);
          }
        }
#pragma unroll
        for (int q = 0; q < kMaxF; ++q) {  // filters: fp32 -> operand type, D folded into tap 0 (y = (f + D delta) * u)
          if (q < R.nf) {
            float4 a = fa[q];
            if (chunk == 0) a.x += (q == 0 ? d0 : d1);
            const uint4 w = make_uint4(Op<T>::pack(a.x, a.y), Op<T>::pack(a.z, a.w), Op<T>::pack(fb[q].x, fb[q].y),
                                       Op<T>::pack(fb[q].z, fb[q].w));
            const int n = q * kN2 + hf * 8;
            *reinterpret_cast<uint4*>(X + (uint32_t)(n >> 3) * 128 + kofs) = w;
            *reinterpret_cast<uint4*>(X + (uint32_t)((R.NC + n) >> 3) * 128 + kofs) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(X + (uint32_t)((2 * R.NC + n) >> 3) * 128 + kofs) =
                make_uint4(w.x ^ 0x80008000u, w.y ^ 0x80008000u, w.z ^ 0x80008000u, w.w ^ 0x80008000u);
          }
        }
      }
    }
  };

  // ---- prologue: constant tables by bulk copies, the first round's inputs
  if (tid == 0) {
    tc::mbar_expect_tx(mbar_tab, 2 * kCBytes + kTwBytes);
    tc::bulk_g2s(ca, Op<T>::ca(), kCBytes, mbar_tab);
    tc::bulk_g2s(cb, Op<T>::cb(), kCBytes, mbar_tab);
    tc::bulk_g2s(s0 + kOTw, g_tw1k, kTwBytes, mbar_tab);
  }
  bool live0 = false, live1 = false;
  RoundCursor cur1 = cur0;
  cur1.advance();
  if (loader && nloc > 0) issue_u(cur0.get(), 0, live0);
  if (loader && nloc > 1) issue_u(cur1.get(), 1, live1);
  // the filter is written by the kernel this one may be launched as a
  // programmatic dependent of: read it only after the wait
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (loader && nloc > 0) {
    mark_out(0, 0);
    issue_f(cur0.get(), 0, live0);
  }
  if (loader && nloc > 1) {
    mark_out(1, 1);
    issue_f(cur1.get(), 1, live1);
  }
  wait_bar(mbar_tab, 0);
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_p;
  if (warp < 4) {  // C = CA[:, :64], S = CA[:, 64:] of this lane's row k1 -> TMEM columns [0, 64)
    const uint8_t* rowp = sm + kOCa + (uint32_t)(row >> 3) * kCSbo + (uint32_t)(row & 7) * 16;
#pragma unroll
    for (int g8 = 0; g8 < 8; ++g8) {
      const uint4 a = *reinterpret_cast<const uint4*>(rowp + (uint32_t)(2 * g8) * 128);
      const uint4 b = *reinterpret_cast<const uint4*>(rowp + (uint32_t)(2 * g8 + 1) * 128);
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      tc::tmem_st8(tmem + lane_off + kTConst + (uint32_t)(8 * g8), w);
    }
    tc::tmem_wait_st();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  if (compute) {
    // ================= register pass: frequency row k1 = row of tuple `slot` of every round; then
    // the previous round's outputs of the same tuple slot (TMEM lane j = row)
    auto epilogue = [&](const Round& R, int buf) {
      if (slot < R.np) {  // lane j -> row b = 2 p + j / 64 of the tuple's channel, n1 = j % 64: 16 outputs
        float v[16];
        tc::tmem_ld16_wait(tmem + lane_off + (buf ? kTB1 : kTB0) + (uint32_t)(kN2 * slot), v);
        const int b = 2 * R.p(slot) + (row >> 6), n1 = row & 63;
        if (b < B && !aborted()) {
          uint4* dst = reinterpret_cast<uint4*>(yb + ((size_t)b * H + R.h(slot)) * kL + (size_t)n1 * kN2);
          dst[0] = make_uint4(Op<T>::pack(v[0], v[1]), Op<T>::pack(v[2], v[3]), Op<T>::pack(v[4], v[5]),
                              Op<T>::pack(v[6], v[7]));
          dst[1] = make_uint4(Op<T>::pack(v[8], v[9]), Op<T>::pack(v[10], v[11]), Op<T>::pack(v[12], v[13]),
                              Op<T>::pack(v[14], v[15]));
        }
      }
    };
    RoundCursor cur = cur0;
    Round Rprev = cur0.get();
    for (int i = 0; i < nloc; ++i, cur.advance()) {
      const Round R = cur.get();
      const int buf = i & 1;
      const bool valid = slot < R.np;
      wait_bar(mbar_a + buf, (uint32_t)(i >> 1) & 1u);
      tc::fence_after_sync();
      float xr[16], xi[16];
      if (valid) {
        const uint32_t ra = tmem + lane_off + (buf ? kTA1 : kTA0);
        float fr[16], fi[16];
        const uint32_t fcol = (uint32_t)(kN2 * R.fidx(slot)), pcol = (uint32_t)(kN2 * (R.nf + slot));
        tc::tmem_ld16x2_wait(ra + fcol, ra + (uint32_t)R.NC + fcol, fr, fi);
        twiddle<false>(fr, fi, twp);
        dft16<false>(fr, fi);
        const float sc = 1.0f / (float)kM, sci = conj_filter ? -sc : sc;  // conj(F^): correlation (input gradient)
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          fr[k] *= sc;
          fi[k] *= sci;
        }
        tc::tmem_ld16x2_wait(ra + pcol, ra + (uint32_t)R.NC + pcol, xr, xi);
        twiddle<false>(xr, xi, twp);
        dft16<false>(xr, xi);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float r = xr[k];
          xr[k] = r * fr[k] - xi[k] * fi[k];
          xi[k] = r * fi[k] + xi[k] * fr[k];
        }
        dft16<true>(xr, xi);
        twiddle<true>(xr, xi, twp);
      }
      // the one Z buffer was read by stage A' of round i - 1, whose completion also releases the
      // previous round's outputs for the epilogue below (stage A' of round i - 1 is issued after
      // that round's arrivals, so this round's arrival cannot fall into the same phase of mbar_z)
      if (i >= 1) {
        wait_bar(mbar_b + (buf ^ 1), (uint32_t)((i - 1) >> 1) & 1u);
        tc::fence_after_sync();
      }
      if (valid) {
        const uint32_t lboZ = (uint32_t)(R.np * kN2 / 8) * 128;  // Z: MN-major, 256 K-rows (re k1 | im k1) x np*16
        uint8_t* z = sm + kOZ + (uint32_t)(2 * slot) * 128 + (uint32_t)(row >> 3) * lboZ +
                     (uint32_t)(row & 7) * 16;
        *reinterpret_cast<uint4*>(z) = make_uint4(Op<T>::pack(xr[0], xr[1]), Op<T>::pack(xr[2], xr[3]),
                                                  Op<T>::pack(xr[4], xr[5]), Op<T>::pack(xr[6], xr[7]));
        *reinterpret_cast<uint4*>(z + 128) = make_uint4(Op<T>::pack(xr[8], xr[9]), Op<T>::pack(xr[10], xr[11]),
                                                        Op<T>::pack(xr[12], xr[13]), Op<T>::pack(xr[14], xr[15]));
        *reinterpret_cast<uint4*>(z + 16 * lboZ) = make_uint4(Op<T>::pack(xi[0], xi[1]), Op<T>::pack(xi[2], xi[3]),
                                                              Op<T>::pack(xi[4], xi[5]), Op<T>::pack(xi[6], xi[7]));
        *reinterpret_cast<uint4*>(z + 16 * lboZ + 128) =
            make_uint4(Op<T>::pack(xi[8], xi[9]), Op<T>::pack(xi[10], xi[11]), Op<T>::pack(xi[12], xi[13]),
                       Op<T>::pack(xi[14], xi[15]));
      }
      // this round's accumulator is read and its Z written; the previous round's outputs
      // (read below) stay in their own accumulator until stage A' of round i + 1
      tc::fence_before_sync();
      tc::fence_smem_to_async();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(mbar_z + buf);
      if (i >= 1) {
        epilogue(Rprev, buf ^ 1);
        tc::fence_before_sync();
      }
      Rprev = R;
    }
    if (nloc > 0) {
      const int last = nloc - 1;
      wait_bar(mbar_b + (last & 1), (uint32_t)(last >> 1) & 1u);
      tc::fence_after_sync();
      epilogue(Rprev, last & 1);
    }
  } else if (filler) {
    // ================= operand warps: round j's operand (operand buffer j % 2) from its staged
    // inputs (staging buffer j % 2), then the copies of round j + 2 into that staging buffer
    float dc0 = 0.f, dc1 = 0.f;  // D of the round being filled (operand thread 0)
    RoundCursor cf = cur0, cl = cur1;  // rounds to fill, to load (two ahead)
    cl.advance();
    if (ft == 0 && nloc > 0) {  // D of round 0; the D of round j + 1 is loaded during round j
      const Round R0 = cur0.get();
      dc0 = __ldg(D + R0.ch(0));
      dc1 = __ldg(D + R0.ch(R0.nf - 1));
    }
    for (int j = 0; j < nloc; ++j) {
      const int sb = j & 1;
      wait_bar(sb ? mbar_ld1 : mbar_ld0, (uint32_t)(j >> 1) & 1u);
      ld_out &= ~(1u << sb);
      if (j >= 2) wait_bar(mbar_a + sb, (uint32_t)((j - 2) >> 1) & 1u);  // stage A of round j - 2 read X[sb]
      const Round Rj = cf.get();
      cf.advance();
      fill_x(Rj, sb, dc0, dc1);
      tc::fence_smem_to_async();
      nbar_sync(1, 32 * (kFillWarps + 1));  // operand of round j complete (the MMA warp waits here)
      if (loader && j + 2 < nloc) {  // every operand thread is past its reads of staging buffer sb
        bool live;
        mark_out(sb, j + 2);
        const Round Rn = cl.get();
        issue_u(Rn, sb, live);
        issue_f(Rn, sb, live);
      }
      cl.advance();
      if (ft == 0 && j + 1 < nloc) {
        const Round Rn = cf.get();
        dc0 = __ldg(D + Rn.ch(0));
        dc1 = __ldg(D + Rn.ch(Rn.nf - 1));
      }
    }
    // copies still in flight (only after a wait that ran out) have landed
    if (loader && (ld_out & 1u)) (void)tc::mbar_wait_bounded(mbar_ld0, ld_par & 1u, kWaitNs);
    if (loader && (ld_out & 2u)) (void)tc::mbar_wait_bounded(mbar_ld1, (ld_par >> 1) & 1u, kWaitNs);
  } else if (mma_warp) {
    // ================= MMA warp: stage A of round j + 1 once its operand is filled, stage A' of
    // round j once the register pass is done
    auto issue_a = [&](const Round& R, int buf) {  // D = C [Xr | Xi] + S [Xi | -Xr] = [Yr | Yi]
      if (aborted()) {
        tc::mbar_arrive(mbar_a + buf);
        return;
      }
      const uint32_t lbo = (uint32_t)(3 * R.NC / 8) * 128;
      const uint32_t idA = tc::idesc_f16(128, 2 * R.NC, Op<T>::bf16, 0, 1);
      const uint32_t dA = tmem + (buf ? kTA1 : kTA0);
      const uint32_t xa = s0 + kOX + (uint32_t)buf * kXBytes;
      const uint64_t b0 = tc::desc_kmajor(xa, lbo, 128);
      const uint64_t b1 = tc::desc_kmajor(xa + (uint32_t)(R.NC / 8) * 128, lbo, 128);
      const uint64_t step = (uint64_t)((2 * lbo) >> 4);  // next 16 K-rows (address field in 16-byte units)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc::mma_f16_tmem_a(dA, tmem + kTConst + (uint32_t)(8 * kk), b0 + kk * step, idA, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc::mma_f16_tmem_a(dA, tmem + kTConst + 32u + (uint32_t)(8 * kk), b1 + kk * step, idA, 1u);
      tc::mma_commit(mbar_a + buf);
    };
    auto issue_a2 = [&](const Round& R, int buf) {  // y = CA^T Zr + CB^T Zi
      if (aborted()) {
        tc::mbar_arrive(mbar_b + buf);
        return;
      }
      const uint32_t lboZ = (uint32_t)(R.np * kN2 / 8) * 128;
      const uint32_t idB = tc::idesc_f16(128, R.np * kN2, Op<T>::bf16, 1, 1);
      const uint32_t zr = s0 + kOZ;
      const uint64_t a0 = tc::desc_kmajor(ca, kCSbo, kCLbo), a1 = tc::desc_kmajor(cb, kCSbo, kCLbo);
      const uint64_t z0 = tc::desc_kmajor(zr, lboZ, 128), z1 = tc::desc_kmajor(zr + 16 * lboZ, lboZ, 128);
      const uint64_t astep = (uint64_t)((2 * kCSbo) >> 4), zstep = (uint64_t)((2 * lboZ) >> 4);
      const uint32_t dB = tmem + (buf ? kTB1 : kTB0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) tc::mma_f16(dB, a0 + kk * astep, z0 + kk * zstep, idB, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) tc::mma_f16(dB, a1 + kk * astep, z1 + kk * zstep, idB, 1u);
      tc::mma_commit(mbar_b + buf);
    };
    RoundCursor ca_ = cur0, cz = cur0;  // rounds for stage A, for stage A'
    for (int j = 0; j <= nloc; ++j) {
      if (j < nloc) {  // stage A of round j
        nbar_sync(1, 32 * (kFillWarps + 1));
        if (issuer) {
          tc::fence_after_sync();
          issue_a(ca_.get(), j & 1);
        }
        ca_.advance();
      }
      if (j >= 1 && issuer) {  // stage A' of round j - 1
        wait_bar(mbar_z + ((j - 1) & 1), (uint32_t)((j - 1) >> 1) & 1u);
        tc::fence_after_sync();
        issue_a2(cz.get(), (j - 1) & 1);
        cz.advance();
      }
      __syncwarp();
    }
    if (issuer) {  // drain: every MMA issued here has completed
      tc::mma_commit(mbar_fin);
      (void)tc::mbar_wait_bounded(mbar_fin, 0, kWaitNs);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

template <typename T>
static cudaError_t fftconv_tc_t(const void* u, const float* f, const float* D, void* y, int B, int H, bool pdl,
                                cudaStream_t st, bool conj_filter) {
  cudaError_t e = smem_optin<fftconv_tc_kernel<T>>(kSmem);
  if (e != cudaSuccess) return e;
  const long long rounds = ((long long)H * ((B + 1) / 2) + kSlots - 1) / kSlots;
  const int sms = num_sms();
  const int grid = (int)(rounds < sms ? rounds : sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThr);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fftconv_tc_kernel<T>, (const T*)u, f, D, (T*)y, B, H, conj_filter ? 1 : 0);
}

bool fftconv_tc_supported(int L, int dtype, int B) { return L == kL && (dtype == 1 || dtype == 2) && B >= 3; }

cudaError_t launch_fftconv_tc(const void* u, const float* f, const float* D, void* y, int B, int H, int L, int dtype,
                              bool after_filter_kernel, cudaStream_t st, bool conj_filter) {
  if (!fftconv_tc_supported(L, dtype, B)) return cudaErrorInvalidValue;
  return dtype == 1 ? fftconv_tc_t<__half>(u, f, D, y, B, H, after_filter_kernel, st, conj_filter)
                    : fftconv_tc_t<__nv_bfloat16>(u, f, D, y, B, H, after_filter_kernel, st, conj_filter);
}

unsigned int fftconv_tc_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_fftconv_tc_timeouts, sizeof(v));
  return v;
}

}  // namespace fc
