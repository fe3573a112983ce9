// Diagonal-SSM filter generation (A1):
//   f[h,k] = 2 Re sum_n C[h,n] B[h,n] A[h,n]^k,  A = exp(dt * lambda)
// (H3 blog "The Convolution Connection": f = [CB, CAB, CA^2B, ...]).
//
// Two kernels: for N <= 64 a tensor-core GEMM per 2048 taps (below); for
// larger N a CUDA-core kernel in which one CTA evaluates 1024 taps of one
// channel with the factored tables of ssm_tables.cuh (a real contraction over
// the modes, blocks of 64 modes).
#include "kernels.cuh"

#include "ssm_tables.cuh"
#include "tc100.cuh"

namespace fc {

constexpr int kGenTile = 1024;    // taps per CTA
constexpr int kGenThreads = 128;
constexpr int kGenMB = 64;        // modes per table block
constexpr int kGenKH = kGenTile / 64;  // 16
constexpr size_t kGenSmem = sizeof(float2) * ((size_t)kGenMB * 64 + (size_t)kGenKH * kGenMB +
                                              (size_t)kGenMB * ssm_scratch_per_mode(kGenKH));

// Thread t owns taps e in {2(t%32), 2(t%32)+1} x kh in {4(t/32) .. 4(t/32)+3}:
// per mode one 16-byte Q load (two consecutive e) and four broadcast 8-byte W
// loads (the warp shares its kh group) feed 16 FMAs.
__global__ void __launch_bounds__(kGenThreads) ssm_gen_kernel(const float* __restrict__ dt,
                                                             const float2* __restrict__ lam,
                                                             const float2* __restrict__ Bp,
                                                             const float2* __restrict__ Cp, int H, int N,
                                                             int L, float* __restrict__ f) {
  asm volatile("griddepcontrol.launch_dependents;");  // see ssm_gen_tc_kernel
  extern __shared__ __align__(16) float2 gsm[];
  float2* Q = gsm;                       // [m][64]
  float2* Wt = Q + kGenMB * 64;          // [kh][kGenMB] as written by ssm_fill_tables
  float2* X = Wt + kGenKH * kGenMB;      // scratch
  const int h = blockIdx.y;
  const long long k0 = (long long)blockIdx.x * kGenTile;
  const int ntap = (int)min((long long)kGenTile, (long long)L - k0);
  const int KH = (ntap + 63) >> 6;
  const int lane = threadIdx.x & 31;
  const int g = threadIdx.x >> 5;  // kh group 0..3
  float acc[2][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
  for (int m0 = 0; m0 < N; m0 += kGenMB) {
    const int mb = min(kGenMB, N - m0);
    __syncthreads();  // previous block's readers are done
    ssm_fill_tables(dt, lam, Bp, Cp, h, N, m0, mb, kGenMB, k0, KH, Q, Wt, X, threadIdx.x, kGenThreads);
    for (int m = 0; m < mb; ++m) {
      const float4 q = *reinterpret_cast<const float4*>(Q + m * 64 + 2 * lane);
      float2 w[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int kh = 4 * g + c;
        w[c] = kh < KH ? Wt[kh * kGenMB + m] : make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[0][c] = fmaf(w[c].x, q.x, fmaf(-w[c].y, q.y, acc[0][c]));
        acc[1][c] = fmaf(w[c].x, q.z, fmaf(-w[c].y, q.w, acc[1][c]));
      }
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int k = 64 * (4 * g + c) + 2 * lane + a;
      if (k < ntap && FC_OK_IDX(20, (long long)h * L + k0 + k, (long long)H * L)) f[(size_t)h * L + k0 + k] = acc[a][c];
    }
}

// ---------------------------------------------------------------- tensor-core variant (N <= 64)
// With t = 16 th + tl (tl < 16) the filter is one real GEMM per 2048 taps:
//   f[16 th + tl] = sum_k AH[th][k] Q[tl][k]        (M = 128 rows th, N = 16, K = 128)
//   AH[th][2n] + i AH[th][2n+1] = A_n^(16 th)
//   Q[tl][2n]  - i Q[tl][2n+1]  = 2 C_n B_n A_n^tl   (scaled by a power of two)
// Both tables are split into fp16 high and remainder parts (three MMAs,
// about 22 significant bits).  AH[th] = A^(16 th0) A^(128 g) A^(16 m) for
// th = th0 + 8 g + m; A^(16 th0) is an exactly phase-reduced power, the other
// factors at most 7 products of the exact powers A, A^4, A^16, A^128, A^512.  One CTA owns up to kGUnits consecutive 2048-tap units
// of one channel and builds Q once.
static __device__ unsigned int g_gen_tc_timeouts;

namespace {
constexpr int kGThr = 256;
constexpr int kGUnits = 4;
constexpr int kGRows = 128, kGNC = 16, kGUnitTaps = kGRows * kGNC;
constexpr uint32_t kGLbo = 144, kGSbo = 16 * 144;  // padded K-major, K = 128
constexpr uint32_t kGTab = (kGRows / 8) * kGSbo;
constexpr uint32_t kGQ = (kGNC / 8) * kGSbo;
constexpr uint64_t kGWaitNs = 2000000000ull;
// Shared-memory layout (byte offsets).  With at most 64 rows (L <= 1024,
// SHORT) the rows 64..127 that the M = 128 MMA reads past each AH tile are
// never stored, so those reads may land on the next tile: the tiles then take
// 18 KB each instead of 36 KB and four CTAs fit on an SM.  The control words
// sit past every byte an MMA reads.
// COMPACT (SHORT with single tables): no remainder tables, and Q and the exact
// powers sit in the never-stored stretch of the AH tile, which leaves 36 KB per
// CTA (six CTAs of 128 threads per SM).
template <bool SHORT, bool COMPACT = false>
struct GenLayout {
  static constexpr uint32_t tab = SHORT ? kGTab / 2 : kGTab;
  static constexpr uint32_t ahh = 0, ahl = COMPACT ? 0 : tab, qh = COMPACT ? tab : 2 * tab,
                            ql = COMPACT ? qh : qh + kGQ;
  static constexpr uint32_t mma_end = COMPACT ? kGTab : ((ahl + kGTab > ql + kGQ) ? ahl + kGTab : ql + kGQ);
  // exact powers A, A^4, A^16, A^128, A^512 per mode; in SHORT they sit in the
  // stretch that only feeds never-stored rows
  static constexpr uint32_t pw = SHORT ? (COMPACT ? qh + kGQ : ql + kGQ) : mma_end;
  // the control words sit past every byte an MMA reads
  static constexpr uint32_t red = COMPACT ? mma_end : pw + 64 * 5 * 8, mbar = red + 32, tmem = mbar + 8;
  static constexpr uint32_t bytes = (tmem + 8 > mma_end) ? tmem + 8 : mma_end;
  static_assert(!COMPACT || pw + 64 * 5 * 8 <= kGTab, "COMPACT: Q and the powers inside the AH tile's extent");
};
__device__ __forceinline__ uint32_t gsplit(float a, float b, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
  lo = *reinterpret_cast<const uint32_t*>(&l);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t goff(int r, int n) {  // K elements (2n, 2n+1) of row r
  return (uint32_t)(r >> 3) * kGSbo + (uint32_t)(n >> 2) * kGLbo + (uint32_t)(r & 7) * 16u + (uint32_t)(n & 3) * 4u;
}
}  // namespace

// THR = 128 (SHORT with single tables): each thread covers two row-group
// phases, so that all of a 768-channel launch fits one wave of CTAs.
template <bool SHORT, bool HI, int THR = kGThr>
__global__ void __launch_bounds__(THR, THR == 128 ? 6 : (SHORT ? 4 : 2)) ssm_gen_tc_kernel(const float* __restrict__ dt,
                                                                          const float2* __restrict__ lam,
                                                                          const float2* __restrict__ Bp,
                                                                          const float2* __restrict__ Cp, int H, int N,
                                                                          int L, float* __restrict__ f) {
  // a convolution launched as this kernel's programmatic dependent may start
  // its prologue now; it reads f only after this grid has completed
  asm volatile("griddepcontrol.launch_dependents;");
  static_assert(THR == kGThr || (THR == 128 && SHORT && HI), "128 threads only for short single-table rows");
  using LY = GenLayout<SHORT, THR == 128>;
  constexpr int NG = SHORT ? 2 : 4;  // row groups g = gq + 4 r a phase gq may fill
  constexpr int NV = kGThr / THR;     // row-group phases per thread: gq = tid / 64 + 2 v
  extern __shared__ __align__(1024) uint8_t gtsm[];
  struct {
    uint8_t* ahh;
    uint8_t* ahl;
    uint8_t* qh;
    uint8_t* ql;
    float2* pw;
    float* red;
    uint64_t* mbar;
    uint32_t* tmem_p;
  } sm{gtsm + LY::ahh, gtsm + LY::ahl, gtsm + LY::qh, gtsm + LY::ql, reinterpret_cast<float2*>(gtsm + LY::pw),
       reinterpret_cast<float*>(gtsm + LY::red), reinterpret_cast<uint64_t*>(gtsm + LY::mbar),
       reinterpret_cast<uint32_t*>(gtsm + LY::tmem)};
  const int h = blockIdx.y;
  const int units = (L + kGUnitTaps - 1) / kGUnitTaps;
  const int u0 = blockIdx.x * kGUnits, u1 = min(units, u0 + kGUnits);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int n = tid & 63, gq0 = tid >> 6;  // this thread's mode and first row-group phase
  const float d = dt[h];
  if (warp == 0) tc::tmem_alloc(sm.tmem_p, 32);
  if (tid == 0) {
    tc::mbar_init(sm.mbar, 1);
    tc::fence_mbar_init();
  }
  // exact powers, five per mode, spread over the CTA
  for (int idx = tid; idx < 64 * 5; idx += THR) {
    const int m = idx / 5, e = idx - 5 * m;
    float2 v = make_float2(0.f, 0.f);
    if (m < N) {
      const float2 l = lam[(size_t)h * N + m];
      v = ssm_pow(d, l.x, l.y, e == 0 ? 1.0 : e == 1 ? 4.0 : e == 2 ? 16.0 : e == 3 ? 128.0 : 512.0);
    }
    sm.pw[idx] = v;
  }
  float2 lm = make_float2(0.f, 0.f), w = make_float2(0.f, 0.f);
  if (n < N) {
    lm = lam[(size_t)h * N + n];
    const float2 cb = cmul(Cp[(size_t)h * N + n], Bp[(size_t)h * N + n]);
    w = make_float2(2.f * cb.x, 2.f * cb.y);
  }
  // power-of-two scale: the largest |Re|, |Im| of any 2 C B just below 2^13
  float mx = fmaxf(fabsf(w.x), fabsf(w.y));
  mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
  if ((tid & 31) == 0) sm.red[warp] = mx;
  __syncthreads();
  mx = 0.f;
#pragma unroll
  for (int i = 0; i < THR / 32; ++i) mx = fmaxf(mx, sm.red[i]);
  float scale = 1.f, inv = 1.f;
  if (mx > 0.f && mx <= 3.0e38f) {
    int ex = 0;
    (void)frexpf(mx, &ex);
    scale = ldexpf(1.f, 13 - ex);
    inv = ldexpf(1.f, ex - 13);
  }
  // this thread's factors: A^(16 m) (m < 8), A^(128 (gq + 4 r)), A^(4 gq); each at
  // most 7 products of exact powers (zero for padding modes)
  const float2 a1 = sm.pw[n * 5 + 0], a4 = sm.pw[n * 5 + 1], a16 = sm.pw[n * 5 + 2];
  const float2 a128 = sm.pw[n * 5 + 3], a512 = sm.pw[n * 5 + 4];
  const float2 one = n < N ? make_float2(1.f, 0.f) : make_float2(0.f, 0.f);
  float2 m8[8], G[NV][NG];
  m8[0] = one;
#pragma unroll
  for (int m = 1; m < 8; ++m) m8[m] = cmul(m8[m - 1], a16);
#pragma unroll
  for (int vv = 0; vv < NV; ++vv) {
    const int gq = gq0 + 2 * vv;
    float2 g128 = one, p4 = one;
#pragma unroll
    for (int i = 0; i < 3; ++i)
      if (i < gq) {
        g128 = cmul(g128, a128);
        p4 = cmul(p4, a4);
      }
    G[vv][0] = g128;
#pragma unroll
    for (int r = 1; r < NG; ++r) G[vv][r] = cmul(G[vv][r - 1], a512);
    // Q rows tl = 4 gq .. 4 gq + 3
    float2 p = cmul(make_float2(w.x * scale, w.y * scale), p4);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t lo;
      const uint32_t hi = gsplit(p.x, -p.y, lo);
      *reinterpret_cast<uint32_t*>(sm.qh + goff(4 * gq + j, n)) = hi;
      if constexpr (!HI) *reinterpret_cast<uint32_t*>(sm.ql + goff(4 * gq + j, n)) = lo;
      p = cmul(p, a1);
    }
  }
  const uint32_t idesc = tc::idesc_f16(kGRows, kGNC, 0);
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const bool vec_ok = (L & 3) == 0;
  uint32_t phase = 0;
  bool failed = false;
  for (int u = u0; u < u1; ++u) {
    const int th0 = u * kGRows;
    const int rows = min(kGRows, (L - th0 * kGNC + kGNC - 1) / kGNC);
    const float2 base = n >= N ? make_float2(0.f, 0.f)
                        : th0 == 0 ? make_float2(1.f, 0.f) : ssm_pow(d, lm.x, lm.y, 16.0 * th0);
#pragma unroll
    for (int vr = 0; vr < NV * NG; ++vr) {
      const int vv = vr / NG, r = vr - vv * NG;
      const int g = gq0 + 2 * vv + 4 * r;
      if (8 * g >= rows) continue;  // rows past the end are never stored
      const float2 pg = cmul(base, G[vv][r]);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float2 v = cmul(pg, m8[m]);
        uint32_t lo;
        const uint32_t hi = gsplit(v.x, v.y, lo);
        *reinterpret_cast<uint32_t*>(sm.ahh + goff(8 * g + m, n)) = hi;
        if constexpr (!HI) *reinterpret_cast<uint32_t*>(sm.ahl + goff(8 * g + m, n)) = lo;
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *sm.tmem_p;
    if (tid == 0) {
      const uint32_t ah = tc::smem_u32(sm.ahh), al = tc::smem_u32(sm.ahl);
      const uint32_t qh = tc::smem_u32(sm.qh), ql = tc::smem_u32(sm.ql);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(ah + kk * 2 * kGLbo, kGLbo, kGSbo),
                    tc::desc_kmajor(qh + kk * 2 * kGLbo, kGLbo, kGSbo), idesc, kk > 0 ? 1u : 0u);
      if constexpr (!HI) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_f16(tmem, tc::desc_kmajor(ah + kk * 2 * kGLbo, kGLbo, kGSbo),
                      tc::desc_kmajor(ql + kk * 2 * kGLbo, kGLbo, kGSbo), idesc, 1u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_f16(tmem, tc::desc_kmajor(al + kk * 2 * kGLbo, kGLbo, kGSbo),
                      tc::desc_kmajor(qh + kk * 2 * kGLbo, kGLbo, kGSbo), idesc, 1u);
      }
      tc::mma_commit(sm.mbar);
    }
    const bool ok = tc::mbar_wait_bounded(sm.mbar, phase, kGWaitNs);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    if (warp < 4) {
      float v[16];
      tc::tmem_ld16_wait(tmem + lane_off, v);
      const int r = tid;  // TMEM lane = row
      if (r < rows) {
        const long long t0 = (long long)(th0 + r) * kGNC;
        float* fp = f + (size_t)h * L + t0;
        if (vec_ok && t0 + kGNC <= L) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            reinterpret_cast<float4*>(fp)[q] =
                make_float4(v[4 * q] * inv, v[4 * q + 1] * inv, v[4 * q + 2] * inv, v[4 * q + 3] * inv);
        } else {
#pragma unroll
          for (int j = 0; j < kGNC; ++j)
            if (t0 + j < L) fp[j] = v[j] * inv;
        }
      }
    }
  }
  if (failed && tid == 0) atomicAdd(&g_gen_tc_timeouts, 1u);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(*sm.tmem_p, 32);
}

// Long filters (L > 2048): 64-tap rows, t = 64 th + tl (tl < 64), one GEMM per 8192 taps,
//   f[64 th + tl] = sum_k AH[th][k] Q[tl][k]        (M = 128 rows th, N = 64, K = 128)
//   AH[th][2n] + i AH[th][2n+1] = A_n^(64 th),  Q[tl][2n] - i Q[tl][2n+1] = 2 C_n B_n A_n^tl,
// split hi/lo as above.  Four times the taps per MMA group and per table of the 16-tap form, so
// the tables, the 24 MMAs and the waits are paid once per 8192 taps instead of per 2048.
// AH[th] = A^(8192 u) A^(2048 r) A^(512 gq) A^(64 m) for th = 8 (gq + 4 r) + m (exact powers A,
// A^16, A^64, A^512, A^2048; at most 7 products each); Q[tl] = w A^(16 gq) A^j, tl = 16 gq + j.
namespace {
constexpr int kG64Units = 2;                    // 8192-tap units per CTA
constexpr int kG64Cols = 64, kG64UnitTaps = kGRows * kG64Cols;
constexpr uint32_t kG64Q = (kG64Cols / 8) * kGSbo;
// COMPACT (single tables): no remainder tables, 58 KB, three CTAs of 128 threads per SM.
template <bool COMPACT = false>
struct Gen64Layout {
  static constexpr uint32_t ahh = 0, ahl = COMPACT ? 0 : kGTab, qh = COMPACT ? kGTab : 2 * kGTab,
                            ql = COMPACT ? qh : qh + kG64Q, pw = ql + kG64Q;
  static constexpr uint32_t red = pw + 64 * 5 * 8, mbar = red + 32, tmem = mbar + 8, bytes = tmem + 8;
};
}  // namespace

// THR = 128 (single tables): each thread covers two row-group phases, so three
// CTAs fit an SM.
template <bool HI, int THR = kGThr>
__global__ void __launch_bounds__(THR, THR == 128 ? 3 : 2) ssm_gen_tc64_kernel(const float* __restrict__ dt,
                                                                const float2* __restrict__ lam,
                                                                const float2* __restrict__ Bp,
                                                                const float2* __restrict__ Cp, int H, int N, int L,
                                                                float* __restrict__ f) {
  asm volatile("griddepcontrol.launch_dependents;");  // see ssm_gen_tc_kernel
  static_assert(THR == kGThr || (THR == 128 && HI), "128 threads only with single tables");
  using LY = Gen64Layout<THR == 128>;
  constexpr int NV = kGThr / THR;  // row-group phases per thread: gq = tid / 64 + 2 v
  extern __shared__ __align__(1024) uint8_t gtsm[];
  uint8_t* ahh = gtsm + LY::ahh;
  uint8_t* ahl = gtsm + LY::ahl;
  uint8_t* qh = gtsm + LY::qh;
  uint8_t* ql = gtsm + LY::ql;
  float2* pw = reinterpret_cast<float2*>(gtsm + LY::pw);
  float* red = reinterpret_cast<float*>(gtsm + LY::red);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(gtsm + LY::mbar);
  uint32_t* tmem_p = reinterpret_cast<uint32_t*>(gtsm + LY::tmem);
  const int h = blockIdx.y;
  const int units = (L + kG64UnitTaps - 1) / kG64UnitTaps;
  const int u0 = blockIdx.x * kG64Units, u1 = min(units, u0 + kG64Units);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int n = tid & 63, gq0 = tid >> 6;  // this thread's mode and first row-group phase
  const float d = dt[h];
  if (warp == 0) tc::tmem_alloc(tmem_p, 64);
  if (tid == 0) {
    tc::mbar_init(mbar, 1);
    tc::fence_mbar_init();
  }
  for (int idx = tid; idx < 64 * 5; idx += THR) {
    const int m = idx / 5, e = idx - 5 * m;
    float2 v = make_float2(0.f, 0.f);
    if (m < N) {
      const float2 l = lam[(size_t)h * N + m];
      v = ssm_pow(d, l.x, l.y, e == 0 ? 1.0 : e == 1 ? 16.0 : e == 2 ? 64.0 : e == 3 ? 512.0 : 2048.0);
    }
    pw[idx] = v;
  }
  float2 lm = make_float2(0.f, 0.f), w = make_float2(0.f, 0.f);
  if (n < N) {
    lm = lam[(size_t)h * N + n];
    const float2 cb = cmul(Cp[(size_t)h * N + n], Bp[(size_t)h * N + n]);
    w = make_float2(2.f * cb.x, 2.f * cb.y);
  }
  // power-of-two scale: the largest |Re|, |Im| of any 2 C B just below 2^13
  float mx = fmaxf(fabsf(w.x), fabsf(w.y));
  mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
  if ((tid & 31) == 0) red[warp] = mx;
  __syncthreads();
  mx = 0.f;
#pragma unroll
  for (int i = 0; i < THR / 32; ++i) mx = fmaxf(mx, red[i]);
  float scale = 1.f, inv = 1.f;
  if (mx > 0.f && mx <= 3.0e38f) {
    int ex = 0;
    (void)frexpf(mx, &ex);
    scale = ldexpf(1.f, 13 - ex);
    inv = ldexpf(1.f, ex - 13);
  }
  const float2 a1 = pw[n * 5 + 0], a16 = pw[n * 5 + 1], a64 = pw[n * 5 + 2];
  const float2 a512 = pw[n * 5 + 3], a2048 = pw[n * 5 + 4];
  const float2 one = n < N ? make_float2(1.f, 0.f) : make_float2(0.f, 0.f);
  float2 m8[8], G[NV][4];
  m8[0] = one;
#pragma unroll
  for (int m = 1; m < 8; ++m) m8[m] = cmul(m8[m - 1], a64);
#pragma unroll
  for (int vv = 0; vv < NV; ++vv) {
    const int gq = gq0 + 2 * vv;
    float2 g512 = one, p16 = one;
#pragma unroll
    for (int i = 0; i < 3; ++i)
      if (i < gq) {
        g512 = cmul(g512, a512);
        p16 = cmul(p16, a16);
      }
    G[vv][0] = g512;
#pragma unroll
    for (int r = 1; r < 4; ++r) G[vv][r] = cmul(G[vv][r - 1], a2048);
    // Q rows tl = 16 gq .. 16 gq + 15
    float2 p = cmul(make_float2(w.x * scale, w.y * scale), p16);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      uint32_t lo;
      const uint32_t hi = gsplit(p.x, -p.y, lo);
      *reinterpret_cast<uint32_t*>(qh + goff(16 * gq + j, n)) = hi;
      if constexpr (!HI) *reinterpret_cast<uint32_t*>(ql + goff(16 * gq + j, n)) = lo;
      p = cmul(p, a1);
    }
  }
  const uint32_t idesc = tc::idesc_f16(kGRows, kG64Cols, 0);
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const int half0 = warp >> 2;  // output columns 32 half .. 32 half + 31 (both halves with 128 threads)
  const bool vec_ok = (L & 3) == 0;
  uint32_t phase = 0;
  bool failed = false;
  for (int u = u0; u < u1; ++u) {
    const int th0 = u * kGRows;
    const int rows = min(kGRows, (L - th0 * kG64Cols + kG64Cols - 1) / kG64Cols);
    const float2 base = n >= N ? make_float2(0.f, 0.f)
                        : th0 == 0 ? make_float2(1.f, 0.f) : ssm_pow(d, lm.x, lm.y, 64.0 * th0);
    if (u > u0) {  // the previous unit's MMAs have read the tables (its wait is behind us)
      tc::fence_before_sync();
      __syncthreads();
    }
#pragma unroll
    for (int vr = 0; vr < NV * 4; ++vr) {
      const int vv = vr / 4, r = vr - 4 * vv;
      const int g = gq0 + 2 * vv + 4 * r;
      const float2 pg = cmul(base, G[vv][r]);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        // rows past the end feed only never-stored outputs: zero them
        const float2 v = 8 * g + m < rows ? cmul(pg, m8[m]) : make_float2(0.f, 0.f);
        uint32_t lo;
        const uint32_t hi = gsplit(v.x, v.y, lo);
        *reinterpret_cast<uint32_t*>(ahh + goff(8 * g + m, n)) = hi;
        if constexpr (!HI) *reinterpret_cast<uint32_t*>(ahl + goff(8 * g + m, n)) = lo;
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_p;
    if (tid == 0) {
      const uint32_t ah = tc::smem_u32(ahh), al = tc::smem_u32(ahl);
      const uint32_t bh = tc::smem_u32(qh), bl = tc::smem_u32(ql);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(ah + kk * 2 * kGLbo, kGLbo, kGSbo),
                    tc::desc_kmajor(bh + kk * 2 * kGLbo, kGLbo, kGSbo), idesc, kk > 0 ? 1u : 0u);
      if constexpr (!HI) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_f16(tmem, tc::desc_kmajor(ah + kk * 2 * kGLbo, kGLbo, kGSbo),
                      tc::desc_kmajor(bl + kk * 2 * kGLbo, kGLbo, kGSbo), idesc, 1u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_f16(tmem, tc::desc_kmajor(al + kk * 2 * kGLbo, kGLbo, kGSbo),
                      tc::desc_kmajor(bh + kk * 2 * kGLbo, kGLbo, kGSbo), idesc, 1u);
      }
      tc::mma_commit(mbar);
    }
    const bool ok = tc::mbar_wait_bounded(mbar, phase, kGWaitNs);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
#pragma unroll 1
    for (int half = half0; half < 2; half += 2 / NV) {
    float v[32];
    tc::tmem_ld16x2_wait(tmem + lane_off + (uint32_t)(32 * half), tmem + lane_off + (uint32_t)(32 * half + 16), v,
                         v + 16);
    const int r = (warp & 3) * 32 + (tid & 31);  // TMEM lane = row
    if (r < rows) {
      const long long t0 = (long long)(th0 + r) * kG64Cols + 32 * half;
      float* fp = f + (size_t)h * L + t0;
      if (vec_ok && t0 + 32 <= L) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          reinterpret_cast<float4*>(fp)[q] =
              make_float4(v[4 * q] * inv, v[4 * q + 1] * inv, v[4 * q + 2] * inv, v[4 * q + 3] * inv);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (t0 + j < L) fp[j] = v[j] * inv;
      }
    }
    }
  }
  if (failed && tid == 0) atomicAdd(&g_gen_tc_timeouts, 1u);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(*tmem_p, 64);
}

unsigned int gen_tc_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_gen_tc_timeouts, sizeof(v));
  return v;
}

template <bool HI>
static cudaError_t gen_tc(const float* dt, const float* lam, const float* Bp, const float* Cp, int H, int N, int L,
                          float* f, cudaStream_t st) {
  const float2* l2 = reinterpret_cast<const float2*>(lam);
  const float2* b2 = reinterpret_cast<const float2*>(Bp);
  const float2* c2 = reinterpret_cast<const float2*>(Cp);
  if (L > 2 * kGUnitTaps) {
    const int units = (L + kG64UnitTaps - 1) / kG64UnitTaps;
    dim3 grid((units + kG64Units - 1) / kG64Units, H);
    if constexpr (HI) {  // 128-thread CTAs in the compact layout
      constexpr size_t csm = Gen64Layout<true>::bytes;
      cudaError_t e = smem_optin<ssm_gen_tc64_kernel<true, 128>>(csm);
      if (e != cudaSuccess) return e;
      ssm_gen_tc64_kernel<true, 128><<<grid, 128, csm, st>>>(dt, l2, b2, c2, H, N, L, f);
      return cudaGetLastError();
    }
    cudaError_t e = smem_optin<ssm_gen_tc64_kernel<HI>>(Gen64Layout<>::bytes);
    if (e != cudaSuccess) return e;
    ssm_gen_tc64_kernel<HI><<<grid, kGThr, Gen64Layout<>::bytes, st>>>(dt, l2, b2, c2, H, N, L, f);
    return cudaGetLastError();
  }
  const int units = (L + kGUnitTaps - 1) / kGUnitTaps;
  const bool short_rows = L <= kGUnitTaps / 2;
  if constexpr (HI) {
    if (short_rows) {  // 128-thread CTAs in the compact layout
      constexpr size_t csm = GenLayout<true, true>::bytes;
      cudaError_t e = smem_optin<ssm_gen_tc_kernel<true, true, 128>>(csm);
      if (e != cudaSuccess) return e;
      ssm_gen_tc_kernel<true, true, 128><<<dim3((units + kGUnits - 1) / kGUnits, H), 128, csm, st>>>(dt, l2, b2, c2, H,
                                                                                                   N, L, f);
      return cudaGetLastError();
    }
  }
  auto kern = short_rows ? ssm_gen_tc_kernel<true, HI> : ssm_gen_tc_kernel<false, HI>;
  const size_t smem = short_rows ? GenLayout<true>::bytes : GenLayout<false>::bytes;
  cudaError_t e = short_rows ? smem_optin<ssm_gen_tc_kernel<true, HI>>(smem)
                             : smem_optin<ssm_gen_tc_kernel<false, HI>>(smem);
  if (e != cudaSuccess) return e;
  dim3 grid((units + kGUnits - 1) / kGUnits, H);
  kern<<<grid, kGThr, smem, st>>>(dt, l2, b2, c2, H, N, L, f);
  return cudaGetLastError();
}

cudaError_t launch_ssm_gen(const float* dt, const float* lam, const float* Bp, const float* Cp, int H, int N,
                           int L, float* f, cudaStream_t st, bool hi_only) {
  if (N <= 64)
    return hi_only ? gen_tc<true>(dt, lam, Bp, Cp, H, N, L, f, st) : gen_tc<false>(dt, lam, Bp, Cp, H, N, L, f, st);

  const int tiles = (L + kGenTile - 1) / kGenTile;
  cudaError_t e = smem_optin<ssm_gen_kernel>(kGenSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(tiles, H);
  ssm_gen_kernel<<<grid, kGenThreads, kGenSmem, st>>>(dt, reinterpret_cast<const float2*>(lam),
                                                      reinterpret_cast<const float2*>(Bp),
                                                      reinterpret_cast<const float2*>(Cp), H, N, L, f);
  return cudaGetLastError();
}

}  // namespace fc

FC_CHECK_READER(fc_check_ssm_gen)
