// Fused FFT convolution with block-FFT stages on the 5th-generation tensor
// cores (fp16 / bf16 I/O, L = 1024, i.e. M = 2L = 2048 = 128 x 16).
//
// H3 summary section 4 "Short-sequence computation": FFT, pointwise multiply
// and inverse FFT fused in one kernel, with the block FFT written as matrix
// multiplies so that it runs on the tensor cores (H3 blog, "Fused Block
// FFTConv").  Index split n = 16 n1 + n2, k = k1 + 128 k2 (n1, k1 < 128,
// n2, k2 < 16), w_K = exp(-2 pi i / K):
//   stage A   (GEMM)  Y[k1,n2]  = sum_{n1<64} w_128^(n1 k1) x[16 n1 + n2]   (n1 >= 64: zero padding)
//   registers         Y'        = Y w_2048^(k1 n2) / 32                      (fp16 tile, K = re|im n2)
//   stage B   (GEMM)  X^[k1,k2] = sum_n2 w_16^(n2 k2) Y'[k1,n2]              (32 x 32 real DFT-16 block)
//   registers         V         = X^ . 32 F^ / M                             (fp16 tile, K = re|im k2)
//   stage B'  (GEMM)  W[k1,n2]  = sum_k2 w_16^(-n2 k2) V[k1,k2]
//   registers         Z         = W w_2048^(-k1 n2)
//   stage A'  (GEMM)  y[16 n1 + n2] = sum_{k1} w_128^(-n1 k1) Z[k1, n2],      n1 < 64
// (X^[k1 + 128 k2] is the 2048-point transform; F^ that of the filter, which
// goes through stages A and B as one more sequence.)  Complex products are
// split into real GEMMs with fp32 accumulation in TMEM.  Two constant 128x128
// matrices hold the real DFT-128 blocks,
//   CA[k1][j] = j<64 ?  cos(2 pi k1 j/128) : sin(2 pi k1 (j-64)/128)
//   CB[k1][j] = j<64 ? -sin(2 pi k1 j/128) : cos(2 pi k1 (j-64)/128)
// read K-major by stage A and (the DFT matrix being symmetric) MN-major by
// stage A':
//   stage A : Yr = CA[:, :64] Xr + CA[:, 64:] Xi,   Yi = CA[:, :64] Xi + CB[:, :64] Xr
//   stage A': rows j<64 give Re y[n1=j], rows j>=64 give Im y[n1=j-64]:
//             y = CA^T Zr + CB^T Zi
// and two 32x32 fp16 blocks the forward and inverse DFT-16 (stages B, B').
// Stage-B operands are always fp16 (scaled by 1/32 so that |Y'| <= 2 max|u|);
// stages A and A' use the I/O type.
// One CTA takes one channel at a time: its filter and up to 4 row pairs (two
// real rows packed as one complex sequence u0 + i u1; f is real, so the real
// and imaginary outputs are the two convolutions) form one batch of
// N = 16 x (1 + pairs) stage-A columns.  The CTA has two groups of four warps
// (each group covers the four TMEM lane quarters, thread row k1 = tid % 128);
// the register passes alternate sequences between the groups, and every
// thread keeps its row's 16 filter bins in registers for the whole channel.
// The next work item's inputs are copied in with cp.async during the
// epilogue.  Waits on MMA completion are bounded; a CTA that gives up records
// it in a device counter, skips its remaining work and frees its TMEM.
#include "fft_stockham.cuh"
#include "kernels.cuh"
#include "tc100.cuh"

namespace fc {

static __device__ unsigned int g_fftconv_tc_timeouts;

namespace {
constexpr int kN1 = 128, kN2 = 16, kM = kN1 * kN2, kL = kM / 2;
constexpr int kThr = 256;                  // two groups of four warps
constexpr int kMaxPairs = 4;               // row pairs per batch
constexpr uint32_t kTmemCols = 256;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kCLbo = 128, kCSbo = (kN1 / 8) * 128;  // CA / CB K-major: 128 rows x 128 K
constexpr uint32_t kCBytes = kN1 * kN1 * 2;
// Stage-B tiles: per sequence a K-major 128 (k1) x 32 (re n2 | im n2) fp16 tile
constexpr uint32_t kYLbo = 128, kYSbo = 4 * 128, kYTile = kN1 * 32 * 2;
// X (stage A input), the stage-B tiles, then Z (stage A' input) share one buffer
constexpr uint32_t kXZBytes = (kMaxPairs + 1) * kYTile;
static_assert(kXZBytes >= kMaxPairs * kN2 * 2 * kN1 * 2, "Z must fit");
// fp32 filter staging inside the X/Z buffer, past the largest X (2 planes x 64 K-rows x 80 columns)
constexpr uint32_t kFStage = 2 * 64 * (kMaxPairs + 1) * kN2 * 2;
static_assert(kFStage + kL * 4 <= kXZBytes, "filter staging must fit in the X/Z buffer");

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

struct TcSmem {
  uint8_t ca[kCBytes];
  uint8_t cb[kCBytes];
  uint8_t xz[kXZBytes];   // stage-A input X, then the stage-B tiles, then the stage-A' input Z
  uint8_t wf[32 * 32 * 2];  // DFT-16 as a real 32 x 32 block (B operand, rows = output re/im k2)
  uint8_t wi[32 * 32 * 2];  // inverse DFT-16
  float2 costab[kN1];
  uint64_t mbar;
  uint32_t tmem_base;
};

template <typename T> struct Op;
template <> struct Op<__half> {
  static constexpr int bf16 = 0;
  static __device__ __forceinline__ uint16_t bits(float x) { return __half_as_ushort(__float2half_rn(x)); }
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ float2 unpack(uint32_t w) {
    return __half22float2(*reinterpret_cast<__half2*>(&w));
  }
};
template <> struct Op<__nv_bfloat16> {
  static constexpr int bf16 = 1;
  static __device__ __forceinline__ uint16_t bits(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ float2 unpack(uint32_t w) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w));
  }
};
}  // namespace

// u, y: B x H x 1024 (T); f: H x 1024 fp32 filters; D: H.
template <typename T>
__global__ void __launch_bounds__(kThr, 2) fftconv_tc_kernel(const T* __restrict__ u, const float* __restrict__ f,
                                                             const float* __restrict__ D, T* __restrict__ y, int B,
                                                             int H, int conj_filter) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  TcSmem& sm = *reinterpret_cast<TcSmem*>(smraw);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int row = tid & (kN1 - 1);  // TMEM lane / frequency row k1 / output lane j
  const int grp = tid >> 7;         // 0 or 1
  const uint16_t* ub = reinterpret_cast<const uint16_t*>(u);
  uint16_t* yb = reinterpret_cast<uint16_t*>(y);

  if (warp == 0) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
  if (tid == 0) {
    tc::mbar_init(&sm.mbar, 1);
    tc::fence_mbar_init();
  }
  if (tid < kN1) {
    float s, c;
    sincospif(2.0f * (float)tid / (float)kN1, &s, &c);
    sm.costab[tid] = make_float2(c, s);
  }
  __syncthreads();
  // constant DFT-128 blocks, K-major (rows k1, K = j), 8 consecutive j per 16-byte store
  for (int idx = tid; idx < kN1 * (kN1 / 8); idx += kThr) {
    const int k1 = idx >> 4, j0 = (idx & 15) * 8;
    float a[8], b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = j0 + i, jj = j & 63;
      const float2 cs = sm.costab[(k1 * jj) & 127];
      a[i] = j < 64 ? cs.x : cs.y;
      b[i] = j < 64 ? -cs.y : cs.x;
    }
    const uint32_t off = tc::kmaj_off(k1, j0, kN1);
    *reinterpret_cast<uint4*>(sm.ca + off) =
        make_uint4(Op<T>::pack(a[0], a[1]), Op<T>::pack(a[2], a[3]), Op<T>::pack(a[4], a[5]), Op<T>::pack(a[6], a[7]));
    *reinterpret_cast<uint4*>(sm.cb + off) =
        make_uint4(Op<T>::pack(b[0], b[1]), Op<T>::pack(b[2], b[3]), Op<T>::pack(b[4], b[5]), Op<T>::pack(b[6], b[7]));
  }
  // DFT-16 blocks (fp16, K-major 32 x 32): row c = output (k2 = c % 16, imaginary part if c >= 16),
  // column j = input (n2 = j % 16, imaginary part if j >= 16); angle 2 pi n2 k2 / 16
  for (int idx = tid; idx < 32 * 4; idx += kThr) {
    const int c = idx >> 2, j0 = (idx & 3) * 8;
    float a[8], b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = j0 + i;
      const float2 cs = sm.costab[(8 * (j & 15) * (c & 15)) & 127];
      const bool oim = c >= 16, iim = j >= 16;
      // forward (e^{-i theta}): Re += xr cos + xi sin, Im += xi cos - xr sin; inverse flips sin
      const float fw = (oim == iim) ? cs.x : (iim ? cs.y : -cs.y);
      a[i] = fw;
      b[i] = (oim == iim) ? cs.x : -fw;
    }
    const uint32_t off = (uint32_t)(c >> 3) * kYSbo + (uint32_t)(j0 >> 3) * kYLbo + (uint32_t)(c & 7) * 16;
    *reinterpret_cast<uint4*>(sm.wf + off) = make_uint4(Op<__half>::pack(a[0], a[1]), Op<__half>::pack(a[2], a[3]),
                                                        Op<__half>::pack(a[4], a[5]), Op<__half>::pack(a[6], a[7]));
    *reinterpret_cast<uint4*>(sm.wi + off) = make_uint4(Op<__half>::pack(b[0], b[1]), Op<__half>::pack(b[2], b[3]),
                                                        Op<__half>::pack(b[4], b[5]), Op<__half>::pack(b[6], b[7]));
  }
  // this thread's stage twiddles w_2048^(k1 n2) / 32, k1 = row: the 1/32 keeps the
  // fp16 stage-B tile at |Y| / 32 <= 2 max|u|; the filter bins carry the factor 32
  // back, and the inverse twiddle is 32 conj(tws).
  float2 tws[kN2];
#pragma unroll
  for (int n2 = 0; n2 < kN2; ++n2) {
    float s, c;
    sincospif(-2.0f * (float)(row * n2) / (float)kM, &s, &c);
    tws[n2] = make_float2(c * (1.f / 32.f), s * (1.f / 32.f));
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t ca = tc::smem_u32(sm.ca), cb = tc::smem_u32(sm.cb), xz = tc::smem_u32(sm.xz);
  const int npairs = (B + 1) / 2;
  uint32_t phase = 0;
  bool failed = false;
  float2 fh[kN2];

  // Work items of this CTA, in order: channels h = blockIdx.x, + gridDim.x, ...,
  // each in batches of up to kMaxPairs row pairs (the first batch also carries
  // the filter).  The next item's inputs are copied into the X/Z buffer with
  // cp.async while the current item's epilogue runs.
  int h = blockIdx.x, p0 = 0;
  // u rows of item (h, p0) -> X planes (zero rows written directly)
  auto issue_u = [&](int hh, int pp0) {
    const bool wf = (pp0 == 0);
    const int P = min(kMaxPairs, npairs - pp0);
    const int NS = P + (wf ? 1 : 0);
    const uint32_t lboX = (uint32_t)(NS * kN2 / 8) * 128;
    for (int idx = tid; idx < P * 64 * 2; idx += kThr) {
      const int half = idx & 1, n1 = (idx >> 1) & 63, pc = idx >> 7;
      const int s = pc + (wf ? 1 : 0);
      const int n = s * kN2 + half * 8;
      const uint32_t off = (uint32_t)(n >> 3) * 128 + (uint32_t)(n1 >> 3) * lboX + (uint32_t)(n1 & 7) * 16;
      const int t = n1 * kN2 + half * 8;
      const int b0 = 2 * (pp0 + pc), b1 = b0 + 1;
      cp_async16(xz + off, ub + ((size_t)b0 * H + hh) * kL + t);
      if (b1 < B)
        cp_async16(xz + 8 * lboX + off, ub + ((size_t)b1 * H + hh) * kL + t);
      else
        *reinterpret_cast<uint4*>(sm.xz + 8 * lboX + off) = make_uint4(0, 0, 0, 0);
    }
  };
  // fp32 filter row of channel hh -> staging area past the X planes
  auto issue_f = [&](int hh) {
    for (int idx = tid; idx < kL / 4; idx += kThr)
      cp_async16(xz + kFStage + idx * 16, f + (size_t)hh * kL + idx * 4);
  };
  if (h < H) issue_u(h, 0);
  // the filter is written by the preceding kernel when launched as its
  // programmatic dependent (no-op otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (h < H) issue_f(h);
  cp_async_commit();

  while (h < H && !failed) {
    const bool with_filter = (p0 == 0);
    const int P = min(kMaxPairs, npairs - p0);
    const int NS = P + (with_filter ? 1 : 0);
    const int NC = NS * kN2;                         // stage-A columns per real/imag half
    const uint32_t lboX = (uint32_t)(NC / 8) * 128;  // X: MN-major, 64 K-rows (n1) x NC
    const uint32_t xr = xz, xi = xz + 8 * lboX;
    cp_async_wait_all();  // this thread's copies; the barrier makes everyone's visible
    __syncthreads();
    if (with_filter) {  // filter block: fp32 staging -> operand type, D folded into tap 0
      for (int idx = tid; idx < 64 * 2; idx += kThr) {
        const int half = idx & 1, n1 = idx >> 1;
        const int t = n1 * kN2 + half * 8;
        const uint32_t off = (uint32_t)half * 128 + (uint32_t)(n1 >> 3) * lboX + (uint32_t)(n1 & 7) * 16;
        float4 a = *reinterpret_cast<const float4*>(sm.xz + kFStage + t * 4);
        const float4 b = *reinterpret_cast<const float4*>(sm.xz + kFStage + t * 4 + 16);
        if (t == 0) a.x += D[h];  // y = f * u + D u = (f + D delta) * u
        *reinterpret_cast<uint4*>(sm.xz + off) = make_uint4(Op<T>::pack(a.x, a.y), Op<T>::pack(a.z, a.w),
                                                            Op<T>::pack(b.x, b.y), Op<T>::pack(b.z, b.w));
        *reinterpret_cast<uint4*>(sm.xz + 8 * lboX + off) = make_uint4(0, 0, 0, 0);
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // ---- stage A: D_re at TMEM columns [0, NC), D_im at [NC, 2 NC)
    if (tid == 0) {
      const uint32_t idA = tc::idesc_f16(128, NC, Op<T>::bf16, 0, 1);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(ca + kk * 256, kCLbo, kCSbo), tc::desc_kmajor(xr + kk * 2 * lboX, lboX, 128),
                    idA, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(ca + (4 + kk) * 256, kCLbo, kCSbo),
                    tc::desc_kmajor(xi + kk * 2 * lboX, lboX, 128), idA, 1u);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc::mma_f16(tmem + NC, tc::desc_kmajor(ca + kk * 256, kCLbo, kCSbo),
                    tc::desc_kmajor(xi + kk * 2 * lboX, lboX, 128), idA, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc::mma_f16(tmem + NC, tc::desc_kmajor(cb + kk * 256, kCLbo, kCSbo),
                    tc::desc_kmajor(xr + kk * 2 * lboX, lboX, 128), idA, 1u);
      tc::mma_commit(&sm.mbar);
    }
    bool ok = tc::mbar_wait_bounded(&sm.mbar, phase, kWaitNs);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    // ---- 2a: Y' = twiddled stage-A output / 32 as fp16 stage-B tiles (sequences alternate between groups)
#pragma unroll 1
    for (int s = grp; s < NS; s += 2) {
      float yr[16], yi[16];
      tc::tmem_ld16x2_wait(tmem + lane_off + (uint32_t)(s * kN2), tmem + lane_off + (uint32_t)(NC + s * kN2), yr, yi);
      uint32_t pr[8], pi[8];
#pragma unroll
      for (int n2 = 0; n2 < kN2; n2 += 2) {
        const float2 a = cmul(make_float2(yr[n2], yi[n2]), tws[n2]);
        const float2 b = cmul(make_float2(yr[n2 + 1], yi[n2 + 1]), tws[n2 + 1]);
        pr[n2 / 2] = Op<__half>::pack(a.x, b.x);
        pi[n2 / 2] = Op<__half>::pack(a.y, b.y);
      }
      uint8_t* tile = sm.xz + (uint32_t)s * kYTile + (uint32_t)(row >> 3) * kYSbo + (uint32_t)(row & 7) * 16;
      *reinterpret_cast<uint4*>(tile) = make_uint4(pr[0], pr[1], pr[2], pr[3]);
      *reinterpret_cast<uint4*>(tile + kYLbo) = make_uint4(pr[4], pr[5], pr[6], pr[7]);
      *reinterpret_cast<uint4*>(tile + 2 * kYLbo) = make_uint4(pi[0], pi[1], pi[2], pi[3]);
      *reinterpret_cast<uint4*>(tile + 3 * kYLbo) = make_uint4(pi[4], pi[5], pi[6], pi[7]);
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // ---- stage B: X^ = DFT16(Y') per sequence into TMEM columns [32 s, 32 s + 32) (re k2 | im k2)
    const uint32_t idY = tc::idesc_f16(128, 32, 0);
    if (tid == 0) {
      const uint32_t wfa = tc::smem_u32(sm.wf);
      for (int s = 0; s < NS; ++s) {
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          tc::mma_f16(tmem + (uint32_t)(32 * s), tc::desc_kmajor(xz + s * kYTile + kk * 2 * kYLbo, kYLbo, kYSbo),
                      tc::desc_kmajor(wfa + kk * 2 * kYLbo, kYLbo, kYSbo), idY, kk > 0 ? 1u : 0u);
      }
      tc::mma_commit(&sm.mbar);
    }
    ok = tc::mbar_wait_bounded(&sm.mbar, phase, kWaitNs);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    // ---- 2c: filter bins 32 f^/M (every thread keeps its row's 16), then V = X^ . f^ / M
    // (X^ here is 1/32 of the transform) for this group's pairs
    if (with_filter) {
      float xr[16], xi[16];
      tc::tmem_ld16x2_wait(tmem + lane_off, tmem + lane_off + 16u, xr, xi);
      constexpr float sc = 32.0f * 32.0f / (float)kM;  // undo the 1/32 of stage B, x32 for the pairs, 1/M
      // conj_filter: conj(F^), i.e. correlation with f (the input gradient)
      const float sci = conj_filter ? -sc : sc;
#pragma unroll
      for (int k2 = 0; k2 < kN2; ++k2) fh[k2] = make_float2(xr[k2] * sc, xi[k2] * sci);
    }
#pragma unroll 1
    for (int p = grp; p < P; p += 2) {
      const int s = p + (with_filter ? 1 : 0);
      float xr[16], xi[16];
      tc::tmem_ld16x2_wait(tmem + lane_off + (uint32_t)(32 * s), tmem + lane_off + (uint32_t)(32 * s + 16), xr, xi);
      uint32_t pr[8], pi[8];
#pragma unroll
      for (int k2 = 0; k2 < kN2; k2 += 2) {
        const float2 a = cmul(make_float2(xr[k2], xi[k2]), fh[k2]);
        const float2 b = cmul(make_float2(xr[k2 + 1], xi[k2 + 1]), fh[k2 + 1]);
        pr[k2 / 2] = Op<__half>::pack(a.x, b.x);
        pi[k2 / 2] = Op<__half>::pack(a.y, b.y);
      }
      uint8_t* tile = sm.xz + (uint32_t)s * kYTile + (uint32_t)(row >> 3) * kYSbo + (uint32_t)(row & 7) * 16;
      *reinterpret_cast<uint4*>(tile) = make_uint4(pr[0], pr[1], pr[2], pr[3]);
      *reinterpret_cast<uint4*>(tile + kYLbo) = make_uint4(pr[4], pr[5], pr[6], pr[7]);
      *reinterpret_cast<uint4*>(tile + 2 * kYLbo) = make_uint4(pi[0], pi[1], pi[2], pi[3]);
      *reinterpret_cast<uint4*>(tile + 3 * kYLbo) = make_uint4(pi[4], pi[5], pi[6], pi[7]);
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // ---- stage B': IDFT16(V) per pair into TMEM columns [32 p, 32 p + 32)
    if (tid == 0) {
      const uint32_t wia = tc::smem_u32(sm.wi);
      for (int p = 0; p < P; ++p) {
        const int s = p + (with_filter ? 1 : 0);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          tc::mma_f16(tmem + (uint32_t)(32 * p), tc::desc_kmajor(xz + s * kYTile + kk * 2 * kYLbo, kYLbo, kYSbo),
                      tc::desc_kmajor(wia + kk * 2 * kYLbo, kYLbo, kYSbo), idY, kk > 0 ? 1u : 0u);
      }
      tc::mma_commit(&sm.mbar);
    }
    ok = tc::mbar_wait_bounded(&sm.mbar, phase, kWaitNs);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    // ---- 2d: Z = stage-B' output x conj twiddle, MN-major (K rows re k1 | im k1) for stage A'
    const uint32_t lboZ = (uint32_t)(P * kN2 / 8) * 128;  // Z: MN-major, 256 K-rows (re k1 | im k1) x P*16
#pragma unroll 1
    for (int p = grp; p < P; p += 2) {
      float zr[16], zi[16];
      tc::tmem_ld16x2_wait(tmem + lane_off + (uint32_t)(32 * p), tmem + lane_off + (uint32_t)(32 * p + 16), zr, zi);
      float2 v[kN2];
#pragma unroll
      for (int n2 = 0; n2 < kN2; ++n2) {
        const float2 z = cmul(make_float2(zr[n2], zi[n2]), cconj(tws[n2]));
        v[n2] = make_float2(32.f * z.x, 32.f * z.y);
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int n = p * kN2 + half * 8;
        const uint32_t offr = (uint32_t)(n >> 3) * 128 + (uint32_t)(row >> 3) * lboZ + (uint32_t)(row & 7) * 16;
        const uint32_t offi = offr + 16 * lboZ;  // K rows 128 + k1
        const float2* w = v + half * 8;
        *reinterpret_cast<uint4*>(sm.xz + offr) =
            make_uint4(Op<T>::pack(w[0].x, w[1].x), Op<T>::pack(w[2].x, w[3].x), Op<T>::pack(w[4].x, w[5].x),
                       Op<T>::pack(w[6].x, w[7].x));
        *reinterpret_cast<uint4*>(sm.xz + offi) =
            make_uint4(Op<T>::pack(w[0].y, w[1].y), Op<T>::pack(w[2].y, w[3].y), Op<T>::pack(w[4].y, w[5].y),
                       Op<T>::pack(w[6].y, w[7].y));
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // ---- stage A': y = CA^T Zr + CB^T Zi into TMEM columns [0, P*16)
    if (tid == 0) {
      const uint32_t idB = tc::idesc_f16(128, P * kN2, Op<T>::bf16, 1, 1);
      const uint32_t zr = xz, zi = xz + 16 * lboZ;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(ca + kk * 2 * kCSbo, kCSbo, kCLbo),
                    tc::desc_kmajor(zr + kk * 2 * lboZ, lboZ, 128), idB, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(cb + kk * 2 * kCSbo, kCSbo, kCLbo),
                    tc::desc_kmajor(zi + kk * 2 * lboZ, lboZ, 128), idB, 1u);
      tc::mma_commit(&sm.mbar);
    }
    ok = tc::mbar_wait_bounded(&sm.mbar, phase, kWaitNs);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    // ---- the X/Z buffer is free: start copying the next item's inputs
    const int h_cur = h, p0_cur = p0;
    p0 += kMaxPairs;
    if (p0 >= npairs) {
      p0 = 0;
      h += gridDim.x;
    }
    if (h < H) {
      issue_u(h, p0);
      if (p0 == 0) issue_f(h);
    }
    cp_async_commit();
    // ---- epilogue: lane j -> (part c = j / 64, n1 = j % 64); the D u term rode
    // through the transform with the filter (its tap 0 carries D)
    const int c = row >> 6, n1 = row & 63;
#pragma unroll 1
    for (int p = grp; p < P; p += 2) {
      float yv[16];
      tc::tmem_ld16_wait(tmem + lane_off + (uint32_t)(p * kN2), yv);
      const int brow = 2 * (p0_cur + p) + c;
      if (brow < B) {
        const size_t rbase = ((size_t)brow * H + h_cur) * kL + (size_t)n1 * kN2;
        uint32_t ow[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) ow[i] = Op<T>::pack(yv[2 * i], yv[2 * i + 1]);
        *reinterpret_cast<uint4*>(yb + rbase) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        *reinterpret_cast<uint4*>(yb + rbase + 8) = make_uint4(ow[4], ow[5], ow[6], ow[7]);
      }
    }
  }
  cp_async_wait_all();
  if (failed && tid == 0) atomicAdd(&g_fftconv_tc_timeouts, 1u);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

template <typename T>
static cudaError_t fftconv_tc_t(const void* u, const float* f, const float* D, void* y, int B, int H, bool pdl,
                                cudaStream_t st, bool conj_filter) {
  auto kern = fftconv_tc_kernel<T>;
  const size_t smem = sizeof(TcSmem);
  cudaError_t e = smem_optin<fftconv_tc_kernel<T>>(smem);
  if (e != cudaSuccess) return e;
  const int sms = num_sms();
  const int grid = H < 2 * sms ? H : 2 * sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThr);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, (const T*)u, f, D, (T*)y, B, H, conj_filter ? 1 : 0);
}

bool fftconv_tc_supported(int L, int dtype) { return L == kL && (dtype == 1 || dtype == 2); }

cudaError_t launch_fftconv_tc(const void* u, const float* f, const float* D, void* y, int B, int H, int L, int dtype,
                              bool after_filter_kernel, cudaStream_t st, bool conj_filter) {
  if (!fftconv_tc_supported(L, dtype)) return cudaErrorInvalidValue;
  return dtype == 1 ? fftconv_tc_t<__half>(u, f, D, y, B, H, after_filter_kernel, st, conj_filter)
                    : fftconv_tc_t<__nv_bfloat16>(u, f, D, y, B, H, after_filter_kernel, st, conj_filter);
}

unsigned int fftconv_tc_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_fftconv_tc_timeouts, sizeof(v));
  return v;
}

}  // namespace fc
