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
// stages A and A' use the I/O type.  All constant blocks and twiddles come
// from tables built with the library (tc_tables.inc) and are copied into
// shared memory once per CTA.
//
// Work: an item is one channel's filter plus up to 4 row pairs (two real
// rows packed as one complex sequence u0 + i u1; f is real, so the real and
// imaginary outputs are the two convolutions): N = 16 x (1 + pairs) stage-A
// columns.  One CTA per SM runs two independent pipelines of 8 warps that
// share the tables; each has its own named barrier, MMA barrier, half of the
// tensor memory, input buffer and work buffer, so one pipeline's register
// passes overlap the other's MMAs and loads.  Pipeline c of CTA b takes the
// items b + G (2 k + c) (G = grid size), so every SM gets an equal share.  The
// next item's inputs are copied in with cp.async as soon as stage A has read
// the current ones.  In a pipeline, warp w serves TMEM lane quarter w % 4
// and column half w / 4 of every 16-column block.  Waits on MMA completion
// are bounded; a pipeline that gives up records it in a device counter,
// skips its remaining work and the CTA still frees its TMEM.
#include "kernels.cuh"
#include "tc100.cuh"

#define FC_TABLES_DFT128
#define FC_TABLES_1K
#include "tc_tables.inc"

namespace fc {

static __device__ unsigned int g_fftconv_tc_timeouts;

namespace {
constexpr int kN1 = 128, kN2 = 16, kM = kN1 * kN2, kL = kM / 2;
constexpr int kPipes = 2, kPipeThr = 256, kThr = kPipes * kPipeThr;
constexpr int kMaxPairs = 4;
constexpr uint32_t kPipeCols = 256;                       // TMEM columns per pipeline
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kCLbo = 128, kCSbo = (kN1 / 8) * 128;  // CA / CB K-major: 128 rows x 128 K
constexpr uint32_t kCBytes = kN1 * kN1 * 2;
constexpr uint32_t kYLbo = 128, kYSbo = 4 * 128, kYTile = kN1 * 32 * 2;  // 128 x 32 fp16 tiles, K-major
constexpr uint32_t kXBytes = 2 * 64 * (kMaxPairs + 1) * kN2 * 2;        // X planes for 5 sequences
constexpr uint32_t kFBytes = kL * 4;                                     // fp32 filter staging
constexpr uint32_t kWBytes = (kMaxPairs + 1) * kYTile;                   // stage-B tiles, then Z
static_assert(kWBytes >= kMaxPairs * kN2 * 2 * kN1 * 2, "Z must fit the work buffer");
// shared memory layout (bytes)
constexpr uint32_t kTwBytes = kN1 * kN2 * 8;  // fp32 twiddles w_2048^(k1 n2) / 32
constexpr uint32_t kOCa = 0, kOCb = kCBytes, kOWf = 2 * kCBytes, kOWi = kOWf + 2048, kOTw = kOWi + 2048,
                   kOPipe = kOTw + kTwBytes;
constexpr uint32_t kPipeBytes = kXBytes + kFBytes + kWBytes;
constexpr uint32_t kOX = 0, kOF = kXBytes, kOW = kXBytes + kFBytes;  // within a pipeline's part
constexpr uint32_t kOMbar = kOPipe + kPipes * kPipeBytes, kOTmem = kOMbar + 8 * kPipes;
constexpr uint32_t kSmem = kOTmem + 16;

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
__device__ __forceinline__ uint32_t pack_h(float a, float b) { return Op<__half>::pack(a, b); }

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// named barrier of one pipeline (ids 1, 2; id 0 is __syncthreads)
__device__ __forceinline__ void pipe_sync(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(kPipeThr) : "memory");
}
__device__ __forceinline__ bool pipe_or(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "n"(kPipeThr)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float2 ldf2(const float* p) { return *reinterpret_cast<const float2*>(p); }
}  // namespace

// u, y: B x H x 1024 (T); f: H x 1024 fp32 filters; D: H.
template <typename T>
__global__ void __launch_bounds__(kThr, 1) fftconv_tc_kernel(const T* __restrict__ u, const float* __restrict__ f,
                                                             const float* __restrict__ D, T* __restrict__ y, int B,
                                                             int H, int conj_filter) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int pipe = tid / kPipeThr;           // 0 or 1
  const int pt = tid - pipe * kPipeThr;      // thread within the pipeline
  const int half = (pt >> 5) >> 2;           // column half of every 16-column block
  const int row = tid & (kN1 - 1);           // TMEM lane / frequency row k1 / output lane j
  const int bar_id = 1 + pipe;
  const uint16_t* ub = reinterpret_cast<const uint16_t*>(u);
  uint16_t* yb = reinterpret_cast<uint16_t*>(y);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + kOMbar) + pipe;
  uint32_t* tmem_p = reinterpret_cast<uint32_t*>(sm + kOTmem);
  const uint32_t s0 = tc::smem_u32(sm);
  const uint32_t ca = s0 + kOCa, cb = s0 + kOCb, wfa = s0 + kOWf, wia = s0 + kOWi;
  const float2* tws = reinterpret_cast<const float2*>(sm + kOTw);  // [k1][n2]
  const uint32_t pbase = kOPipe + (uint32_t)pipe * kPipeBytes;
  const uint32_t xs = s0 + pbase + kOX, fs = s0 + pbase + kOF, ws = s0 + pbase + kOW;
  uint8_t* const wsp = sm + pbase + kOW;

  if (warp == 0) tc::tmem_alloc(tmem_p, kPipes * kPipeCols);
  if (tid == 0) {
    for (int i = 0; i < kPipes; ++i) tc::mbar_init(reinterpret_cast<uint64_t*>(sm + kOMbar) + i, 1);
    tc::fence_mbar_init();
  }
  // constant blocks: CA, CB in the I/O type, the DFT-16 blocks in fp16 (already in the operand layout)
  {
    const uint8_t* gca = reinterpret_cast<const uint8_t*>(Op<T>::ca());
    const uint8_t* gcb = reinterpret_cast<const uint8_t*>(Op<T>::cb());
    for (int i = tid; i < (int)(kCBytes / 16); i += kThr) {
      cp_async16(ca + i * 16, gca + i * 16);
      cp_async16(cb + i * 16, gcb + i * 16);
    }
    if (tid < 128) cp_async16(wfa + tid * 16, reinterpret_cast<const uint8_t*>(g_wf16_f16) + tid * 16);
    else if (tid < 256) cp_async16(wia + (tid - 128) * 16, reinterpret_cast<const uint8_t*>(g_wi16_f16) + (tid - 128) * 16);
    for (int i = tid; i < (int)(kTwBytes / 16); i += kThr)
      cp_async16(s0 + kOTw + i * 16, reinterpret_cast<const uint8_t*>(g_tw1k) + i * 16);
  }
  cp_async_commit();

  const int npairs = (B + 1) / 2;
  const int ngroups = (npairs + kMaxPairs - 1) / kMaxPairs;
  const long long nitems = (long long)H * ngroups;
  const long long stride = 2LL * gridDim.x;
  auto pairs_of = [&](int g) { return min(kMaxPairs, npairs - g * kMaxPairs); };
  // u rows of item it -> X planes of this pipeline (filter column block 0 left for the filter)
  auto issue_u = [&](long long it) {
    const int h = (int)(it / ngroups), g = (int)(it - (long long)h * ngroups);
    const int P = pairs_of(g);
    const uint32_t lboX = (uint32_t)((P + 1) * kN2 / 8) * 128;
    for (int idx = pt; idx < P * 64 * 2; idx += kPipeThr) {
      const int hf = idx & 1, n1 = (idx >> 1) & 63, pc = idx >> 7;
      const int n = (pc + 1) * kN2 + hf * 8;
      const uint32_t off = (uint32_t)(n >> 3) * 128 + (uint32_t)(n1 >> 3) * lboX + (uint32_t)(n1 & 7) * 16;
      const int t = n1 * kN2 + hf * 8;
      const int b0 = 2 * (g * kMaxPairs + pc), b1 = b0 + 1;
      cp_async16(xs + off, ub + ((size_t)b0 * H + h) * kL + t);
      if (b1 < B)
        cp_async16(xs + 8 * lboX + off, ub + ((size_t)b1 * H + h) * kL + t);
      else
        *reinterpret_cast<uint4*>(sm + pbase + kOX + 8 * lboX + off) = make_uint4(0, 0, 0, 0);
    }
  };
  auto issue_f = [&](long long it) {
    const int h = (int)(it / ngroups);
    for (int idx = pt; idx < kL / 4; idx += kPipeThr) cp_async16(fs + idx * 16, f + (size_t)h * kL + idx * 4);
  };
  long long it = blockIdx.x + (long long)gridDim.x * pipe;
  if (it < nitems) issue_u(it);
  float d_next = 0.f;  // D of the next item's channel, loaded with its inputs
  // the filter is written by the kernel this one may be launched as a
  // programmatic dependent of: read it only after the wait
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (it < nitems) {
    issue_f(it);
    d_next = D[(int)(it / ngroups)];
  }
  cp_async_commit();
  cp_async_wait_all();
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_p + (uint32_t)pipe * kPipeCols;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  uint32_t phase = 0;
  bool failed = false;

  auto to_mma = [&]() {  // this pipeline's generic shared-memory writes -> its next MMAs
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    pipe_sync(bar_id);
    tc::fence_after_sync();
  };
  auto mma_wait = [&]() -> bool {
    const bool ok = tc::mbar_wait_bounded(mbar, phase, kWaitNs);
    phase ^= 1u;
    if (pipe_or(bar_id, !ok)) return false;
    tc::fence_after_sync();
    return true;
  };

  for (; it < nitems; it += stride) {
    const int h = (int)(it / ngroups), g = (int)(it - (long long)h * ngroups);
    const int P = pairs_of(g);
    const int NS = P + 1;                              // the filter, then the pairs
    const int NC = NS * kN2;                           // stage-A columns per real/imag half
    const uint32_t lboX = (uint32_t)(NC / 8) * 128;    // X: MN-major, 64 K-rows (n1) x NC
    const uint32_t xr = xs, xi = xs + 8 * lboX;
    const float dh = d_next;
    cp_async_wait_all();
    pipe_sync(bar_id);  // every thread's copies have landed
    // filter block (column block 0): fp32 staging -> operand type, D folded into tap 0
    if (pt < 128) {
      const int hf = pt & 1, n1 = pt >> 1;
      const int t = n1 * kN2 + hf * 8;
      float4 a = *reinterpret_cast<const float4*>(sm + pbase + kOF + t * 4);
      const float4 b = *reinterpret_cast<const float4*>(sm + pbase + kOF + t * 4 + 16);
      if (t == 0) a.x += dh;  // y = f * u + D u = (f + D delta) * u
      const uint32_t off = (uint32_t)hf * 128 + (uint32_t)(n1 >> 3) * lboX + (uint32_t)(n1 & 7) * 16;
      *reinterpret_cast<uint4*>(sm + pbase + kOX + off) = make_uint4(Op<T>::pack(a.x, a.y), Op<T>::pack(a.z, a.w),
                                                                    Op<T>::pack(b.x, b.y), Op<T>::pack(b.z, b.w));
      *reinterpret_cast<uint4*>(sm + pbase + kOX + 8 * lboX + off) = make_uint4(0, 0, 0, 0);
    }
    to_mma();
    // ---- stage A: D_re at TMEM columns [0, NC), D_im at [NC, 2 NC)
    if (pt == 0) {
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
      tc::mma_commit(mbar);
    }
    if (!mma_wait()) { failed = true; break; }
    // ---- the X planes and the filter staging are free: prefetch the next item
    if (it + stride < nitems) {
      issue_u(it + stride);
      issue_f(it + stride);
      d_next = D[(int)((it + stride) / ngroups)];
    }
    cp_async_commit();
    // ---- pass 1: Y' = Y w_2048^(k1 n2) / 32 -> fp16 stage-B tile per sequence (this thread: n2 = 8 half + i)
    {
      float2 tw[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) tw[i] = tws[row * kN2 + 8 * half + i];
#pragma unroll 1
      for (int s = 0; s < NS; s += 2) {
        const bool two = s + 1 < NS;
        uint32_t yr[2][8], yi[2][8];
        tc::tmem_ld8(tmem + lane_off + (uint32_t)(s * kN2 + 8 * half), yr[0]);
        tc::tmem_ld8(tmem + lane_off + (uint32_t)(NC + s * kN2 + 8 * half), yi[0]);
        if (two) {
          tc::tmem_ld8(tmem + lane_off + (uint32_t)((s + 1) * kN2 + 8 * half), yr[1]);
          tc::tmem_ld8(tmem + lane_off + (uint32_t)(NC + (s + 1) * kN2 + 8 * half), yi[1]);
        }
        tc::tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            tc::tmem_regs_ready(yr[q][i]);
            tc::tmem_regs_ready(yi[q][i]);
          }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (q == 1 && !two) break;
          uint32_t pr[4], pi[4];
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            const float2 a = cmul(make_float2(__uint_as_float(yr[q][i]), __uint_as_float(yi[q][i])), tw[i]);
            const float2 b = cmul(make_float2(__uint_as_float(yr[q][i + 1]), __uint_as_float(yi[q][i + 1])), tw[i + 1]);
            pr[i / 2] = pack_h(a.x, b.x);
            pi[i / 2] = pack_h(a.y, b.y);
          }
          uint8_t* tile = wsp + (uint32_t)(s + q) * kYTile + (uint32_t)(row >> 3) * kYSbo + (uint32_t)(row & 7) * 16;
          *reinterpret_cast<uint4*>(tile + (uint32_t)half * kYLbo) = make_uint4(pr[0], pr[1], pr[2], pr[3]);
          *reinterpret_cast<uint4*>(tile + (uint32_t)(2 + half) * kYLbo) = make_uint4(pi[0], pi[1], pi[2], pi[3]);
        }
      }
    }
    to_mma();
    // ---- stage B: X^ = DFT16(Y') per sequence into TMEM columns [32 s, 32 s + 32) (re k2 | im k2)
    const uint32_t idY = tc::idesc_f16(128, 32, 0);
    if (pt == 0) {
      for (int s = 0; s < NS; ++s) {
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          tc::mma_f16(tmem + (uint32_t)(32 * s), tc::desc_kmajor(ws + s * kYTile + kk * 2 * kYLbo, kYLbo, kYSbo),
                      tc::desc_kmajor(wfa + kk * 2 * kYLbo, kYLbo, kYSbo), idY, kk > 0 ? 1u : 0u);
      }
      tc::mma_commit(mbar);
    }
    if (!mma_wait()) { failed = true; break; }
    // ---- pass 2: V = X^ . (32 F^ / M) (X^ here is 1/32 of the transform) for this thread's bins k2 = 8 half + i
    {
      uint32_t fr_[8], fi_[8];
      tc::tmem_ld8(tmem + lane_off + (uint32_t)(8 * half), fr_);
      tc::tmem_ld8(tmem + lane_off + (uint32_t)(16 + 8 * half), fi_);
      tc::tmem_wait_ld();
      constexpr float sc = 32.0f * 32.0f / (float)kM;  // undo the 1/32 of stage B, x32 for the pairs, 1/M
      const float sci = conj_filter ? -sc : sc;          // conj(F^): correlation (the input gradient)
      float2 fh[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        tc::tmem_regs_ready(fr_[i]);
        tc::tmem_regs_ready(fi_[i]);
        fh[i] = make_float2(__uint_as_float(fr_[i]) * sc, __uint_as_float(fi_[i]) * sci);
      }
#pragma unroll 1
      for (int p = 0; p < P; p += 2) {
        const bool two = p + 1 < P;
        uint32_t xr_[2][8], xi_[2][8];
        tc::tmem_ld8(tmem + lane_off + (uint32_t)(32 * (p + 1) + 8 * half), xr_[0]);
        tc::tmem_ld8(tmem + lane_off + (uint32_t)(32 * (p + 1) + 16 + 8 * half), xi_[0]);
        if (two) {
          tc::tmem_ld8(tmem + lane_off + (uint32_t)(32 * (p + 2) + 8 * half), xr_[1]);
          tc::tmem_ld8(tmem + lane_off + (uint32_t)(32 * (p + 2) + 16 + 8 * half), xi_[1]);
        }
        tc::tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            tc::tmem_regs_ready(xr_[q][i]);
            tc::tmem_regs_ready(xi_[q][i]);
          }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (q == 1 && !two) break;
          uint32_t pr[4], pi[4];
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            const float2 a = cmul(make_float2(__uint_as_float(xr_[q][i]), __uint_as_float(xi_[q][i])), fh[i]);
            const float2 b = cmul(make_float2(__uint_as_float(xr_[q][i + 1]), __uint_as_float(xi_[q][i + 1])), fh[i + 1]);
            pr[i / 2] = pack_h(a.x, b.x);
            pi[i / 2] = pack_h(a.y, b.y);
          }
          uint8_t* tile = wsp + (uint32_t)(p + q + 1) * kYTile + (uint32_t)(row >> 3) * kYSbo + (uint32_t)(row & 7) * 16;
          *reinterpret_cast<uint4*>(tile + (uint32_t)half * kYLbo) = make_uint4(pr[0], pr[1], pr[2], pr[3]);
          *reinterpret_cast<uint4*>(tile + (uint32_t)(2 + half) * kYLbo) = make_uint4(pi[0], pi[1], pi[2], pi[3]);
        }
      }
    }
    to_mma();
    // ---- stage B': IDFT16(V) per pair into TMEM columns [32 p, 32 p + 32)
    if (pt == 0) {
      for (int p = 0; p < P; ++p) {
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          tc::mma_f16(tmem + (uint32_t)(32 * p), tc::desc_kmajor(ws + (p + 1) * kYTile + kk * 2 * kYLbo, kYLbo, kYSbo),
                      tc::desc_kmajor(wia + kk * 2 * kYLbo, kYLbo, kYSbo), idY, kk > 0 ? 1u : 0u);
      }
      tc::mma_commit(mbar);
    }
    if (!mma_wait()) { failed = true; break; }
    // ---- pass 3: Z = W w_2048^(-k1 n2) (= 32 conj(tw)), MN-major (K rows re k1 | im k1) for stage A'
    const uint32_t lboZ = (uint32_t)(P * kN2 / 8) * 128;  // Z: MN-major, 256 K-rows x P*16 columns
    {
      float2 tw[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 w = tws[row * kN2 + 8 * half + i];
        tw[i] = make_float2(32.f * w.x, -32.f * w.y);
      }
#pragma unroll 1
      for (int p = 0; p < P; p += 2) {
        const bool two = p + 1 < P;
        uint32_t zr[2][8], zi[2][8];
        tc::tmem_ld8(tmem + lane_off + (uint32_t)(32 * p + 8 * half), zr[0]);
        tc::tmem_ld8(tmem + lane_off + (uint32_t)(32 * p + 16 + 8 * half), zi[0]);
        if (two) {
          tc::tmem_ld8(tmem + lane_off + (uint32_t)(32 * (p + 1) + 8 * half), zr[1]);
          tc::tmem_ld8(tmem + lane_off + (uint32_t)(32 * (p + 1) + 16 + 8 * half), zi[1]);
        }
        tc::tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            tc::tmem_regs_ready(zr[q][i]);
            tc::tmem_regs_ready(zi[q][i]);
          }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (q == 1 && !two) break;
          uint32_t pr[4], pi[4];
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            const float2 a = cmul(make_float2(__uint_as_float(zr[q][i]), __uint_as_float(zi[q][i])), tw[i]);
            const float2 b = cmul(make_float2(__uint_as_float(zr[q][i + 1]), __uint_as_float(zi[q][i + 1])), tw[i + 1]);
            pr[i / 2] = Op<T>::pack(a.x, b.x);
            pi[i / 2] = Op<T>::pack(a.y, b.y);
          }
          const int n = (p + q) * kN2 + 8 * half;
          const uint32_t offr = (uint32_t)(n >> 3) * 128 + (uint32_t)(row >> 3) * lboZ + (uint32_t)(row & 7) * 16;
          *reinterpret_cast<uint4*>(wsp + offr) = make_uint4(pr[0], pr[1], pr[2], pr[3]);
          *reinterpret_cast<uint4*>(wsp + offr + 16 * lboZ) = make_uint4(pi[0], pi[1], pi[2], pi[3]);
        }
      }
    }
    to_mma();
    // ---- stage A': y = CA^T Zr + CB^T Zi into TMEM columns [0, P*16)
    if (pt == 0) {
      const uint32_t idB = tc::idesc_f16(128, P * kN2, Op<T>::bf16, 1, 1);
      const uint32_t zr = ws, zi = ws + 16 * lboZ;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(ca + kk * 2 * kCSbo, kCSbo, kCLbo),
                    tc::desc_kmajor(zr + kk * 2 * lboZ, lboZ, 128), idB, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(cb + kk * 2 * kCSbo, kCSbo, kCLbo),
                    tc::desc_kmajor(zi + kk * 2 * lboZ, lboZ, 128), idB, 1u);
      tc::mma_commit(mbar);
    }
    if (!mma_wait()) { failed = true; break; }
    // ---- epilogue: lane j -> (row of the pair c = j / 64, n1 = j % 64), columns n2 = 8 half .. +8 of each pair
    {
      const int c = row >> 6, n1 = row & 63;
#pragma unroll 1
      for (int p = 0; p < P; p += 2) {
        const bool two = p + 1 < P;
        uint32_t v[2][8];
        tc::tmem_ld8(tmem + lane_off + (uint32_t)(p * kN2 + 8 * half), v[0]);
        if (two) tc::tmem_ld8(tmem + lane_off + (uint32_t)((p + 1) * kN2 + 8 * half), v[1]);
        tc::tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int i = 0; i < 8; ++i) tc::tmem_regs_ready(v[q][i]);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (q == 1 && !two) break;
          const int brow = 2 * (g * kMaxPairs + p + q) + c;
          if (brow < B) {
            const size_t o = ((size_t)brow * H + h) * kL + (size_t)n1 * kN2 + 8 * half;
            *reinterpret_cast<uint4*>(yb + o) =
                make_uint4(Op<T>::pack(__uint_as_float(v[q][0]), __uint_as_float(v[q][1])),
                           Op<T>::pack(__uint_as_float(v[q][2]), __uint_as_float(v[q][3])),
                           Op<T>::pack(__uint_as_float(v[q][4]), __uint_as_float(v[q][5])),
                           Op<T>::pack(__uint_as_float(v[q][6]), __uint_as_float(v[q][7])));
          }
        }
      }
    }
    tc::fence_before_sync();  // the epilogue's TMEM reads precede the next item's MMAs (ordered by to_mma)
  }
  cp_async_wait_all();
  if (failed && pt == 0) atomicAdd(&g_fftconv_tc_timeouts, 1u);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(*tmem_p, kPipes * kPipeCols);
}

template <typename T>
static cudaError_t fftconv_tc_t(const void* u, const float* f, const float* D, void* y, int B, int H, bool pdl,
                                cudaStream_t st, bool conj_filter) {
  cudaError_t e = smem_optin<fftconv_tc_kernel<T>>(kSmem);
  if (e != cudaSuccess) return e;
  const long long items = (long long)H * (((B + 1) / 2 + kMaxPairs - 1) / kMaxPairs);
  const long long per_cta = 2;  // two pipelines per CTA
  const int sms = num_sms();
  const int grid = (int)((items + per_cta - 1) / per_cta < sms ? (items + per_cta - 1) / per_cta : sms);
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
