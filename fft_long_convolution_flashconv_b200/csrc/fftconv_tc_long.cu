// Fused FFT convolution for L = 2048, 4096, 8192 with the block-FFT stages on
// the 5th-generation tensor cores (fp16 / bf16 I/O).
//
// H3 summary section 4 "Short-sequence computation": FFT, pointwise multiply
// and inverse FFT fused in one kernel, the FFT written as matrix multiplies
// (a block FFT) so it runs on the tensor cores, up to 8K (H3 blog, "Fused
// Block FFTConv").
//
// M = 2L = 128 N2, N2 = 16 R (R = 2, 4, 8).  Index split n = N2 n1 + n2,
// k = k1 + 128 k2 (n1, k1 < 128; n2, k2 < N2), w_K = exp(-2 pi i / K):
//   X[k1 + 128 k2] = sum_n2 w_N2^(n2 k2) w_M^(n2 k1) sum_{n1<64} w_128^(n1 k1) x[N2 n1 + n2]
// The column DFT over n2 is split once more, n2 = n2a + 16 n2b and
// k2 = R k2a + k2b (n2a, k2a < 16; n2b, k2b < R):
//   w_N2^(n2 k2) = w_16^(n2a k2a) w_N2^(n2a k2b) w_R^(n2b k2b)
// so the forward transform is
//   stage A  (GEMM)   Y[k1][n2]       = sum_{n1<64} w_128^(n1 k1) x[N2 n1 + n2]     (zero padding: n1 < 64)
//   pass 1  (regs)    Z[k1][n2a][k2b] = w_M^(k1 n2a) sum_n2b w_R^(n2b k2b) w_M^(16 k1 n2b) Y[k1][n2a + 16 n2b] / (32 R)
//   stage B  (GEMM)   X[k1 + 128 (R k2a + k2b)] = sum_n2a G_k2b[n2a][k2a] Z[k1][n2a][k2b]
//                     with G_k2b[n2a][k2a] = w_N2^(n2a (R k2a + k2b))  (one 32 x 32 real block per k2b)
// and the inverse runs the same steps backwards with conjugate factors:
//   pass 2  (regs)    V = X . F^ . 32 R / M            (F^ the filter's transform, kept in TMEM)
//   stage B' (GEMM)   W[k1][n2a][k2b] = sum_k2a conj(G_k2b[n2a][k2a]) V[k1 + 128 (R k2a + k2b)]
//   pass 3  (regs)    Z'[k1][n2a + 16 n2b] = 32 R w_M^(-k1 (n2a + 16 n2b)) sum_k2b w_R^(-n2b k2b) W[k1][n2a][k2b]
//   stage A' (GEMM)   y[N2 n1 + n2] = sum_k1 w_128^(-n1 k1) Z'[k1][n2],  n1 < 64
// The R-point DFTs of passes 1 and 3 run in registers; every other DFT is a
// GEMM with fp32 accumulation in TMEM.  Stages A and A' use the constant
// DFT-128 blocks CA, CB of the L = 1024 kernel (data operands in the I/O
// type); stages B and B' take fp16 operands, scaled by 1/(32 R) so that the
// stage-B input stays within 2 max|u|.  The constant blocks and twiddle
// bases come from tables built with the library (tc_tables.inc).
//
// Work: one CTA per SM walks a contiguous range of (channel, row pair)
// items; two real rows are packed as u0 + i u1 (f is real, so the real and
// imaginary outputs are the two convolutions).  When the channel changes,
// the filter (with D added to its tap 0) goes through stages A and B into a
// TMEM region that every pair of the channel then reads in pass 2.  The next
// pair's rows (or the next channel's filter) are copied in (the rows by two
// tensor-map copies from one thread, the filter with cp.async) as
// soon as stage A has released the input buffer.  All 16 warps take part in
// every pass: warp w serves TMEM lane quarter w % 4 and the column group
// w / 4.  Waits on MMA completion are bounded; a CTA that gives up counts it
// in a device word, skips its remaining work and frees its TMEM.
#include "fft_stockham.cuh"
#include "kernels.cuh"
#include "tc100.cuh"
#include "tmap.cuh"

#define FC_TABLES_DFT128
#define FC_TABLES_LONG
#include "tc_tables.inc"

namespace fc {

static __device__ unsigned int g_fftconv_tcl_timeouts;

namespace {
constexpr int kThrL = 512;
constexpr uint64_t kWaitNsL = 2000000000ull;
constexpr uint32_t kCLbo = 128, kCSbo = 16 * 128;  // CA / CB: 128 rows x 128 K, K-major
constexpr uint32_t kCBytes = 128 * 128 * 2;
constexpr uint32_t kTLbo = 128, kTSbo = 512, kTile = 128 * 32 * 2;  // stage-B tiles: 128 rows x 32 K, K-major

template <int R>
struct LG {
  static constexpr int N2 = 16 * R, Lc = 64 * N2, M = 2 * Lc;
  static constexpr uint32_t lboX = (N2 / 8) * 128;  // X planes: MN-major, 64 K-rows (n1) x N2 columns (n2)
  static constexpr uint32_t xplane = 64 * N2 * 2;
  static constexpr uint32_t lboZ = (N2 / 8) * 128;  // Z: MN-major, 256 K-rows (re k1 | im k1) x N2 columns
  static constexpr uint32_t yv = R * kTile;         // R stage-B tiles, later Z (256 * N2 * 2 bytes, the same)
  static constexpr uint32_t tcols = 4 * N2;         // TMEM: work [0, 2 N2) | filter [2 N2, 4 N2)
  static constexpr uint32_t o_ca = 0, o_cb = kCBytes, o_gf = 2 * kCBytes, o_gi = o_gf + R * 2048,
                            o_x = o_gi + R * 2048, o_yv = o_x + 2 * xplane, o_fst = o_yv + yv,
                            o_mbar = o_fst + 4 * Lc, o_tmem = o_mbar + 16,  // MMA and row-copy barriers
                            bytes = o_tmem + 8;
  static_assert(256u * N2 * 2 == yv, "Z must fit the stage-B tiles");
};

template <typename T> struct OpL;
template <> struct OpL<__half> {
  static constexpr int bf16 = 0;
  static __device__ __forceinline__ const uint16_t* ca() { return g_ca_f16; }
  static __device__ __forceinline__ const uint16_t* cb() { return g_cb_f16; }
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};
template <> struct OpL<__nv_bfloat16> {
  static constexpr int bf16 = 1;
  static __device__ __forceinline__ const uint16_t* ca() { return g_ca_bf16; }
  static __device__ __forceinline__ const uint16_t* cb() { return g_cb_bf16; }
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};
__device__ __forceinline__ uint32_t pack_h(float a, float b) { return OpL<__half>::pack(a, b); }

// per-R tables: stage-B blocks [k2b][forward, inverse], ta[k1][n2a], tb[k1][n2b]
template <int R> struct LT;
template <> struct LT<2> {
  static __device__ __forceinline__ const uint16_t* blocks() { return g_gblk_r2; }
  static __device__ __forceinline__ const float* ta() { return g_ta_r2; }
  static __device__ __forceinline__ const float* tb() { return g_tb_r2; }
};
template <> struct LT<4> {
  static __device__ __forceinline__ const uint16_t* blocks() { return g_gblk_r4; }
  static __device__ __forceinline__ const float* ta() { return g_ta_r4; }
  static __device__ __forceinline__ const float* tb() { return g_tb_r4; }
};
template <> struct LT<8> {
  static __device__ __forceinline__ const uint16_t* blocks() { return g_gblk_r8; }
  static __device__ __forceinline__ const float* ta() { return g_ta_r8; }
  static __device__ __forceinline__ const float* tb() { return g_tb_r8; }
};

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ float2 f2(uint32_t re, uint32_t im) { return make_float2(__uint_as_float(re), __uint_as_float(im)); }
}  // namespace

// u, y: rows of a B x H x Lrow array, each holding C chunks of length Lc
// (sub-row q of channel h at ((q / C) H + h) Lrow + (q % C) Lc); f: H rows of
// fstride floats (Lc taps used); D: H.
template <typename T, int R>
__global__ void __launch_bounds__(kThrL, 1)
    fftconv_tcl_kernel(const T* __restrict__ u, const float* __restrict__ f, int fstride, const float* __restrict__ D,
                       T* __restrict__ y, int B, int H, long long Lrow, int C, int conj_filter,
                       const __grid_constant__ CUtensorMap umap) {
  using G = LG<R>;
  constexpr int N2 = G::N2, Lc = G::Lc, M = G::M;
  extern __shared__ __align__(1024) uint8_t sm[];
  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + G::o_mbar);
  uint64_t* mbar_ld = mbar + 1;  // a pair's rows landed in the X planes (tensor-map copies)
  uint32_t* tmem_p = reinterpret_cast<uint32_t*>(sm + G::o_tmem);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int row = tid & 127;  // TMEM lane: k1 in the passes, output lane j in the epilogue
  const int set = warp >> 2;  // column group 0..3
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  uint16_t* yb = reinterpret_cast<uint16_t*>(y);
  const uint32_t s_base = tc::smem_u32(sm);
  const uint32_t ca = s_base + G::o_ca, cb = s_base + G::o_cb, gf = s_base + G::o_gf, gi = s_base + G::o_gi;
  const uint32_t xr = s_base + G::o_x, xi = xr + G::xplane, yv = s_base + G::o_yv, fst = s_base + G::o_fst;

  if (warp == 0) tc::tmem_alloc(tmem_p, G::tcols);
  if (tid == 0) {
    tc::mbar_init(mbar, 1);
    tc::mbar_init(mbar_ld, 1);
    tc::fence_mbar_init();
  }
  // constant blocks (tables built with the library, already in the operand layouts): CA, CB in the
  // I/O type; the forward / inverse stage-B blocks of every k2b in fp16
  {
    const uint8_t* gca = reinterpret_cast<const uint8_t*>(OpL<T>::ca());
    const uint8_t* gcb = reinterpret_cast<const uint8_t*>(OpL<T>::cb());
    const uint8_t* gbl = reinterpret_cast<const uint8_t*>(LT<R>::blocks());
    for (int i = tid; i < (int)(kCBytes / 16); i += kThrL) {
      cp_async16(ca + i * 16, gca + i * 16);
      cp_async16(cb + i * 16, gcb + i * 16);
    }
    for (int i = tid; i < R * 2 * 128; i += kThrL) {  // block (2 k2b + inv), 128 chunks of 16 bytes each
      const int blk = i >> 7, k2b = blk >> 1, inv = blk & 1;
      cp_async16((inv ? gi : gf) + k2b * 2048 + (i & 127) * 16, gbl + i * 16);
    }
    cp_async_commit();
  }
  // this thread's twiddle factors: k1 = row, n2a = 4 set + l, n2b < R (from the tables)
  float2 ta_s[4], ta_c[4], tb[R];
#pragma unroll
  for (int l = 0; l < 4; ++l) {
    const float2 t = *reinterpret_cast<const float2*>(LT<R>::ta() + 2 * (row * 16 + 4 * set + l));
    ta_s[l] = make_float2(t.x * (1.f / (32.f * R)), t.y * (1.f / (32.f * R)));
    ta_c[l] = make_float2(t.x * (32.f * R), -t.y * (32.f * R));
  }
#pragma unroll
  for (int b2 = 0; b2 < R; ++b2) tb[b2] = *reinterpret_cast<const float2*>(LT<R>::tb() + 2 * (row * R + b2));
  cp_async_wait_all();
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_p;
  const uint32_t tw = tmem, tf = tmem + 2 * N2;  // work / filter regions

  const int Q = B * C;
  const int NP = (Q + 1) / 2;
  const long long total = (long long)H * NP;
  const long long it0 = (long long)blockIdx.x * total / gridDim.x;
  const long long it1 = (long long)(blockIdx.x + 1) * total / gridDim.x;
  auto row_off = [&](int h, int q) -> size_t {
    return ((size_t)(q / C) * H + h) * (size_t)Lrow + (size_t)(q % C) * Lc;
  };
  // a pair's rows into the X planes: one tensor-map copy per row (thread 0), each box
  // (8 n2, 8 n1 % 8, N2 / 8 column groups, 8 n1 / 8) landing in the operand layout; a
  // missing second row lies past the last row of the map and arrives as zeros
  uint32_t ph_ld = 0;
  bool ld_pend = false;  // a pair's copies are in flight
  auto issue_pair = [&](long long it) {
    if (tid == 0) {
      const int h = (int)(it / NP), p = (int)(it - (long long)h * NP);
      const int q0 = 2 * p, q1 = 2 * p + 1;
      tc::mbar_expect_tx(mbar_ld, 2u * G::xplane);
      tc::tma_load_5d(xr, &umap, 0, 0, 0, 8 * (q0 % C), (q0 / C) * H + h, mbar_ld);
      tc::tma_load_5d(xi, &umap, 0, 0, 0, 8 * (q1 % C), (q1 / C) * H + h, mbar_ld);
    }
  };
  auto wait_pair = [&]() -> bool {  // all threads; bounded
    const bool ok = tc::mbar_wait_bounded(mbar_ld, ph_ld, kWaitNsL);
    ph_ld ^= 1u;
    return ok;
  };
  auto issue_filter = [&](int h) {
    const float* fr = f + (size_t)h * fstride;
    for (int idx = tid; idx < Lc / 4; idx += kThrL) cp_async16(fst + idx * 16, fr + idx * 4);
  };

  uint32_t phase = 0;
  bool failed = false;
  int hcur = -1;
  auto mma_wait = [&]() -> bool {  // all threads: wait for the MMAs committed to mbar
    const bool ok = tc::mbar_wait_bounded(mbar, phase, kWaitNsL);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) return false;
    tc::fence_after_sync();
    return true;
  };
  auto smem_to_mma = [&]() {
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
  };
  // pass 1: TMEM (Y at [base, base + 2 N2)) -> twiddle, DFT-R, twiddle -> the R stage-B tiles
  auto pass1 = [&](uint32_t base) {
#pragma unroll
    for (int lp = 0; lp < 2; ++lp) {
      uint32_t yr[R][2], yi[R][2];
#pragma unroll
      for (int b2 = 0; b2 < R; ++b2) {
        const uint32_t col = (uint32_t)(16 * b2 + 4 * set + 2 * lp);
        tc::tmem_ld2(base + lane_off + col, yr[b2]);
        tc::tmem_ld2(base + lane_off + N2 + col, yi[b2]);
      }
      tc::tmem_wait_ld();
#pragma unroll
      for (int b2 = 0; b2 < R; ++b2)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          tc::tmem_regs_ready(yr[b2][e]);
          tc::tmem_regs_ready(yi[b2][e]);
        }
      float2 z[2][R];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float2 v[R];
#pragma unroll
        for (int b2 = 0; b2 < R; ++b2) {
          v[b2] = f2(yr[b2][e], yi[b2][e]);
          if (b2 > 0) v[b2] = cmul(v[b2], tb[b2]);
        }
        dft<R, -1>(v);
#pragma unroll
        for (int k2b = 0; k2b < R; ++k2b) z[e][k2b] = cmul(v[k2b], ta_s[2 * lp + e]);
      }
#pragma unroll
      for (int k2b = 0; k2b < R; ++k2b) {
        uint8_t* tile = sm + G::o_yv + (uint32_t)k2b * kTile + (uint32_t)(row >> 3) * kTSbo + (uint32_t)(row & 7) * 16;
        const int K = 4 * set + 2 * lp;  // re at K, im at 16 + K
        *reinterpret_cast<uint32_t*>(tile + (uint32_t)(K >> 3) * kTLbo + (uint32_t)(K & 7) * 2) =
            pack_h(z[0][k2b].x, z[1][k2b].x);
        *reinterpret_cast<uint32_t*>(tile + (uint32_t)((16 + K) >> 3) * kTLbo + (uint32_t)(K & 7) * 2) =
            pack_h(z[0][k2b].y, z[1][k2b].y);
      }
    }
  };
  // stage B / B': per k2b, D[dst + 32 k2b] = tile_k2b x blocks_k2b
  auto issue_stage_b = [&](uint32_t dst, uint32_t blocks) {
    const uint32_t idY = tc::idesc_f16(128, 32, 0);
#pragma unroll
    for (int k2b = 0; k2b < R; ++k2b)
#pragma unroll
      for (int kk = 0; kk < 2; ++kk)
        tc::mma_f16(dst + (uint32_t)(32 * k2b), tc::desc_kmajor(yv + k2b * kTile + kk * 2 * kTLbo, kTLbo, kTSbo),
                    tc::desc_kmajor(blocks + k2b * 2048 + kk * 2 * kTLbo, kTLbo, kTSbo), idY, kk > 0 ? 1u : 0u);
  };
  // stage A for the pair (with_xi) or the real filter sequence, into TMEM [dst, dst + 2 N2)
  auto issue_stage_a = [&](uint32_t dst, bool with_xi) {
    const uint32_t idA = tc::idesc_f16(128, N2, OpL<T>::bf16, 0, 1);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      tc::mma_f16(dst, tc::desc_kmajor(ca + kk * 256, kCLbo, kCSbo), tc::desc_kmajor(xr + kk * 2 * G::lboX, G::lboX, 128),
                  idA, kk > 0 ? 1u : 0u);
    if (with_xi) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc::mma_f16(dst, tc::desc_kmajor(ca + (4 + kk) * 256, kCLbo, kCSbo),
                    tc::desc_kmajor(xi + kk * 2 * G::lboX, G::lboX, 128), idA, 1u);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc::mma_f16(dst + N2, tc::desc_kmajor(ca + kk * 256, kCLbo, kCSbo),
                    tc::desc_kmajor(xi + kk * 2 * G::lboX, G::lboX, 128), idA, kk > 0 ? 1u : 0u);
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      tc::mma_f16(dst + N2, tc::desc_kmajor(cb + kk * 256, kCLbo, kCSbo),
                  tc::desc_kmajor(xr + kk * 2 * G::lboX, G::lboX, 128), idA, (with_xi || kk > 0) ? 1u : 0u);
  };

  // the first item always starts a channel: its filter (written by the kernel
  // this one may be launched as a programmatic dependent of) is read after the wait
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (it0 < it1) issue_filter((int)(it0 / NP));
  cp_async_commit();

  for (long long it = it0; it < it1 && !failed; ++it) {
    const int h = (int)(it / NP), p = (int)(it - (long long)h * NP);
    if (h != hcur) {
      // ---- filter of channel h: fp32 staging -> X real plane in the I/O type (D folded into tap 0)
      cp_async_wait_all();
      __syncthreads();
      const float dh = D[h];
      for (int idx = tid; idx < 64 * (N2 / 8); idx += kThrL) {
        const int n1 = idx / (N2 / 8), c8 = idx - n1 * (N2 / 8);
        const int t = n1 * N2 + c8 * 8;
        float4 a = *reinterpret_cast<const float4*>(sm + G::o_fst + t * 4);
        const float4 b = *reinterpret_cast<const float4*>(sm + G::o_fst + t * 4 + 16);
        if (t == 0) a.x += dh;  // y = f * u + D u = (f + D delta) * u
        const uint32_t off = (uint32_t)c8 * 128 + (uint32_t)(n1 >> 3) * G::lboX + (uint32_t)(n1 & 7) * 16;
        *reinterpret_cast<uint4*>(sm + G::o_x + off) = make_uint4(OpL<T>::pack(a.x, a.y), OpL<T>::pack(a.z, a.w),
                                                                 OpL<T>::pack(b.x, b.y), OpL<T>::pack(b.z, b.w));
      }
      smem_to_mma();
      if (tid == 0) {
        issue_stage_a(tw, false);
        tc::mma_commit(mbar);
      }
      if (!mma_wait()) { failed = true; break; }
      issue_pair(it);  // the X planes are free again
      ld_pend = true;
      pass1(tw);
      smem_to_mma();
      if (tid == 0) {
        issue_stage_b(tf, gf);  // F^ / (32 R) into the filter region
        tc::mma_commit(mbar);
      }
      if (!mma_wait()) { failed = true; break; }
      hcur = h;
    }
    // ---- the pair: stage A (its rows were copied in during the previous item, or above)
    if (__syncthreads_or(!wait_pair())) { failed = true; break; }
    ld_pend = false;
    smem_to_mma();
    if (tid == 0) {
      issue_stage_a(tw, true);
      tc::mma_commit(mbar);
    }
    if (!mma_wait()) { failed = true; break; }
    // the X planes (and the filter staging) are free: prefetch the next item
    if (it + 1 < it1) {
      const int hn = (int)((it + 1) / NP);
      if (hn == h) {
        issue_pair(it + 1);
        ld_pend = true;
      } else {
        issue_filter(hn);
      }
    }
    cp_async_commit();
    pass1(tw);
    smem_to_mma();
    if (tid == 0) {
      issue_stage_b(tw, gf);
      tc::mma_commit(mbar);
    }
    if (!mma_wait()) { failed = true; break; }
    // ---- pass 2: V = X . F^ . 32 R / M into the stage-B tiles (conj(F^) for the correlation)
    {
      constexpr float sc = 32.0f * R / (float)M;
      const float sci = conj_filter ? -sc : sc;
      for (int k2b = set; k2b < R; k2b += 4) {
        float xr_[16], xi_[16], fr_[16], fi_[16];
        tc::tmem_ld16x2_wait(tw + lane_off + (uint32_t)(32 * k2b), tw + lane_off + (uint32_t)(32 * k2b + 16), xr_, xi_);
        tc::tmem_ld16x2_wait(tf + lane_off + (uint32_t)(32 * k2b), tf + lane_off + (uint32_t)(32 * k2b + 16), fr_, fi_);
        uint32_t pr[8], pi[8];
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          const float2 a = cmul(make_float2(xr_[k], xi_[k]), make_float2(fr_[k] * sc, fi_[k] * sci));
          const float2 b = cmul(make_float2(xr_[k + 1], xi_[k + 1]), make_float2(fr_[k + 1] * sc, fi_[k + 1] * sci));
          pr[k / 2] = pack_h(a.x, b.x);
          pi[k / 2] = pack_h(a.y, b.y);
        }
        uint8_t* tile = sm + G::o_yv + (uint32_t)k2b * kTile + (uint32_t)(row >> 3) * kTSbo + (uint32_t)(row & 7) * 16;
        *reinterpret_cast<uint4*>(tile) = make_uint4(pr[0], pr[1], pr[2], pr[3]);
        *reinterpret_cast<uint4*>(tile + kTLbo) = make_uint4(pr[4], pr[5], pr[6], pr[7]);
        *reinterpret_cast<uint4*>(tile + 2 * kTLbo) = make_uint4(pi[0], pi[1], pi[2], pi[3]);
        *reinterpret_cast<uint4*>(tile + 3 * kTLbo) = make_uint4(pi[4], pi[5], pi[6], pi[7]);
      }
    }
    smem_to_mma();
    if (tid == 0) {
      issue_stage_b(tw, gi);
      tc::mma_commit(mbar);
    }
    if (!mma_wait()) { failed = true; break; }
    // ---- pass 3: Z' = 32 R w_M^(-k1 n2) IDFT-R(W) into the MN-major Z tile (K rows re k1 | im k1)
#pragma unroll
    for (int lp = 0; lp < 2; ++lp) {
      uint32_t wr[R][2], wi[R][2];
#pragma unroll
      for (int k2b = 0; k2b < R; ++k2b) {
        const uint32_t col = (uint32_t)(32 * k2b + 4 * set + 2 * lp);
        tc::tmem_ld2(tw + lane_off + col, wr[k2b]);
        tc::tmem_ld2(tw + lane_off + col + 16, wi[k2b]);
      }
      tc::tmem_wait_ld();
#pragma unroll
      for (int k2b = 0; k2b < R; ++k2b)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          tc::tmem_regs_ready(wr[k2b][e]);
          tc::tmem_regs_ready(wi[k2b][e]);
        }
      float2 z[2][R];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float2 v[R];
#pragma unroll
        for (int k2b = 0; k2b < R; ++k2b) v[k2b] = cmul(f2(wr[k2b][e], wi[k2b][e]), ta_c[2 * lp + e]);
        dft<R, 1>(v);
#pragma unroll
        for (int b2 = 0; b2 < R; ++b2) z[e][b2] = b2 > 0 ? cmul(v[b2], cconj(tb[b2])) : v[b2];
      }
#pragma unroll
      for (int b2 = 0; b2 < R; ++b2) {
        const int n2 = 4 * set + 2 * lp + 16 * b2;
        const uint32_t offr = (uint32_t)(n2 >> 3) * 128 + (uint32_t)(row >> 3) * G::lboZ + (uint32_t)(row & 7) * 16 +
                              (uint32_t)(n2 & 7) * 2;
        *reinterpret_cast<uint32_t*>(sm + G::o_yv + offr) = OpL<T>::pack(z[0][b2].x, z[1][b2].x);
        *reinterpret_cast<uint32_t*>(sm + G::o_yv + offr + 16 * G::lboZ) = OpL<T>::pack(z[0][b2].y, z[1][b2].y);
      }
    }
    smem_to_mma();
    if (tid == 0) {  // stage A': y = CA^T Zr + CB^T Zi into TMEM [0, N2)
      const uint32_t idB = tc::idesc_f16(128, N2, OpL<T>::bf16, 1, 1);
      const uint32_t zr = yv, zi = yv + 16 * G::lboZ;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        tc::mma_f16(tw, tc::desc_kmajor(ca + kk * 2 * kCSbo, kCSbo, kCLbo), tc::desc_kmajor(zr + kk * 2 * G::lboZ, G::lboZ, 128),
                    idB, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        tc::mma_f16(tw, tc::desc_kmajor(cb + kk * 2 * kCSbo, kCSbo, kCLbo), tc::desc_kmajor(zi + kk * 2 * G::lboZ, G::lboZ, 128),
                    idB, 1u);
      tc::mma_commit(mbar);
    }
    if (!mma_wait()) { failed = true; break; }
    // ---- epilogue: lane j -> (row of the pair c = j / 64, n1 = j % 64), columns n2 of this warp's group
    {
      const int c = row >> 6, n1 = row & 63;
      const int q = 2 * p + c;
      if (q < Q) {
        uint16_t* yr = yb + row_off(h, q) + (size_t)n1 * N2;
        constexpr int CPS = N2 / 4;  // columns per warp group
        uint32_t v[CPS / 8][8];
#pragma unroll
        for (int c8 = 0; c8 < CPS / 8; ++c8) tc::tmem_ld8(tw + lane_off + (uint32_t)(set * CPS + c8 * 8), v[c8]);
        tc::tmem_wait_ld();  // one wait for all of this thread's columns
#pragma unroll
        for (int c8 = 0; c8 < CPS / 8; ++c8) {
#pragma unroll
          for (int e = 0; e < 8; ++e) tc::tmem_regs_ready(v[c8][e]);
          *reinterpret_cast<uint4*>(yr + set * CPS + c8 * 8) =
              make_uint4(OpL<T>::pack(__uint_as_float(v[c8][0]), __uint_as_float(v[c8][1])),
                         OpL<T>::pack(__uint_as_float(v[c8][2]), __uint_as_float(v[c8][3])),
                         OpL<T>::pack(__uint_as_float(v[c8][4]), __uint_as_float(v[c8][5])),
                         OpL<T>::pack(__uint_as_float(v[c8][6]), __uint_as_float(v[c8][7])));
        }
      }
    }
    tc::fence_before_sync();  // the epilogue's TMEM reads precede the next item's MMAs
  }
  cp_async_wait_all();
  if (ld_pend) (void)tc::mbar_wait_bounded(mbar_ld, ph_ld, kWaitNsL);  // copies in flight land first
  if (failed && tid == 0) atomicAdd(&g_fftconv_tcl_timeouts, 1u);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, G::tcols);
}

template <int R>
static cudaError_t make_row_map(CUtensorMap* m, const void* u, int B, int H, long long Lrow, int C) {
  constexpr int N2 = LG<R>::N2;
  const cuuint64_t dims[5] = {8, 8, (cuuint64_t)(N2 / 8), (cuuint64_t)(8 * C), (cuuint64_t)B * (cuuint64_t)H};
  const cuuint64_t strides[4] = {(cuuint64_t)(2 * N2), 16, (cuuint64_t)(16 * N2), (cuuint64_t)(2 * Lrow)};
  const cuuint32_t box[5] = {8, 8, (cuuint32_t)(N2 / 8), 8, 1};
  return encode_map_5d_u16(m, u, dims, strides, box);
}

template <typename T, int R>
static cudaError_t tcl_t(const void* u, const float* f, int fstride, const float* D, void* y, int B, int H,
                         long long Lrow, int C, bool pdl, int conj_filter, cudaStream_t st) {
  CUtensorMap umap;
  cudaError_t e0 = make_row_map<R>(&umap, u, B, H, Lrow, C);
  if (e0 != cudaSuccess) return e0;
  const size_t smem = LG<R>::bytes;
  cudaError_t e = smem_optin<fftconv_tcl_kernel<T, R>>(smem);
  if (e != cudaSuccess) return e;
  const long long items = (long long)H * ((B * C + 1) / 2);
  const int grid = (int)(items < num_sms() ? items : num_sms());
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThrL);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fftconv_tcl_kernel<T, R>, (const T*)u, f, fstride, D, (T*)y, B, H, Lrow, C,
                            conj_filter, umap);
}

bool fftconv_tcl_supported(int Lc, int dtype) { return (dtype == 1 || dtype == 2) && (Lc == 2048 || Lc == 4096 || Lc == 8192); }

cudaError_t launch_fftconv_tcl(const void* u, const float* f, int fstride, const float* D, void* y, int B, int H,
                               long long Lrow, int Lc, int C, int dtype, bool after_filter_kernel, bool conj_filter,
                               cudaStream_t st) {
  if (!fftconv_tcl_supported(Lc, dtype)) return cudaErrorInvalidValue;
  const int cj = conj_filter ? 1 : 0;
  if (dtype == 1) {
    switch (Lc) {
      case 2048: return tcl_t<__half, 2>(u, f, fstride, D, y, B, H, Lrow, C, after_filter_kernel, cj, st);
      case 4096: return tcl_t<__half, 4>(u, f, fstride, D, y, B, H, Lrow, C, after_filter_kernel, cj, st);
      default: return tcl_t<__half, 8>(u, f, fstride, D, y, B, H, Lrow, C, after_filter_kernel, cj, st);
    }
  }
  switch (Lc) {
    case 2048: return tcl_t<__nv_bfloat16, 2>(u, f, fstride, D, y, B, H, Lrow, C, after_filter_kernel, cj, st);
    case 4096: return tcl_t<__nv_bfloat16, 4>(u, f, fstride, D, y, B, H, Lrow, C, after_filter_kernel, cj, st);
    default: return tcl_t<__nv_bfloat16, 8>(u, f, fstride, D, y, B, H, Lrow, C, after_filter_kernel, cj, st);
  }
}

unsigned int fftconv_tcl_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_fftconv_tcl_timeouts, sizeof(v));
  return v;
}

}  // namespace fc
