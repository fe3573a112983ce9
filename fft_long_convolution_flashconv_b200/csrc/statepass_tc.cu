// State passing (A7, A9) on the 5th-generation tensor cores, for fp16 / bf16
// I/O, chunks T = 128 * NC with NC in {16, 32, 64} and N <= 64 modes.
//
// H3 summary section 4 "Long-sequence computation" and appendix C "State
// Passing": per chunk c of a (b, h) row,
//   end state    s_c[n] = B_n sum_{i<T} A_n^(T-1-i) u_c[i]                 (A7)
//   correction   y_c[t] += 2 Re sum_n C_n A_n^(t+1) x_{c-1,n}               (A9)
// Both are dense contractions once the sequence index is factored.
//
// A7, i = 128 ih + il (il < 128, ih < NC):
//   Z[r][ih] = sum_il P[r][il] u[128 ih + il],  P[2n][il] + i P[2n+1][il] = A_n^(127-il)
// is one M=128 (64 modes x re/im) N=NC K=128 GEMM whose B operand is the
// chunk of u exactly as it lies in memory; the rest,
//   sum_ih A_n^(128 (NC-1-ih)) Z_n[ih],
// is a Horner recurrence in A_n^128 along the TMEM columns of each lane.
//
// A9, t = NC th + tl (th < 128, tl < NC):
//   y[t] += sum_k AH[th][k] Q[tl][k]
//   AH[th][2n] + i AH[th][2n+1] = A_n^(NC th)                  (per head, built once)
//   Q[tl][2n]  - i Q[tl][2n+1]  = 2 C_n x_n A_n^(tl+1)          (per chunk)
// is one M=128 N=NC K=128 GEMM per chunk.
//
// Precision: every table operand is split into a 16-bit high part and a
// 16-bit remainder (hi + lo), and the MMAs sum hi*hi + hi*lo + lo*hi in fp32,
// so each table carries ~22 significant bits (16 for bf16 u-side tables);
// u itself is an exact 16-bit operand.  The correction's per-chunk operand is
// scaled by a power of two so that its largest entry sits near 2^13 (fp16
// range); the epilogue multiplies the scale back out exactly.  The powers
// assume |A_n| <= 1 (Re lambda <= 0), as for any stable SSM.
//
// One CTA owns one (b, h) row and walks its chunks; the next chunk of u is
// copied in (cp.async) while the current one is contracted.  Every wait on
// MMA completion is bounded; on a timeout the CTA counts it in a device
// word, writes nothing more and still frees its TMEM.
#include "kernels.cuh"
#include "tc100.cuh"

namespace fc {

static __device__ unsigned int g_sp_tc_timeouts;

namespace {

constexpr int kThr = 128;                                // 4 warps = 128 TMEM lanes
constexpr int kKS = 128;                                 // K of both GEMMs
constexpr uint32_t kLbo = 144, kSbo = (kKS / 8) * 144;   // padded K-major: conflict-free 16-byte stores
constexpr uint32_t kTab = (128 / 8) * kSbo;              // 128-row table, bytes
constexpr uint64_t kWaitNs = 2000000000ull;

template <typename T> struct Op16;
template <> struct Op16<__half> {
  static constexpr int bf16 = 0;
  static __device__ __forceinline__ uint32_t bits(float x) { return __half_as_ushort(__float2half_rn(x)); }
  static __device__ __forceinline__ float back(uint32_t b) { return __half2float(__ushort_as_half((unsigned short)b)); }
};
template <> struct Op16<__nv_bfloat16> {
  static constexpr int bf16 = 1;
  static __device__ __forceinline__ uint32_t bits(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
  static __device__ __forceinline__ float back(uint32_t b) {
    return __bfloat162float(__ushort_as_bfloat16((unsigned short)b));
  }
};

// hi / lo 16-bit parts of a and b, packed as (a, b) pairs (a at the lower address).
template <typename T>
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const uint32_t ha = Op16<T>::bits(a), hb = Op16<T>::bits(b);
  const uint32_t la = Op16<T>::bits(a - Op16<T>::back(ha)), lb = Op16<T>::bits(b - Op16<T>::back(hb));
  hi = ha | (hb << 16);
  lo = la | (lb << 16);
}

// Byte offset of the 16-byte group holding K elements 8*k8 .. 8*k8+7 of row r.
__device__ __forceinline__ uint32_t toff(int r, int k8) {
  return (uint32_t)(r >> 3) * kSbo + (uint32_t)k8 * kLbo + (uint32_t)(r & 7) * 16u;
}

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int K>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(K) : "memory");
}

template <int NC>
struct StateSmem {
  uint8_t ph[kTab];                // A: P hi, 128 rows (2n + re/im) x 128 K (il)
  uint8_t pl[kTab];                // A: P lo
  uint8_t ub[2][(NC / 8) * kSbo];  // B: u chunk, NC rows (ih) x 128 K (il), double-buffered
  uint64_t mbar;
  uint32_t tmem_base;
};

template <int NC>
struct CorrSmem {
  uint8_t ahh[kTab];               // A: AH hi, 128 rows (th) x 128 K (2n + re/im)
  uint8_t ahl[kTab];               // A: AH lo
  uint8_t qh[(NC / 8) * kSbo];     // B: Q hi, NC rows (tl) x 128 K
  uint8_t ql[(NC / 8) * kSbo];     // B: Q lo
  float red[kThr / 32];
  uint64_t mbar;
  uint32_t tmem_base;
};

template <int NC>
constexpr uint32_t tmem_cols() {
  return NC < 32 ? 32u : (uint32_t)NC;
}

// u chunk (NC * 128 contiguous 16-bit elements) -> K-major B tile, 16 bytes per copy.
template <int NC>
__device__ __forceinline__ void stage_u(uint8_t* dst, const uint16_t* src, int tid) {
  const uint32_t d0 = tc::smem_u32(dst);
#pragma unroll
  for (int i = 0; i < NC * 16 / kThr; ++i) {
    const int q = tid + i * kThr;  // 16-byte vector: row ih = q / 16, K group q % 16
    cp_async16(d0 + toff(q >> 4, q & 15), src + (size_t)q * 8);
  }
}

}  // namespace

// ---------------------------------------------------------------- A7: local end-states
// grid (H, B), 128 threads; s_ws[((b H + h) C + c) N + n] = s_c[n].
template <typename T, int NC>
__global__ void __launch_bounds__(kThr, 2) sp_state_tc_kernel(const T* __restrict__ u, const float* __restrict__ dt,
                                                               const float2* __restrict__ lam,
                                                               const float2* __restrict__ Bp, int H, int L, int N,
                                                               float2* __restrict__ s_ws) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  StateSmem<NC>& sm = *reinterpret_cast<StateSmem<NC>*>(smraw);
  constexpr int Tc = NC * kKS;
  const int h = blockIdx.x, b = blockIdx.y;
  const int C = L / Tc;
  const int tid = threadIdx.x, warp = tid >> 5;
  const float d = dt[h];
  const uint16_t* urow = reinterpret_cast<const uint16_t*>(u) + ((size_t)b * H + h) * (size_t)L;

  if (warp == 0) tc::tmem_alloc(&sm.tmem_base, tmem_cols<NC>());
  if (tid == 0) {
    tc::mbar_init(&sm.mbar, 1);
    tc::fence_mbar_init();
  }
  stage_u<NC>(sm.ub[0], urow, tid);
  cp_async_commit();

  // P[2n][il] + i P[2n+1][il] = A_n^(127 - il): one exact power per 8 il, then a short chain.
  for (int it = tid; it < 64 * 16; it += kThr) {
    const int n = it >> 4, g = it & 15;
    float re[8], im[8];
    if (n < N) {
      const float2 lm = lam[(size_t)h * N + n];
      const float2 a1 = ssm_pow(d, lm.x, lm.y, 1.0);
      float2 p = ssm_pow(d, lm.x, lm.y, (double)(120 - 8 * g));  // il = 8g + 7
#pragma unroll
      for (int m = 7; m >= 0; --m) {
        re[m] = p.x;
        im[m] = p.y;
        p = cmul(p, a1);
      }
    } else {
#pragma unroll
      for (int m = 0; m < 8; ++m) re[m] = im[m] = 0.f;
    }
    uint32_t rh[4], rl[4], ih_[4], il_[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      split2<T>(re[2 * m], re[2 * m + 1], rh[m], rl[m]);
      split2<T>(im[2 * m], im[2 * m + 1], ih_[m], il_[m]);
    }
    *reinterpret_cast<uint4*>(sm.ph + toff(2 * n, g)) = make_uint4(rh[0], rh[1], rh[2], rh[3]);
    *reinterpret_cast<uint4*>(sm.pl + toff(2 * n, g)) = make_uint4(rl[0], rl[1], rl[2], rl[3]);
    *reinterpret_cast<uint4*>(sm.ph + toff(2 * n + 1, g)) = make_uint4(ih_[0], ih_[1], ih_[2], ih_[3]);
    *reinterpret_cast<uint4*>(sm.pl + toff(2 * n + 1, g)) = make_uint4(il_[0], il_[1], il_[2], il_[3]);
  }

  // this lane's mode: row r = tid -> mode tid / 2, real (even) or imaginary (odd) part
  const int n = tid >> 1, part = tid & 1;
  float2 w128 = make_float2(0.f, 0.f), bn = make_float2(0.f, 0.f);
  if (n < N) {
    const float2 lm = lam[(size_t)h * N + n];
    w128 = ssm_pow(d, lm.x, lm.y, (double)kKS);
    bn = Bp[(size_t)h * N + n];
  }
  const uint32_t idesc = tc::idesc_f16(128, NC, Op16<T>::bf16);
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  uint32_t phase = 0;
  bool failed = false;
  uint32_t tmem = 0;

  for (int c = 0; c < C; ++c) {
    if (c + 1 < C) {
      stage_u<NC>(sm.ub[(c + 1) & 1], urow + (size_t)(c + 1) * Tc, tid);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    tmem = sm.tmem_base;
    if (tid == 0) {
      const uint32_t pa = tc::smem_u32(sm.ph), pb = tc::smem_u32(sm.pl), ua = tc::smem_u32(sm.ub[c & 1]);
#pragma unroll
      for (int kk = 0; kk < kKS / 16; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(pa + kk * 2 * kLbo, kLbo, kSbo),
                    tc::desc_kmajor(ua + kk * 2 * kLbo, kLbo, kSbo), idesc, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < kKS / 16; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(pb + kk * 2 * kLbo, kLbo, kSbo),
                    tc::desc_kmajor(ua + kk * 2 * kLbo, kLbo, kSbo), idesc, 1u);
      tc::mma_commit(&sm.mbar);
    }
    const bool ok = tc::mbar_wait_bounded(&sm.mbar, phase, kWaitNs);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    float z[NC];
#pragma unroll
    for (int j = 0; j < NC; j += 16) tc::tmem_ld16_wait(tmem + lane_off + (uint32_t)j, z + j);
    // Horner in A^128 over ih: R = sum_ih z[ih] A^(128 (NC-1-ih)) (complex, from a real row)
    float ar = 0.f, ai = 0.f;
#pragma unroll
    for (int ih = 0; ih < NC; ++ih) {
      const float nr = fmaf(ar, w128.x, fmaf(-ai, w128.y, z[ih]));
      ai = fmaf(ar, w128.y, ai * w128.x);
      ar = nr;
    }
    // even lane holds R_re-row, odd lane R_im-row: sum = R_re + i R_im
    const float pr = __shfl_xor_sync(0xffffffffu, ar, 1);
    const float pi = __shfl_xor_sync(0xffffffffu, ai, 1);
    if (part == 0 && n < N) {
      const float2 s = make_float2(ar - pi, ai + pr);
      s_ws[(((size_t)b * H + h) * C + c) * N + n] = cmul(s, bn);
    }
  }
  cp_async_wait<0>();
  if (failed && tid == 0) atomicAdd(&g_sp_tc_timeouts, 1u);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(sm.tmem_base, tmem_cols<NC>());
}

// ---------------------------------------------------------------- A9: correction
// grid (H, B), 128 threads; y[b, h, c T + t] += correction, chunks c >= c_begin.
template <typename T, int NC>
__global__ void __launch_bounds__(kThr, 2) sp_corr_tc_kernel(T* __restrict__ y, const float* __restrict__ dt,
                                                              const float2* __restrict__ lam,
                                                              const float2* __restrict__ Cp,
                                                              const float2* __restrict__ x_ws, int H, int L, int N,
                                                              int c_begin) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  CorrSmem<NC>& sm = *reinterpret_cast<CorrSmem<NC>*>(smraw);
  constexpr int Tc = NC * kKS;
  const int h = blockIdx.x, b = blockIdx.y;
  const int C = L / Tc;
  const int tid = threadIdx.x, warp = tid >> 5;
  const float d = dt[h];

  if (warp == 0) tc::tmem_alloc(&sm.tmem_base, tmem_cols<NC>());
  if (tid == 0) {
    tc::mbar_init(&sm.mbar, 1);
    tc::fence_mbar_init();
  }
  // AH[th][2n] + i AH[th][2n+1] = A_n^(NC th): one exact power per 8 rows, then a chain in A^NC.
  for (int it = tid; it < 64 * 16; it += kThr) {
    const int n = it & 63, g = it >> 6;
    float2 p = make_float2(0.f, 0.f), step = make_float2(0.f, 0.f);
    if (n < N) {
      const float2 lm = lam[(size_t)h * N + n];
      p = ssm_pow(d, lm.x, lm.y, (double)NC * 8.0 * g);
      step = ssm_pow(d, lm.x, lm.y, (double)NC);
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      uint32_t hi, lo;
      split2<__half>(p.x, p.y, hi, lo);
      const uint32_t off = toff(8 * g + m, n >> 2) + (uint32_t)(n & 3) * 4u;
      *reinterpret_cast<uint32_t*>(sm.ahh + off) = hi;
      *reinterpret_cast<uint32_t*>(sm.ahl + off) = lo;
      p = cmul(p, step);
    }
  }
  // this thread's mode and Q row groups: n = tid % 64, tl groups (tid / 64) + 2 r
  constexpr int kGr = NC / 16;
  const int n = tid & 63;
  float2 a1 = make_float2(0.f, 0.f), cn = make_float2(0.f, 0.f), st[kGr];
#pragma unroll
  for (int r = 0; r < kGr; ++r) st[r] = make_float2(0.f, 0.f);
  if (n < N) {
    const float2 lm = lam[(size_t)h * N + n];
    a1 = ssm_pow(d, lm.x, lm.y, 1.0);
    cn = Cp[(size_t)h * N + n];
#pragma unroll
    for (int r = 0; r < kGr; ++r) st[r] = ssm_pow(d, lm.x, lm.y, 8.0 * ((tid >> 6) + 2 * r) + 1.0);
  }
  const uint32_t idesc = tc::idesc_f16(128, NC, 0);
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  uint32_t phase = 0;
  bool failed = false;
  uint32_t tmem = 0;
  const size_t rowoff = ((size_t)b * H + h) * (size_t)L;

  for (int c = c_begin; c < C; ++c) {
    // this lane's NC outputs t = NC * tid + tl: issue the loads of y early
    uint16_t* yp = reinterpret_cast<uint16_t*>(y) + rowoff + (size_t)c * Tc + (size_t)NC * tid;
    uint4 yv[NC / 8];
#pragma unroll
    for (int i = 0; i < NC / 8; ++i) yv[i] = *reinterpret_cast<const uint4*>(yp + 8 * i);
    float2 w = make_float2(0.f, 0.f);
    if (n < N) {
      const float2 x = x_ws[(((size_t)b * H + h) * C + c) * N + n];
      w = cmul(cn, x);
      w.x *= 2.f;
      w.y *= 2.f;
    }
    // power-of-two scale: largest |Re|, |Im| of any w_n just below 2^13
    float mx = fmaxf(fabsf(w.x), fabsf(w.y));
    mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
    if ((tid & 31) == 0) sm.red[warp] = mx;
    __syncthreads();
    mx = fmaxf(fmaxf(sm.red[0], sm.red[1]), fmaxf(sm.red[2], sm.red[3]));
    int ex = 0;
    float scale = 1.f, inv = 1.f;
    if (mx > 0.f && mx <= 3.0e38f) {
      (void)frexpf(mx, &ex);
      scale = ldexpf(1.f, 13 - ex);
      inv = ldexpf(1.f, ex - 13);
    }
    w.x *= scale;
    w.y *= scale;
    // Q[tl][2n] - i Q[tl][2n+1] = w_n A_n^(tl+1)
#pragma unroll
    for (int r = 0; r < kGr; ++r) {
      const int tg = (tid >> 6) + 2 * r;
      float2 p = cmul(w, st[r]);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        uint32_t hi, lo;
        split2<__half>(p.x, -p.y, hi, lo);
        const uint32_t off = toff(8 * tg + m, n >> 2) + (uint32_t)(n & 3) * 4u;
        *reinterpret_cast<uint32_t*>(sm.qh + off) = hi;
        *reinterpret_cast<uint32_t*>(sm.ql + off) = lo;
        p = cmul(p, a1);
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    tmem = sm.tmem_base;
    if (tid == 0) {
      const uint32_t ah = tc::smem_u32(sm.ahh), al = tc::smem_u32(sm.ahl);
      const uint32_t qh = tc::smem_u32(sm.qh), ql = tc::smem_u32(sm.ql);
#pragma unroll
      for (int kk = 0; kk < kKS / 16; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(ah + kk * 2 * kLbo, kLbo, kSbo),
                    tc::desc_kmajor(qh + kk * 2 * kLbo, kLbo, kSbo), idesc, kk > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < kKS / 16; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(ah + kk * 2 * kLbo, kLbo, kSbo),
                    tc::desc_kmajor(ql + kk * 2 * kLbo, kLbo, kSbo), idesc, 1u);
#pragma unroll
      for (int kk = 0; kk < kKS / 16; ++kk)
        tc::mma_f16(tmem, tc::desc_kmajor(al + kk * 2 * kLbo, kLbo, kSbo),
                    tc::desc_kmajor(qh + kk * 2 * kLbo, kLbo, kSbo), idesc, 1u);
      tc::mma_commit(&sm.mbar);
    }
    const bool ok = tc::mbar_wait_bounded(&sm.mbar, phase, kWaitNs);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
#pragma unroll
    for (int j = 0; j < NC; j += 16) {
      float v[16];
      tc::tmem_ld16_wait(tmem + lane_off + (uint32_t)j, v);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t* wv = reinterpret_cast<uint32_t*>(&yv[j / 8 + q]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float lo = fmaf(v[8 * q + 2 * e], inv, Op16<T>::back(wv[e] & 0xffffu));
          const float hi = fmaf(v[8 * q + 2 * e + 1], inv, Op16<T>::back(wv[e] >> 16));
          wv[e] = Op16<T>::bits(lo) | (Op16<T>::bits(hi) << 16);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < NC / 8; ++i) *reinterpret_cast<uint4*>(yp + 8 * i) = yv[i];
  }
  if (failed && tid == 0) atomicAdd(&g_sp_tc_timeouts, 1u);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(sm.tmem_base, tmem_cols<NC>());
}

// ---------------------------------------------------------------- launchers
bool statepass_tc_supported(int T, int N, int dtype) {
  return (dtype == 1 || dtype == 2) && (T == 2048 || T == 4096 || T == 8192) && N >= 1 && N <= 64;
}

template <typename T, int NC>
static cudaError_t sp_tc_t(const void* u, void* y, const float* dt, const float* lam, const float* Bp,
                           const float* Cp, int B, int H, int L, int N, float* s_ws, const float* x_ws, int c_begin,
                           bool corr, cudaStream_t st) {
  dim3 grid(H, B);
  if (!corr) {
    const size_t smem = sizeof(StateSmem<NC>) + 1024;
    auto kern = sp_state_tc_kernel<T, NC>;
    cudaError_t e = smem_optin<sp_state_tc_kernel<T, NC>>(smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThr, smem, st>>>((const T*)u, dt, (const float2*)lam, (const float2*)Bp, H, L, N, (float2*)s_ws);
  } else {
    const size_t smem = sizeof(CorrSmem<NC>) + 1024;
    auto kern = sp_corr_tc_kernel<T, NC>;
    cudaError_t e = smem_optin<sp_corr_tc_kernel<T, NC>>(smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThr, smem, st>>>((T*)y, dt, (const float2*)lam, (const float2*)Cp, (const float2*)x_ws, H, L, N,
                                   c_begin);
  }
  return cudaGetLastError();
}

template <typename T>
static cudaError_t sp_tc_nc(int T_, const void* u, void* y, const float* dt, const float* lam, const float* Bp,
                            const float* Cp, int B, int H, int L, int N, float* s_ws, const float* x_ws, int c_begin,
                            bool corr, cudaStream_t st) {
  switch (T_) {
    case 2048: return sp_tc_t<T, 16>(u, y, dt, lam, Bp, Cp, B, H, L, N, s_ws, x_ws, c_begin, corr, st);
    case 4096: return sp_tc_t<T, 32>(u, y, dt, lam, Bp, Cp, B, H, L, N, s_ws, x_ws, c_begin, corr, st);
    case 8192: return sp_tc_t<T, 64>(u, y, dt, lam, Bp, Cp, B, H, L, N, s_ws, x_ws, c_begin, corr, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_sp_state_tc(const void* u, const float* dt, const float* lam, const float* Bp, int B, int H, int L,
                               int N, int T_, float* s_ws, int dtype, cudaStream_t st) {
  if (!statepass_tc_supported(T_, N, dtype)) return cudaErrorInvalidValue;
  if (dtype == 1)
    return sp_tc_nc<__half>(T_, u, nullptr, dt, lam, Bp, nullptr, B, H, L, N, s_ws, nullptr, 0, false, st);
  return sp_tc_nc<__nv_bfloat16>(T_, u, nullptr, dt, lam, Bp, nullptr, B, H, L, N, s_ws, nullptr, 0, false, st);
}

cudaError_t launch_sp_corr_tc(void* y, const float* dt, const float* lam, const float* Cp, const float* x_ws, int B,
                              int H, int L, int N, int T_, int c_begin, int dtype, cudaStream_t st) {
  if (!statepass_tc_supported(T_, N, dtype)) return cudaErrorInvalidValue;
  if (c_begin >= L / T_) return cudaSuccess;
  if (dtype == 1)
    return sp_tc_nc<__half>(T_, nullptr, y, dt, lam, nullptr, Cp, B, H, L, N, nullptr, x_ws, c_begin, true, st);
  return sp_tc_nc<__nv_bfloat16>(T_, nullptr, y, dt, lam, nullptr, Cp, B, H, L, N, nullptr, x_ws, c_begin, true, st);
}

unsigned int statepass_tc_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_sp_tc_timeouts, sizeof(v));
  return v;
}

}  // namespace fc
