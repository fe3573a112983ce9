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
// Precision: the per-head table P is split into a 16-bit high part and a
// 16-bit remainder (hi + lo), ~16 significant bits for bf16 P; u itself is an
// exact 16-bit operand, so the end states sum Phi*u + Plo*u -- with fp16 I/O
// only Phi*u: fp16 P alone carries 11 bits, and the state's rounding stays far
// below the state tolerance.  The correction's tables AH and Q are single fp16
// tables (~11 bits, below the rounding of y itself); Q is scaled by a power of
// two so that its largest entry sits near 2^13 (fp16 range) and the epilogue
// multiplies the scale back out exactly.  The powers
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
// the u chunks arrive by asynchronous copies and go unpadded (K-major, 128-byte core-matrix stride)
constexpr uint32_t kLboU = 128, kSboU = (kKS / 8) * 128;
__device__ __forceinline__ uint32_t toff_u(int r, int k8) {
  return (uint32_t)(r >> 3) * kSboU + (uint32_t)k8 * kLboU + (uint32_t)(r & 7) * 16u;
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
constexpr uint32_t tmem_cols() {
  return NC < 32 ? 32u : (uint32_t)NC;
}

}  // namespace

// ---------------------------------------------------------------- A7: local end-states
// grid (H, B), 256 threads; s_ws[((b H + h) C + c) N + n] = s_c[n].  Warps 0-3 and 4-7
// cover the 128 TMEM lanes twice: each half runs the Horner recurrence over half of the
// chunk's NC columns, and the two partial sums combine with one product by A^(128 NC/2).
// The accumulator is double-buffered in TMEM so that chunk c+1's MMA runs during
// chunk c's recurrence, and the u chunks are double-buffered in shared memory.
constexpr int kThrS = 256;
template <int NC, bool LO>
struct StateSmem2 {
  uint8_t ph[kTab];                 // A: P hi, 128 rows (2n + re/im) x 128 K (il)
  uint8_t pl[LO ? kTab : 16];       // A: P lo (bf16 only)
  uint8_t ub[2][(NC / 8) * kSboU];  // B: u chunk, NC rows (ih) x 128 K (il), double-buffered
  float2 part[128];                // the upper half's partial sums
  uint64_t mbar[2];
  uint32_t tmem_base;
};

template <int NC>
__device__ __forceinline__ void stage_u2(uint8_t* dst, const uint16_t* src, int tid) {
  const uint32_t d0 = tc::smem_u32(dst);
  for (int q = tid; q < NC * 16; q += kThrS)  // 16-byte vector: row ih = q / 16, K group q % 16
    cp_async16(d0 + toff_u(q >> 4, q & 15), src + (size_t)q * 8);
}

template <typename T, int NC>
__global__ void __launch_bounds__(kThrS, Op16<T>::bf16 ? 2 : 3) sp_state_tc_kernel(const T* __restrict__ u, const float* __restrict__ dt,
                                                                const float2* __restrict__ lam,
                                                                const float2* __restrict__ Bp, int H, int L, int N,
                                                                float2* __restrict__ s_ws) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  StateSmem2<NC, Op16<T>::bf16 != 0>& sm = *reinterpret_cast<StateSmem2<NC, Op16<T>::bf16 != 0>*>(smraw);
  constexpr int Tc = NC * kKS;
  constexpr int HC = NC / 2;  // columns per half
  const int h = blockIdx.x, b = blockIdx.y;
  const int C = L / Tc;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int lane = tid & 127, half = tid >> 7;
  const float d = dt[h];
  const uint16_t* urow = reinterpret_cast<const uint16_t*>(u) + ((size_t)b * H + h) * (size_t)L;

  if (warp == 0) tc::tmem_alloc(&sm.tmem_base, 2 * tmem_cols<NC>());
  if (tid == 0) {
    tc::mbar_init(&sm.mbar[0], 1);
    tc::mbar_init(&sm.mbar[1], 1);
    tc::fence_mbar_init();
  }
  stage_u2<NC>(sm.ub[0], urow, tid);
  cp_async_commit();
  if (C > 1) {
    stage_u2<NC>(sm.ub[1], urow + (size_t)Tc, tid);
    cp_async_commit();
  }

  // P[2n][il] + i P[2n+1][il] = A_n^(127 - il): one exact power per 8 il, then a short chain.
  for (int it = tid; it < 64 * 16; it += kThrS) {
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
    *reinterpret_cast<uint4*>(sm.ph + toff(2 * n + 1, g)) = make_uint4(ih_[0], ih_[1], ih_[2], ih_[3]);
    if constexpr (Op16<T>::bf16 != 0) {
      *reinterpret_cast<uint4*>(sm.pl + toff(2 * n, g)) = make_uint4(rl[0], rl[1], rl[2], rl[3]);
      *reinterpret_cast<uint4*>(sm.pl + toff(2 * n + 1, g)) = make_uint4(il_[0], il_[1], il_[2], il_[3]);
    }
  }

  // this lane's mode: row r = lane -> mode lane / 2, real (even) or imaginary (odd) part
  const int n = lane >> 1, part = lane & 1;
  float2 w128 = make_float2(0.f, 0.f), w256 = make_float2(0.f, 0.f), whalf = make_float2(0.f, 0.f),
         bn = make_float2(0.f, 0.f);
  if (n < N) {
    const float2 lm = lam[(size_t)h * N + n];
    w128 = ssm_pow(d, lm.x, lm.y, (double)kKS);
    w256 = ssm_pow(d, lm.x, lm.y, 2.0 * kKS);
    whalf = ssm_pow(d, lm.x, lm.y, (double)kKS * HC);
    bn = Bp[(size_t)h * N + n];
  }
  const uint32_t idesc = tc::idesc_f16(128, NC, Op16<T>::bf16);
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  uint32_t phase = 0;  // bit b: parity of mbar[b]
  bool failed = false;
  auto issue = [&](int c) {  // MMA of chunk c into TMEM buffer c & 1
    const uint32_t pa = tc::smem_u32(sm.ph), pb = tc::smem_u32(sm.pl), ua = tc::smem_u32(sm.ub[c & 1]);
    const uint32_t tm = sm.tmem_base + (uint32_t)((c & 1) * tmem_cols<NC>());
#pragma unroll
    for (int kk = 0; kk < kKS / 16; ++kk)
      tc::mma_f16(tm, tc::desc_kmajor(pa + kk * 2 * kLbo, kLbo, kSbo),
                  tc::desc_kmajor(ua + kk * 2 * kLboU, kLboU, kSboU), idesc, kk > 0 ? 1u : 0u);
    if constexpr (Op16<T>::bf16) {  // fp16 P alone carries 11 bits; bf16 P needs its remainder
#pragma unroll
      for (int kk = 0; kk < kKS / 16; ++kk)
        tc::mma_f16(tm, tc::desc_kmajor(pb + kk * 2 * kLbo, kLbo, kSbo),
                    tc::desc_kmajor(ua + kk * 2 * kLboU, kLboU, kSboU), idesc, 1u);
    }
    tc::mma_commit(&sm.mbar[c & 1]);
  };
  // chunk 0 landed (chunk 1 may still be in flight)
  if (C > 1) cp_async_wait<1>(); else cp_async_wait<0>();
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (tid == 0) issue(0);
  for (int c = 0; c < C; ++c) {
    if (c + 1 < C) {  // chunk c+1's MMA (its u has landed; its TMEM buffer was read by chunk c-1's recurrence)
      cp_async_wait<0>();
      tc::fence_smem_to_async();
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      if (tid == 0) issue(c + 1);
    }
    const bool ok = tc::mbar_wait_bounded(&sm.mbar[c & 1], (phase >> (c & 1)) & 1u, kWaitNs);
    phase ^= 1u << (c & 1);
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    // chunk c's u buffer is free: chunk c+2 comes in
    if (c + 2 < C) {
      stage_u2<NC>(sm.ub[c & 1], urow + (size_t)(c + 2) * Tc, tid);
      cp_async_commit();
    }
    // Horner in A^128 over this half's columns ih = HC half .. HC half + HC - 1
    const uint32_t tm = sm.tmem_base + (uint32_t)((c & 1) * tmem_cols<NC>());
    uint32_t zv[HC];
#pragma unroll
    for (int j = 0; j < HC; j += 8) tc::tmem_ld8(tm + lane_off + (uint32_t)(HC * half + j), zv + j);
    tc::tmem_wait_ld();  // one wait for all of this thread's columns
#pragma unroll
    for (int j = 0; j < HC; ++j) tc::tmem_regs_ready(zv[j]);
    // two interleaved Horner chains in A^256 (even and odd columns), then even * A^128 + odd
    float er = 0.f, ei = 0.f, orr = 0.f, oi = 0.f;
#pragma unroll
    for (int ih = 0; ih < HC; ih += 2) {
      const float ze = __uint_as_float(zv[ih]), zo = __uint_as_float(zv[ih + 1]);
      const float ner = fmaf(er, w256.x, fmaf(-ei, w256.y, ze));
      ei = fmaf(er, w256.y, ei * w256.x);
      er = ner;
      const float nor = fmaf(orr, w256.x, fmaf(-oi, w256.y, zo));
      oi = fmaf(orr, w256.y, oi * w256.x);
      orr = nor;
    }
    float ar = fmaf(er, w128.x, fmaf(-ei, w128.y, orr));
    float ai = fmaf(er, w128.y, fmaf(ei, w128.x, oi));
    // lower half: times A^(128 HC) (its columns come HC blocks earlier), plus the upper half
    if (half == 1) sm.part[lane] = make_float2(ar, ai);
    tc::fence_before_sync();
    __syncthreads();
    if (half == 0) {
      const float2 lo = cmul(make_float2(ar, ai), whalf);
      const float2 hi = sm.part[lane];
      ar = lo.x + hi.x;
      ai = lo.y + hi.y;
      // even lane holds the R_re row, odd lane the R_im row: sum = R_re + i R_im
      const float pr = __shfl_xor_sync(0xffffffffu, ar, 1);
      const float pi = __shfl_xor_sync(0xffffffffu, ai, 1);
      if (part == 0 && n < N) {
        const float2 sres = make_float2(ar - pi, ai + pr);
        s_ws[(((size_t)b * H + h) * C + c) * N + n] = cmul(sres, bn);
      }
    }
  }
  cp_async_wait<0>();
  if (failed && tid == 0) atomicAdd(&g_sp_tc_timeouts, 1u);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(sm.tmem_base, 2 * tmem_cols<NC>());
}

// ---------------------------------------------------------------- A9: correction
// grid (H, B), 256 threads; y[b, h, c T + t] += correction, chunks c >= c_begin.  Warps 0-3
// and 4-7 cover the 128 TMEM lanes twice and split each row's NC outputs in halves.  The
// accumulator is double-buffered in TMEM: chunk c+1's operand is built and its MMA issued
// before chunk c's epilogue runs; each thread's y values of the next chunk are loaded
// while the current chunk finishes.
template <int NC>
struct CorrSmem2 {
  uint8_t ahh[kTab];               // A: AH (fp16), 128 rows (th) x 128 K (2n + re/im)
  uint8_t qh[(NC / 8) * kSbo];     // B: Q (fp16), NC rows (tl) x 128 K
  float red[kThrS / 32];
  uint64_t mbar[2];
  uint32_t tmem_base;
};

template <typename T, int NC>
__global__ void __launch_bounds__(kThrS, 3) sp_corr_tc_kernel(T* __restrict__ y, const float* __restrict__ dt,
                                                               const float2* __restrict__ lam,
                                                               const float2* __restrict__ Cp,
                                                               const float2* __restrict__ x_ws, int H, int L, int N,
                                                               int c_begin) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  CorrSmem2<NC>& sm = *reinterpret_cast<CorrSmem2<NC>*>(smraw);
  constexpr int Tc = NC * kKS;
  constexpr int HC = NC / 2;               // outputs per thread per chunk
  constexpr int kGr = (NC / 8 + 3) / 4;    // Q row groups per thread (groups gq + 4 r < NC / 8)
  const int h = blockIdx.x, b = blockIdx.y;
  const int C = L / Tc;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int lane = tid & 127, half = tid >> 7;
  const float d = dt[h];

  if (warp == 0) tc::tmem_alloc(&sm.tmem_base, 2 * tmem_cols<NC>());
  if (tid == 0) {
    tc::mbar_init(&sm.mbar[0], 1);
    tc::mbar_init(&sm.mbar[1], 1);
    tc::fence_mbar_init();
  }
  // AH[th][2n] + i AH[th][2n+1] = A_n^(NC th): one exact power per 8 rows, then a chain in A^NC.
  for (int it = tid; it < 64 * 16; it += kThrS) {
    const int n = it & 63, g = it >> 6;
    float2 p = make_float2(0.f, 0.f), step = make_float2(0.f, 0.f);
    if (n < N) {
      const float2 lm = lam[(size_t)h * N + n];
      p = ssm_pow(d, lm.x, lm.y, (double)NC * 8.0 * g);
      step = ssm_pow(d, lm.x, lm.y, (double)NC);
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const uint32_t off = toff(8 * g + m, n >> 2) + (uint32_t)(n & 3) * 4u;
      *reinterpret_cast<uint32_t*>(sm.ahh + off) = Op16<__half>::bits(p.x) | (Op16<__half>::bits(p.y) << 16);
      p = cmul(p, step);
    }
  }
  // this thread's mode and Q row groups: n = tid % 64, tl groups gq + 4 r (gq = tid / 64)
  const int n = tid & 63, gq = tid >> 6;
  float2 a1 = make_float2(0.f, 0.f), cn = make_float2(0.f, 0.f), st[kGr];
#pragma unroll
  for (int r = 0; r < kGr; ++r) st[r] = make_float2(0.f, 0.f);
  if (n < N) {
    const float2 lm = lam[(size_t)h * N + n];
    a1 = ssm_pow(d, lm.x, lm.y, 1.0);
    cn = Cp[(size_t)h * N + n];
#pragma unroll
    for (int r = 0; r < kGr; ++r)
      if (gq + 4 * r < NC / 8) st[r] = ssm_pow(d, lm.x, lm.y, 8.0 * (gq + 4 * r) + 1.0);
  }
  const uint32_t idesc = tc::idesc_f16(128, NC, 0);
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  uint32_t phase = 0;  // bit b: parity of mbar[b]
  bool failed = false;
  const size_t rowoff = ((size_t)b * H + h) * (size_t)L;
  // Q of chunk c into shared memory; returns the inverse of its power-of-two scale
  auto build_q = [&](int c) -> float {
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
    mx = 0.f;
#pragma unroll
    for (int i = 0; i < kThrS / 32; ++i) mx = fmaxf(mx, sm.red[i]);
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
      const int tg = gq + 4 * r;
      if (tg >= NC / 8) continue;
      float2 p = cmul(w, st[r]);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const uint32_t off = toff(8 * tg + m, n >> 2) + (uint32_t)(n & 3) * 4u;
        *reinterpret_cast<uint32_t*>(sm.qh + off) = Op16<__half>::bits(p.x) | (Op16<__half>::bits(-p.y) << 16);
        p = cmul(p, a1);
      }
    }
    return inv;
  };
  auto issue = [&](int c) {
    const uint32_t ah = tc::smem_u32(sm.ahh);
    const uint32_t qh = tc::smem_u32(sm.qh);
    const uint32_t tm = sm.tmem_base + (uint32_t)((c & 1) * tmem_cols<NC>());
#pragma unroll
    for (int kk = 0; kk < kKS / 16; ++kk)
      tc::mma_f16(tm, tc::desc_kmajor(ah + kk * 2 * kLbo, kLbo, kSbo), tc::desc_kmajor(qh + kk * 2 * kLbo, kLbo, kSbo),
                  idesc, kk > 0 ? 1u : 0u);
    tc::mma_commit(&sm.mbar[c & 1]);
  };
  // this thread's outputs of chunk c: t = NC lane + HC half + j, j < HC
  auto yptr = [&](int c) {
    return reinterpret_cast<uint16_t*>(y) + rowoff + (size_t)c * Tc + (size_t)NC * lane + (size_t)HC * half;
  };
  if (c_begin < C) {
    float inv_cur = build_q(c_begin);
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0) issue(c_begin);
    uint4 yv[HC / 8];
    {
      const uint16_t* yp = yptr(c_begin);
#pragma unroll
      for (int i = 0; i < HC / 8; ++i) yv[i] = *reinterpret_cast<const uint4*>(yp + 8 * i);
    }
    for (int c = c_begin; c < C; ++c) {
      const bool ok = tc::mbar_wait_bounded(&sm.mbar[c & 1], (phase >> (c & 1)) & 1u, kWaitNs);
      phase ^= 1u << (c & 1);
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      tc::fence_after_sync();
      float inv_next = 1.f;
      if (c + 1 < C) {  // chunk c+1: operand (Q is free: MMA c has read it), then its MMA
        inv_next = build_q(c + 1);
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        if (tid == 0) issue(c + 1);
      }
      // epilogue of chunk c: y += correction (scale multiplied back out exactly)
      const uint32_t tm = sm.tmem_base + (uint32_t)((c & 1) * tmem_cols<NC>());
      uint16_t* yp = yptr(c);
#pragma unroll
      for (int j = 0; j < HC; j += 8) {
        uint32_t v[8];
        tc::tmem_ld8(tm + lane_off + (uint32_t)(HC * half + j), v);
        tc::tmem_wait_ld();
        uint32_t* wv = reinterpret_cast<uint32_t*>(&yv[j / 8]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          tc::tmem_regs_ready(v[2 * e]);
          tc::tmem_regs_ready(v[2 * e + 1]);
          const float lo = fmaf(__uint_as_float(v[2 * e]), inv_cur, Op16<T>::back(wv[e] & 0xffffu));
          const float hi = fmaf(__uint_as_float(v[2 * e + 1]), inv_cur, Op16<T>::back(wv[e] >> 16));
          wv[e] = Op16<T>::bits(lo) | (Op16<T>::bits(hi) << 16);
        }
      }
#pragma unroll
      for (int i = 0; i < HC / 8; ++i) *reinterpret_cast<uint4*>(yp + 8 * i) = yv[i];
      if (c + 1 < C) {
        const uint16_t* yn = yptr(c + 1);
#pragma unroll
        for (int i = 0; i < HC / 8; ++i) yv[i] = *reinterpret_cast<const uint4*>(yn + 8 * i);
      }
      inv_cur = inv_next;
      tc::fence_before_sync();
      __syncthreads();  // TMEM buffer c & 1 read before chunk c+2's MMA is issued into it
    }
  }
  if (failed && tid == 0) atomicAdd(&g_sp_tc_timeouts, 1u);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(sm.tmem_base, 2 * tmem_cols<NC>());
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
    const size_t smem = sizeof(StateSmem2<NC, Op16<T>::bf16 != 0>) + 1024;
    auto kern = sp_state_tc_kernel<T, NC>;
    cudaError_t e = smem_optin<sp_state_tc_kernel<T, NC>>(smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThrS, smem, st>>>((const T*)u, dt, (const float2*)lam, (const float2*)Bp, H, L, N, (float2*)s_ws);
  } else {
    const size_t smem = sizeof(CorrSmem2<NC>) + 1024;
    auto kern = sp_corr_tc_kernel<T, NC>;
    cudaError_t e = smem_optin<sp_corr_tc_kernel<T, NC>>(smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThrS, smem, st>>>((T*)y, dt, (const float2*)lam, (const float2*)Cp, (const float2*)x_ws, H, L, N,
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
