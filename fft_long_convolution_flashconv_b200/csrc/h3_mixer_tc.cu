// H3 mixer forward on the 5th-generation tensor cores (fp16 / bf16 I/O).
//
// H3 blog "The Solution, Part 1": O = Q (.) SSM_diag(SSM_shift(K) (.) V); per
// head the diagonal-SSM convolution of the kv outer product, contracted with
// q, is exactly the causal Toeplitz-weighted product
//   o_j[t] = sum_{s<=t} (f_h[t-s] + D_h [s==t]) (q_t . k~_s) v_s[j]
// (H3 summary appendix D.2 "H3 Complexity": matrix multiplications plus the
// SSM convolution).  Per 128-row tile of t and each 128-row tile of s <= t:
//   S  = Q_t K~_s^T            tcgen05.mma, M=128 N=128 K=64, fp32 in TMEM
//   P  = S (.) T_f(t-s)        4 warps: tcgen05.ld, scale, round, store to SMEM
//   O += P V_s                 tcgen05.mma, M=128 N=64 K=128, fp32 in TMEM
// The shift SSM k~[s,c] = sum_j Cshift[c,j] k[s-j,c] is applied while the K
// tile is staged.  Operands use the K-major no-swizzle layout of tc100.cuh.
// Every wait on MMA completion is bounded; on a timeout the CTA records it in
// a device counter, skips its remaining work and still frees its TMEM.
#include "kernels.cuh"
#include "tc100.cuh"

namespace fc {

static __device__ unsigned int g_mixer_timeouts;

namespace {
constexpr int kHD = 64;         // head_dim
constexpr int kT = 128;         // rows per t / s tile
constexpr int kThr = 128;       // 4 warps: one TMEM lane quarter each
constexpr int kMaxS = 8;        // shift taps
constexpr uint32_t kTmemCols = 256;  // S: cols [0,128), O: [128,192)
constexpr uint64_t kWaitNs = 2000000000ull;

struct MixSmem {
  uint8_t q[kT * kHD * 2];          // A of S-MMA  (rows t, K = i)
  uint8_t k[kT * kHD * 2];          // B of S-MMA  (rows s, K = i)
  uint8_t vt[kHD * kT * 2];         // B of O-MMA  (rows j, K = s)
  uint8_t p[kT * kT * 2];           // A of O-MMA  (rows t, K = s)
  uint16_t kraw[(kT + kMaxS) * kHD];  // raw k rows s0-S+1 .. s0+127 (row-major)
  float cs[kHD * kMaxS];
  float fs[2 * kT];
  uint64_t mbar;
  uint32_t tmem_base;
};
}  // namespace

template <typename T> struct Bits;
template <> struct Bits<__half> {
  static constexpr int bf16 = 0;
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ float tof(uint16_t x) { return __half2float(__ushort_as_half(x)); }
  static __device__ __forceinline__ uint16_t fromf(float x) { return __half_as_ushort(__float2half_rn(x)); }
};
template <> struct Bits<__nv_bfloat16> {
  static constexpr int bf16 = 1;
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ float tof(uint16_t x) { return __bfloat162float(__ushort_as_bfloat16(x)); }
  static __device__ __forceinline__ uint16_t fromf(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
};

template <typename T>
__global__ void __launch_bounds__(kThr, 1) h3_mixer_tc_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                              const T* __restrict__ v,
                                                              const float* __restrict__ Cshift,
                                                              const float* __restrict__ fdiag,
                                                              const float* __restrict__ D, T* __restrict__ o, int L,
                                                              int heads, int S) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  MixSmem& sm = *reinterpret_cast<MixSmem*>(smraw);
  const int tt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int dm = heads * kHD;
  const int t0 = tt * kT;
  const size_t base = (size_t)b * L * dm + (size_t)h * kHD;
  const uint16_t* qb = reinterpret_cast<const uint16_t*>(q) + base;
  const uint16_t* kb = reinterpret_cast<const uint16_t*>(k) + base;
  const uint16_t* vb = reinterpret_cast<const uint16_t*>(v) + base;

  if (warp == 0) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
  if (tid == 0) {
    tc::mbar_init(&sm.mbar, 1);
    tc::fence_mbar_init();
  }
  for (int idx = tid; idx < kHD * S; idx += kThr) sm.cs[idx] = Cshift[(size_t)(h * kHD) * S + idx];
  // Q tile: rows t0..t0+127, 8-element chunks
  for (int idx = tid; idx < kT * (kHD / 8); idx += kThr) {
    const int r = idx >> 3, c8 = (idx & 7) * 8;
    const int t = t0 + r;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (t < L) val = *reinterpret_cast<const uint4*>(qb + (size_t)t * dm + c8);
    *reinterpret_cast<uint4*>(sm.q + tc::kmaj_off(r, c8, kHD)) = val;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const uint32_t idS = tc::idesc_f16(128, 128, Bits<T>::bf16);
  const uint32_t idO = tc::idesc_f16(128, kHD, Bits<T>::bf16);
  const float dh = D[h];
  const float* fh = fdiag + (size_t)h * L;
  uint32_t phase = 0;
  bool failed = false;
  const int row = tid;  // TMEM lane / tile row owned by this thread

  for (int st = 0; st <= tt && !failed; ++st) {
    const int s0 = st * kT;
    // ---- stage raw k rows s0-(S-1) .. s0+127, then k~ (shift SSM) into the K-major tile
    const int nraw = kT + S - 1;
    for (int idx = tid; idx < nraw * (kHD / 8); idx += kThr) {
      const int r = idx >> 3, c8 = (idx & 7) * 8;
      const int s = s0 - (S - 1) + r;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (s >= 0 && s < L) val = *reinterpret_cast<const uint4*>(kb + (size_t)s * dm + c8);
      *reinterpret_cast<uint4*>(&sm.kraw[r * kHD + c8]) = val;
    }
    // V^T tile (rows j, K = s) and the Toeplitz weights for this (t, s) tile pair
    for (int idx = tid; idx < kT * (kHD / 8); idx += kThr) {
      const int r = idx >> 3, c8 = (idx & 7) * 8;
      const int s = s0 + r;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (s < L) val = *reinterpret_cast<const uint4*>(vb + (size_t)s * dm + c8);
      const uint16_t* e = reinterpret_cast<const uint16_t*>(&val);
#pragma unroll
      for (int i = 0; i < 8; ++i) *reinterpret_cast<uint16_t*>(sm.vt + tc::kmaj_off(c8 + i, r, kT)) = e[i];
    }
    for (int idx = tid; idx < 2 * kT - 1; idx += kThr) {
      const int d = idx - (kT - 1) + (t0 - s0);  // t - s
      float w = (d >= 0 && d < L) ? fh[d] : 0.f;
      if (d == 0) w += dh;
      sm.fs[idx] = w;
    }
    __syncthreads();
    for (int idx = tid; idx < kT * (kHD / 8); idx += kThr) {
      const int r = idx >> 3, c8 = (idx & 7) * 8;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      for (int j = 0; j < S; ++j) {
        const uint16_t* kr = &sm.kraw[(r + (S - 1) - j) * kHD + c8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(sm.cs[(c8 + i) * S + j], Bits<T>::tof(kr[i]), acc[i]);
      }
      uint4 pk;
      pk.x = Bits<T>::pack(acc[0], acc[1]);
      pk.y = Bits<T>::pack(acc[2], acc[3]);
      pk.z = Bits<T>::pack(acc[4], acc[5]);
      pk.w = Bits<T>::pack(acc[6], acc[7]);
      *reinterpret_cast<uint4*>(sm.k + tc::kmaj_off(r, c8, kHD)) = pk;
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // ---- S = Q K~^T
    if (tid == 0) {
      const uint32_t qa = tc::smem_u32(sm.q), ka = tc::smem_u32(sm.k);
#pragma unroll
      for (int kk = 0; kk < kHD / 16; ++kk)
        tc::mma_f16(tS, tc::desc_kmajor(qa + kk * 256, 128, (kHD / 8) * 128),
                    tc::desc_kmajor(ka + kk * 256, 128, (kHD / 8) * 128), idS, kk > 0 ? 1u : 0u);
      tc::mma_commit(&sm.mbar);
    }
    bool ok = tc::mbar_wait_bounded(&sm.mbar, phase, kWaitNs);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    // ---- P = S (.) Toeplitz weights, rounded to the operand type, into the K-major A tile
#pragma unroll 1
    for (int c = 0; c < kT; c += 16) {
      float sv[16];
      tc::tmem_ld16_wait(tS + lane_off + (uint32_t)c, sv);
      uint32_t pw[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a = sv[2 * i] * sm.fs[row - (c + 2 * i) + (kT - 1)];
        const float bb = sv[2 * i + 1] * sm.fs[row - (c + 2 * i + 1) + (kT - 1)];
        pw[i] = Bits<T>::pack(a, bb);
      }
      *reinterpret_cast<uint4*>(sm.p + tc::kmaj_off(row, c, kT)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
      *reinterpret_cast<uint4*>(sm.p + tc::kmaj_off(row, c + 8, kT)) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // ---- O += P V
    if (tid == 0) {
      const uint32_t pa = tc::smem_u32(sm.p), va = tc::smem_u32(sm.vt);
#pragma unroll
      for (int kk = 0; kk < kT / 16; ++kk)
        tc::mma_f16(tO, tc::desc_kmajor(pa + kk * 256, 128, (kT / 8) * 128),
                    tc::desc_kmajor(va + kk * 256, 128, (kT / 8) * 128), idO, (st > 0 || kk > 0) ? 1u : 0u);
      tc::mma_commit(&sm.mbar);
    }
    ok = tc::mbar_wait_bounded(&sm.mbar, phase, kWaitNs);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
  }
  if (!failed) {
    const int t = t0 + row;
#pragma unroll 1
    for (int c = 0; c < kHD; c += 16) {
      float ov[16];
      tc::tmem_ld16_wait(tO + lane_off + (uint32_t)c, ov);
      if (t < L) {
        uint4 lo, hi;
        lo.x = Bits<T>::pack(ov[0], ov[1]);
        lo.y = Bits<T>::pack(ov[2], ov[3]);
        lo.z = Bits<T>::pack(ov[4], ov[5]);
        lo.w = Bits<T>::pack(ov[6], ov[7]);
        hi.x = Bits<T>::pack(ov[8], ov[9]);
        hi.y = Bits<T>::pack(ov[10], ov[11]);
        hi.z = Bits<T>::pack(ov[12], ov[13]);
        hi.w = Bits<T>::pack(ov[14], ov[15]);
        uint16_t* orow = reinterpret_cast<uint16_t*>(o) + base + (size_t)t * dm + c;
        *reinterpret_cast<uint4*>(orow) = lo;
        *reinterpret_cast<uint4*>(orow + 8) = hi;
      }
    }
  } else if (tid == 0) {
    atomicAdd(&g_mixer_timeouts, 1u);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

template <typename T>
static cudaError_t mixer_tc_t(const void* q, const void* k, const void* v, const float* Cs, const float* f,
                              const float* D, void* o, int B, int L, int heads, int S, cudaStream_t st) {
  const size_t smem = sizeof(MixSmem) + 1024;
  auto kern = h3_mixer_tc_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((L + kT - 1) / kT, heads, B);
  kern<<<grid, kThr, smem, st>>>((const T*)q, (const T*)k, (const T*)v, Cs, f, D, (T*)o, L, heads, S);
  return cudaGetLastError();
}

cudaError_t launch_h3_mixer_tc(const void* q, const void* k, const void* v, const float* Cshift, const float* fdiag,
                               const float* D, void* o, int B, int L, int heads, int shift_len, int dtype,
                               cudaStream_t st) {
  if (shift_len > kMaxS) return cudaErrorInvalidValue;
  switch (dtype) {
    case 1: return mixer_tc_t<__half>(q, k, v, Cshift, fdiag, D, o, B, L, heads, shift_len, st);
    case 2: return mixer_tc_t<__nv_bfloat16>(q, k, v, Cshift, fdiag, D, o, B, L, heads, shift_len, st);
    default: return cudaErrorInvalidValue;
  }
}

unsigned int mixer_tc_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_mixer_timeouts, sizeof(v));
  return v;
}

}  // namespace fc
