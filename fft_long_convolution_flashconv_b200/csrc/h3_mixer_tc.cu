// H3 mixer forward on the 5th-generation tensor cores (fp16 / bf16 I/O).
//
// H3 blog "The Solution, Part 1": O = Q (.) SSM_diag(SSM_shift(K) (.) V); per
// head the diagonal-SSM convolution of the kv outer product, contracted with
// q, is exactly the causal Toeplitz-weighted product
//   o_j[t] = sum_{s<=t} (f_h[t-s] + D_h [s==t]) (q_t . k~_s) v_s[j]
// (H3 summary appendix D.2 "H3 Complexity": matrix multiplications plus the
// SSM convolution).  Per 128-row tile of t and each 64-row step of s <= t:
//   S  = Q_t K~_s^T            tcgen05.mma, M=128 N=64 K=64, fp32 in TMEM
//   P  = S (.) T_f(t-s)        4 warps: tcgen05.ld, scale, round, store to SMEM
//   O += P V_s                 tcgen05.mma, M=128 N=64 K=64, fp32 in TMEM
// The shift SSM k~[s,c] = sum_j Cshift[c,j] k[s-j,c] runs once, in a small
// elementwise kernel, into a workspace (rounded to the operand type).  Q and
// K~ tiles are K-major with padded core-matrix offsets (LBO 144 bytes) so that
// the row-wise 16-byte staging copies are free of bank conflicts; V is staged
// as it lies in memory and read by the tensor cores as an MN-major operand.
// 64-row s steps keep a CTA at 128 TMEM columns and ~55 KB of shared memory,
// so four CTAs share an SM and hide each other's copy and MMA latency; the
// next step's K~ is copied in as soon as the S-MMA has read the current one,
// V once the O-MMA has, and the next step's Toeplitz weights are loaded a step
// ahead.  CTAs are launched heaviest tile first (a t tile has t / 64 + 2 s
// steps), so the causal imbalance stays inside the first waves.
// Every wait on MMA completion is bounded; on a timeout the CTA records it in
// a device counter, skips its remaining work and still frees its TMEM.
#include "kernels.cuh"
#include "tc100.cuh"

namespace fc {

static __device__ unsigned int g_mixer_timeouts;

namespace {
constexpr int kHD = 64;         // head_dim
constexpr int kT = 128;         // rows per t tile
constexpr int kS = 64;          // rows per s step
constexpr int kThr = 128;       // 4 warps: one TMEM lane quarter each
constexpr int kMaxS = 8;        // shift taps
constexpr uint32_t kTmemCols = 128;  // S: cols [0,64), O: [64,128)
constexpr uint64_t kWaitNs = 2000000000ull;

constexpr uint32_t kQLbo = 144, kQSbo = (kHD / 8) * 144;   // Q, K~: 128 rows x 64 K, padded
constexpr uint32_t kVSbo = 144, kVLbo = (kHD / 8) * 144;   // V: MN-major, 64 N (j) x 64 K (s), padded
constexpr uint32_t kPLbo = 128, kPSbo = (kS / 8) * 128;    // P: 128 rows x 64 K
struct MixSmem {
  uint8_t q[(kT / 8) * kQSbo];      // A of S-MMA  (rows t, K = i)
  uint8_t k[(kS / 8) * kQSbo];      // B of S-MMA  (rows s, K = i)
  uint8_t v[(kS / 8) * kVLbo];      // B of O-MMA  (N = j, K = s), MN-major
  uint8_t p[kT * kS * 2];           // A of O-MMA  (rows t, K = s)
  float fs[2][2 * kT];              // Toeplitz weights of the current and the next s step
  uint64_t mbar;
  uint32_t tmem_base;
};

__device__ __forceinline__ uint32_t qoff(int r, int c8) {
  return (uint32_t)(r >> 3) * kQSbo + (uint32_t)(c8 >> 3) * kQLbo + (uint32_t)(r & 7) * 16;
}
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
// all but the most recently committed group of this thread's copies have landed
__device__ __forceinline__ void cp_async_wait_but_last() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ uint32_t voff(int s, int j8) {  // 8 consecutive j at time s
  return (uint32_t)(j8 >> 3) * kVSbo + (uint32_t)(s >> 3) * kVLbo + (uint32_t)(s & 7) * 16;
}
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

// k~ = shift SSM of k (B x L x dm, same type as k).  A thread owns 8 adjacent
// channels (their taps stay in registers) and kSeg consecutive time steps of
// one sequence: it loads those rows plus the S - 1 rows before them once, all
// up front, then forms the kSeg outputs from registers.  A warp covers 256
// adjacent channels of one time step (512-byte coalesced rows).
constexpr int kSeg = 16;
template <typename T, int S>
__global__ void __launch_bounds__(256) shift_ssm_kernel(const T* __restrict__ k, const float* __restrict__ Cshift,
                                                        T* __restrict__ kt, int B, int L, int dm) {
  const int ng = dm / 8;
  const int nseg = (L + kSeg - 1) / kSeg;
  const long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= (long long)B * nseg * ng) return;
  const int g = (int)(item % ng);
  const long long bs = item / ng;
  const int seg = (int)(bs % nseg), b = (int)(bs / nseg);
  const int c8 = g * 8;
  const uint16_t* kb = reinterpret_cast<const uint16_t*>(k) + (size_t)b * L * dm + c8;
  uint16_t* ob = reinterpret_cast<uint16_t*>(kt) + (size_t)b * L * dm + c8;
  const int t0 = seg * kSeg;
  // rows t0 - (S-1) .. t0 + kSeg - 1, all loads issued before any use (zero outside [0, L))
  uint4 rows[kSeg + S - 1];
#pragma unroll
  for (int i = 0; i < kSeg + S - 1; ++i) {
    const int t = t0 - (S - 1) + i;
    rows[i] = (t >= 0 && t < L) ? *reinterpret_cast<const uint4*>(kb + (size_t)t * dm) : make_uint4(0, 0, 0, 0);
  }
  float cs[S][8];
#pragma unroll
  for (int j = 0; j < S; ++j)
#pragma unroll
    for (int i = 0; i < 8; ++i) cs[j][i] = __ldg(Cshift + (size_t)(c8 + i) * S + j);
#pragma unroll
  for (int i = 0; i < kSeg; ++i) {
    const int t = t0 + i;
    if (t < L) {
      float acc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll
      for (int j = 0; j < S; ++j) {  // tap j reads row t - j
        const uint16_t* e = reinterpret_cast<const uint16_t*>(&rows[i + S - 1 - j]);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(cs[j][c], Bits<T>::tof(e[c]), acc[c]);
      }
      uint4 out;
      out.x = Bits<T>::pack(acc[0], acc[1]);
      out.y = Bits<T>::pack(acc[2], acc[3]);
      out.z = Bits<T>::pack(acc[4], acc[5]);
      out.w = Bits<T>::pack(acc[6], acc[7]);
      *reinterpret_cast<uint4*>(ob + (size_t)t * dm) = out;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThr, 4) h3_mixer_tc_kernel(const T* __restrict__ q, const T* __restrict__ kt,
                                                              const T* __restrict__ v,
                                                              const float* __restrict__ fdiag,
                                                              const float* __restrict__ D, T* __restrict__ o, int L,
                                                              int heads, int B) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  MixSmem& sm = *reinterpret_cast<MixSmem*>(smraw);
  // heaviest t tiles first: CTA i takes tile nt - 1 - i / (heads B), then (head, b)
  const int nt = (L + kT - 1) / kT;
  const int hb = heads * B;
  const int tt = nt - 1 - (int)(blockIdx.x / hb);
  const int rem = (int)(blockIdx.x % hb);
  const int h = rem % heads, b = rem / heads;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int dm = heads * kHD;
  const int t0 = tt * kT;
  const size_t base = (size_t)b * L * dm + (size_t)h * kHD;
  const uint16_t* qb = reinterpret_cast<const uint16_t*>(q) + base;
  const uint16_t* kb = reinterpret_cast<const uint16_t*>(kt) + base;
  const uint16_t* vb = reinterpret_cast<const uint16_t*>(v) + base;

  if (warp == 0) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
  if (tid == 0) {
    tc::mbar_init(&sm.mbar, 1);
    tc::fence_mbar_init();
  }
  // Q tile: rows t0..t0+127, 8-element chunks
  for (int idx = tid; idx < kT * (kHD / 8); idx += kThr) {
    const int r = idx >> 3, c8 = (idx & 7) * 8;
    const int t = t0 + r;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (t < L) val = *reinterpret_cast<const uint4*>(qb + (size_t)t * dm + c8);
    *reinterpret_cast<uint4*>(sm.q + qoff(r, c8)) = val;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tS = tmem, tO = tmem + kS;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const uint32_t idS = tc::idesc_f16(128, kS, Bits<T>::bf16);
  const uint32_t idO = tc::idesc_f16(128, kHD, Bits<T>::bf16, 0, 1);
  const float dh = D[h];
  const float* fh = fdiag + (size_t)h * L;
  uint32_t phase = 0;
  bool failed = false;
  const int row = tid;  // TMEM lane / tile row owned by this thread
  // K~ / V rows s0 .. s0+63 -> shared memory with cp.async (rows past L zeroed)
  auto issue_k = [&](int s0) {
    const uint32_t ka = tc::smem_u32(sm.k);
    for (int idx = tid; idx < kS * (kHD / 8); idx += kThr) {
      const int r = idx >> 3, c8 = (idx & 7) * 8;
      const int s = s0 + r;
      if (s < L)
        cp_async16(ka + qoff(r, c8), kb + (size_t)s * dm + c8);
      else
        *reinterpret_cast<uint4*>(sm.k + qoff(r, c8)) = make_uint4(0, 0, 0, 0);
    }
  };
  auto issue_v = [&](int s0) {
    const uint32_t va = tc::smem_u32(sm.v);
    for (int idx = tid; idx < kS * (kHD / 8); idx += kThr) {
      const int r = idx >> 3, c8 = (idx & 7) * 8;
      const int s = s0 + r;
      if (s < L)
        cp_async16(va + voff(r, c8), vb + (size_t)s * dm + c8);
      else
        *reinterpret_cast<uint4*>(sm.v + voff(r, c8)) = make_uint4(0, 0, 0, 0);
    }
  };
  // Toeplitz weights f[t - s] (+ D on the diagonal) of step (t0, s0) at idx = t - s + 63 - (t0 - s0)
  // (t - s in [t0 - s0 - 63, t0 - s0 + 127]): this thread's two entries, loaded a step ahead
  auto weights = [&](int s0, float& w0, float& w1) {
    const int d0 = tid - (kS - 1) + (t0 - s0), d1 = d0 + kThr;
    w0 = (d0 >= 0 && d0 < L) ? fh[d0] : 0.f;
    w1 = (tid + kThr < kT + kS - 1 && d1 >= 0 && d1 < L) ? fh[d1] : 0.f;
    if (d0 == 0) w0 += dh;
    if (d1 == 0) w1 += dh;
  };
  {
    float w0, w1;
    weights(0, w0, w1);
    sm.fs[0][tid] = w0;
    sm.fs[0][tid + kThr] = w1;
  }
  issue_k(0);
  cp_async_commit();
  issue_v(0);
  cp_async_commit();

  const int nsteps = min((t0 + kT + kS - 1) / kS, (L + kS - 1) / kS);  // s0 = kS st <= t0 + 127, s0 < L
  for (int st = 0; st < nsteps && !failed; ++st) {
    const int s0 = st * kS;
    // ---- this step's K~ has been copied (issued during the previous step; its V, committed
    // after it, may still be in flight and is waited for before the O-MMA)
    cp_async_wait_but_last();
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // ---- S = Q K~^T
    if (tid == 0) {
      const uint32_t qa = tc::smem_u32(sm.q), ka = tc::smem_u32(sm.k);
#pragma unroll
      for (int kk = 0; kk < kHD / 16; ++kk)
        tc::mma_f16(tS, tc::desc_kmajor(qa + kk * 2 * kQLbo, kQLbo, kQSbo),
                    tc::desc_kmajor(ka + kk * 2 * kQLbo, kQLbo, kQSbo), idS, kk > 0 ? 1u : 0u);
      tc::mma_commit(&sm.mbar);
    }
    bool ok = tc::mbar_wait_bounded(&sm.mbar, phase, kWaitNs);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    // ---- the S-MMA has read K~: the next step's K~ can come in now, and its weights
    const bool more = st + 1 < nsteps;
    if (more) issue_k(s0 + kS);
    cp_async_commit();
    float wn0 = 0.f, wn1 = 0.f;
    if (more) weights(s0 + kS, wn0, wn1);
    const float* fsc = sm.fs[st & 1];
    // ---- P = S (.) Toeplitz weights, rounded to the operand type, into the K-major A tile
#pragma unroll
    for (int c = 0; c < kS; c += 32) {
      float sv2[32];
      tc::tmem_ld16x2_wait(tS + lane_off + (uint32_t)c, tS + lane_off + (uint32_t)c + 16u, sv2, sv2 + 16);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
      const float* sv = sv2 + 16 * hh;
      const int c16 = c + 16 * hh;
      uint32_t pw[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a = sv[2 * i] * fsc[row - (c16 + 2 * i) + (kS - 1)];
        const float bb = sv[2 * i + 1] * fsc[row - (c16 + 2 * i + 1) + (kS - 1)];
        pw[i] = Bits<T>::pack(a, bb);
      }
      *reinterpret_cast<uint4*>(sm.p + (uint32_t)(row >> 3) * kPSbo + (uint32_t)(c16 >> 3) * kPLbo + (row & 7) * 16) =
          make_uint4(pw[0], pw[1], pw[2], pw[3]);
      *reinterpret_cast<uint4*>(sm.p + (uint32_t)(row >> 3) * kPSbo + (uint32_t)((c16 + 8) >> 3) * kPLbo +
                                (row & 7) * 16) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
      }
    }
    if (more) {  // the other buffer was last read by the P pass of step st - 1
      sm.fs[(st + 1) & 1][tid] = wn0;
      sm.fs[(st + 1) & 1][tid + kThr] = wn1;
    }
    cp_async_wait_but_last();  // this step's V (only the next step's K~ may still be in flight)
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // ---- O += P V
    if (tid == 0) {
      const uint32_t pa = tc::smem_u32(sm.p), va = tc::smem_u32(sm.v);
#pragma unroll
      for (int kk = 0; kk < kS / 16; ++kk)
        tc::mma_f16(tO, tc::desc_kmajor(pa + kk * 2 * kPLbo, kPLbo, kPSbo),
                    tc::desc_kmajor(va + kk * 2 * kVLbo, kVLbo, kVSbo), idO, (st > 0 || kk > 0) ? 1u : 0u);
      tc::mma_commit(&sm.mbar);
    }
    ok = tc::mbar_wait_bounded(&sm.mbar, phase, kWaitNs);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    // ---- the O-MMA has read V: the next step's V
    if (more) issue_v(s0 + kS);
    cp_async_commit();
  }
  cp_async_wait_all();
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
                              const float* D, void* o, void* kt, int B, int L, int heads, int S, cudaStream_t st) {
  const int dm = heads * kHD;
  const long long items = (long long)B * ((L + kSeg - 1) / kSeg) * (dm / 8);
  const unsigned sg = (unsigned)((items + 255) / 256);
  const T* kk = (const T*)k;
  T* ko = (T*)kt;
  switch (S) {
    case 1: shift_ssm_kernel<T, 1><<<sg, 256, 0, st>>>(kk, Cs, ko, B, L, dm); break;
    case 2: shift_ssm_kernel<T, 2><<<sg, 256, 0, st>>>(kk, Cs, ko, B, L, dm); break;
    case 3: shift_ssm_kernel<T, 3><<<sg, 256, 0, st>>>(kk, Cs, ko, B, L, dm); break;
    case 4: shift_ssm_kernel<T, 4><<<sg, 256, 0, st>>>(kk, Cs, ko, B, L, dm); break;
    case 5: shift_ssm_kernel<T, 5><<<sg, 256, 0, st>>>(kk, Cs, ko, B, L, dm); break;
    case 6: shift_ssm_kernel<T, 6><<<sg, 256, 0, st>>>(kk, Cs, ko, B, L, dm); break;
    case 7: shift_ssm_kernel<T, 7><<<sg, 256, 0, st>>>(kk, Cs, ko, B, L, dm); break;
    case 8: shift_ssm_kernel<T, 8><<<sg, 256, 0, st>>>(kk, Cs, ko, B, L, dm); break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(MixSmem) + 1024;
  auto kern = h3_mixer_tc_kernel<T>;
  e = smem_optin<h3_mixer_tc_kernel<T>>(smem);
  if (e != cudaSuccess) return e;
  const long long ctas = (long long)((L + kT - 1) / kT) * heads * B;
  if (ctas > 0x7fffffffLL) return cudaErrorInvalidValue;
  kern<<<(unsigned)ctas, kThr, smem, st>>>((const T*)q, (const T*)kt, (const T*)v, f, D, (T*)o, L, heads, B);
  return cudaGetLastError();
}

cudaError_t launch_h3_mixer_tc(const void* q, const void* k, const void* v, const float* Cshift, const float* fdiag,
                               const float* D, void* o, void* ktilde, int B, int L, int heads, int shift_len,
                               int dtype, cudaStream_t st) {
  if (shift_len > kMaxS) return cudaErrorInvalidValue;
  switch (dtype) {
    case 1: return mixer_tc_t<__half>(q, k, v, Cshift, fdiag, D, o, ktilde, B, L, heads, shift_len, st);
    case 2: return mixer_tc_t<__nv_bfloat16>(q, k, v, Cshift, fdiag, D, o, ktilde, B, L, heads, shift_len, st);
    default: return cudaErrorInvalidValue;
  }
}

unsigned int mixer_tc_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_mixer_timeouts, sizeof(v));
  return v;
}

}  // namespace fc
