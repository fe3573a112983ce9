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
#include <algorithm>

#include "kernels.cuh"
#include "tc100.cuh"
#include "tmap.cuh"

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

// ---------------------------------------------------------------------------
// Warp-specialised persistent form (L a multiple of 8).  One CTA per SM walks
// a list of (t tile, head, b) items, heaviest tiles first and dealt to the
// CTAs in snake order so the causal work evens out.  Per item, 128-row s
// steps s0 = 0, 128, ..., t0; the roles hand over through mbarriers:
//   warp 0      copies K~ and V tiles of each step (two 5-d tensor-map copies
//               straight into the operand layouts) into a 4-stage ring;
//   warp 1      issues S = Q K~^T (M=128 N=128 K=64, Q from tensor memory)
//               into one of two S buffers, then O += P V (M=128 N=64 K=128, P
//               from tensor memory) of the previous step, so the weighting of
//               step g overlaps the O-MMA of step g - 1;
//   warps 4-7 / 8-11  weight the S tiles of even / odd steps: P = S (.) f[t-s]
//               (+ D on the diagonal), rounded to the operand type and
//               written back over the same tensor-memory columns;
//   warps 12-15 put each item's Q tile into tensor memory and write its O.
// Tensor memory: S/P [0,128) and [128,256), O [256,320) and [320,384),
// Q [384,416) and [416,448).  Every wait is bounded; a role that gives up
// raises a shared flag the others see in their own waits, and the CTA lets
// its copies and MMAs in flight finish before freeing tensor memory.
namespace {
constexpr int kWsS = 128;                   // rows per s step
constexpr int kWsStages = 4;                // K~ / V ring depth
constexpr int kWsThr = 512;
constexpr uint32_t kWsTile = 128 * kHD * 2;  // one 128 x 64 16-bit tile
constexpr int kWinStride = 264;             // floats between the four shifted window copies
constexpr uint32_t kColO = 256, kColQ = 384, kWsCols = 512;

struct WsSmem {
  uint8_t k[kWsStages][kWsTile];
  uint8_t v[kWsStages][kWsTile];
  float win[2][2][4 * kWinStride];          // [weighting group][buffer]: window copies shifted by 0..3
  uint64_t k_full[kWsStages], v_full[kWsStages], kv_empty[kWsStages];
  uint64_t s_full[2], p_full[2], q_full[2], o_full[2], o_empty[2], drain;
  uint32_t tmem_base;
  int abort;
};

// The items of one CTA in order, and the 128-row s steps of each.
struct WsIter {
  int G, cta, nitems, nt, hb, heads;
  int r, n, k, j, nst, g;  // round, ordinal of the item in this CTA, item, step, steps of the item, global step
  int tt, h, b;
  __device__ void set_item() {
    k = r * G + ((r & 1) ? (G - 1 - cta) : cta);
    if (k < nitems) {
      tt = nt - 1 - k / hb;
      const int rem = k - (k / hb) * hb;
      h = rem % heads;
      b = rem / heads;
      nst = tt + 1;
    }
  }
  __device__ void init(int G_, int cta_, int nitems_, int nt_, int heads_, int B) {
    G = G_, cta = cta_, nitems = nitems_, nt = nt_, heads = heads_, hb = heads_ * B;
    r = 0, n = 0, j = 0, g = 0;
    set_item();
  }
  __device__ bool valid() const { return k < nitems; }
  __device__ void next() {
    ++g;
    if (++j == nst) {
      j = 0;
      ++n;
      ++r;
      set_item();
    }
  }
  __device__ void next_item() {
    g += nst - j;
    j = 0;
    ++n;
    ++r;
    set_item();
  }
};

__device__ __forceinline__ void nbar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Named barrier over `count` threads that also ORs a predicate across them.
__device__ __forceinline__ bool nbar_or(int id, int count, bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(out)
      : "r"((uint32_t)v), "r"(id), "r"(count)
      : "memory");
  return out != 0;
}
}  // namespace

template <typename T>
__global__ void __launch_bounds__(kWsThr, 1)
    h3_mixer_ws_kernel(const T* __restrict__ q, const float* __restrict__ fdiag, const float* __restrict__ D,
                       T* __restrict__ o, int L, int heads, int B, const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  WsSmem& sm = *reinterpret_cast<WsSmem*>(smraw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int dm = heads * kHD;
  const int nt = (L + kT - 1) / kT;
  const int nitems = nt * heads * B;
  volatile int* abort_flag = &sm.abort;

  if (tid == 0) {
    for (int i = 0; i < kWsStages; ++i) {
      tc::mbar_init(&sm.k_full[i], 1);
      tc::mbar_init(&sm.v_full[i], 1);
      tc::mbar_init(&sm.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sm.s_full[i], 1);
      tc::mbar_init(&sm.p_full[i], 128);
      tc::mbar_init(&sm.q_full[i], 128);
      tc::mbar_init(&sm.o_full[i], 1);
      tc::mbar_init(&sm.o_empty[i], 128);
    }
    tc::mbar_init(&sm.drain, 1);
    sm.abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(&sm.tmem_base, kWsCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem_base;

  // bounded wait that also gives up as soon as another role has given up
  auto wwait = [&](uint64_t* mb, uint32_t parity) -> bool {
    if (tc::mbar_try_wait(mb, parity)) return true;
    const uint64_t t0 = tc::globaltimer_ns();
    while (!tc::mbar_try_wait(mb, parity)) {
      if (*abort_flag) return false;
      if (tc::globaltimer_ns() - t0 > kWaitNs) {
        *abort_flag = 1;
        return false;
      }
    }
    return true;
  };
  WsIter it;
  it.init((int)gridDim.x, (int)blockIdx.x, nitems, nt, heads, B);

  if (warp == 0) {
    // ---------------- K~ / V copies
    for (; it.valid(); it.next()) {
      const int stg = it.g % kWsStages;
      const uint32_t use = (uint32_t)(it.g / kWsStages);
      bool ok = true;
      if (lane == 0 && use > 0) ok = wwait(&sm.kv_empty[stg], (use - 1) & 1u);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane == 0) {
        const int r8 = (it.j * kWsS) / 8;
        tc::mbar_expect_tx(&sm.k_full[stg], kWsTile);
        tc::tma_load_5d(tc::smem_u32(sm.k[stg]), &kmap, 0, 0, 8 * it.h, r8, it.b, &sm.k_full[stg]);
        tc::mbar_expect_tx(&sm.v_full[stg], kWsTile);
        tc::tma_load_5d(tc::smem_u32(sm.v[stg]), &vmap, 0, 0, 8 * it.h, r8, it.b, &sm.v_full[stg]);
      }
    }
    // copies still in flight (only after a give-up) land before the CTA leaves
    if (lane == 0) {
      for (int g = it.g - kWsStages; g < it.g; ++g) {
        if (g < 0) continue;
        const int stg = g % kWsStages;
        const uint32_t par = (uint32_t)(g / kWsStages) & 1u;
        (void)tc::mbar_wait_bounded(&sm.k_full[stg], par, kWaitNs);
        (void)tc::mbar_wait_bounded(&sm.v_full[stg], par, kWaitNs);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issue (lane 0)
    const uint32_t idS = tc::idesc_f16(128, kWsS, Bits<T>::bf16);
    const uint32_t idO = tc::idesc_f16(128, kHD, Bits<T>::bf16, 0, 1);
    int pg = -1, pstg = 0, pn = 0, pj = 0, plast = 0;  // the step whose O-MMA is still to be issued
    auto issue_o = [&]() -> bool {
      bool ok = true;
      if (lane == 0) {
        if (pj == 0 && pn >= 2) ok = wwait(&sm.o_empty[pn & 1], (uint32_t)((pn - 2) >> 1) & 1u);
        if (ok) ok = wwait(&sm.p_full[pg & 1], (uint32_t)(pg >> 1) & 1u);
        if (ok) ok = wwait(&sm.v_full[pstg], (uint32_t)(pg / kWsStages) & 1u);
        if (ok) {
          tc::fence_after_sync();
          const uint32_t d = tmem + kColO + 64u * (uint32_t)(pn & 1), a = tmem + 128u * (uint32_t)(pg & 1);
          const uint32_t vb = tc::smem_u32(sm.v[pstg]);
#pragma unroll
          for (int kk = 0; kk < kWsS / 16; ++kk)
            tc::mma_f16_tmem_a(d, a + 8u * kk, tc::desc_kmajor(vb + kk * 2048, 1024, 128), idO,
                               (pj > 0 || kk > 0) ? 1u : 0u);
          tc::mma_commit(&sm.kv_empty[pstg]);
          if (plast) tc::mma_commit(&sm.o_full[pn & 1]);
        }
      }
      return __shfl_sync(0xffffffffu, ok, 0);
    };
    bool ok = true;
    for (; it.valid(); it.next()) {
      const int stg = it.g % kWsStages;
      if (lane == 0) {
        if (it.j == 0) ok = wwait(&sm.q_full[it.n & 1], (uint32_t)(it.n >> 1) & 1u);
        if (ok) ok = wwait(&sm.k_full[stg], (uint32_t)(it.g / kWsStages) & 1u);
        if (ok) {
          tc::fence_after_sync();
          const uint32_t d = tmem + 128u * (uint32_t)(it.g & 1), a = tmem + kColQ + 32u * (uint32_t)(it.n & 1);
          const uint32_t kb = tc::smem_u32(sm.k[stg]);
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk)
            tc::mma_f16_tmem_a(d, a + 8u * kk, tc::desc_kmajor(kb + kk * 256, 128, 1024), idS, kk > 0 ? 1u : 0u);
          tc::mma_commit(&sm.s_full[it.g & 1]);
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (pg >= 0 && !issue_o()) {
        ok = false;
        break;
      }
      pg = it.g, pstg = stg, pn = it.n, pj = it.j, plast = (it.j + 1 == it.nst);
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok && pg >= 0) (void)issue_o();
    if (lane == 0) {  // everything issued has completed before tensor memory is freed
      tc::mma_commit(&sm.drain);
      (void)tc::mbar_wait_bounded(&sm.drain, 0, kWaitNs);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 12) {
    // ---------------- weighting: P = S (.) f[t - s], even steps on warps 4-7, odd on 8-11
    const int wg = (warp >> 2) - 1;
    const int row = 32 * (warp & 3) + lane;  // TMEM lane = row of the t tile
    const int wt = tid & 127;                // thread of the group
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    if (wg == 1) it.next();
    WsIter nx = it;
    nx.next();
    nx.next();
    // window of a step: W[x] = f[t0 - s0 - 127 + x] (+ D at 0, 0 below 0), x < 255;
    // this thread loads x = wt and wt + 128
    auto load_win = [&](const WsIter& s, float& w0, float& w1) {
      const float* fh = fdiag + (size_t)s.h * L;
      const float dh = D[s.h];
      const int d0 = (s.tt - s.j) * kT - 127 + wt, d1 = d0 + 128;
      w0 = (d0 >= 0 && d0 < L) ? fh[d0] + (d0 == 0 ? dh : 0.f) : 0.f;
      w1 = (wt < 127 && d1 >= 0 && d1 < L) ? fh[d1] + (d1 == 0 ? dh : 0.f) : 0.f;
    };
    float w0 = 0.f, w1 = 0.f;
    if (it.valid()) load_win(it, w0, w1);
    int buf = 0;
    while (it.valid()) {
      // copy a of the window holds W[x + a] at x, so every 4-column group reads one aligned float4
      float* wb = sm.win[wg][buf];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        if (wt - a >= 0) wb[a * kWinStride + wt - a] = w0;
        wb[a * kWinStride + wt + 128 - a] = w1;
      }
      nbar_sync(1 + wg, 128);
      if (nx.valid()) load_win(nx, w0, w1);
      const bool ok = wwait(&sm.s_full[it.g & 1], (uint32_t)(it.g >> 1) & 1u);
      if (nbar_or(1 + wg, 128, !ok)) break;
      tc::fence_after_sync();
      const uint32_t sb = tmem + 128u * (uint32_t)(it.g & 1) + lane_off;
      // weights of columns c .. c+3 (c = 0 mod 4): W[r-c+124 .. r-c+127] = copy (r & 3) at (r - (r & 3)) - c + 124
      const float* wq = wb + (row & 3) * kWinStride + (row - (row & 3)) + 124;
#pragma unroll
      for (int cb = 0; cb < kWsS / 32; ++cb) {
        float s[32];
        tc::tmem_ld16x2_wait(sb + (uint32_t)(32 * cb), sb + (uint32_t)(32 * cb + 16), s, s + 16);
        uint32_t pk[16];
#pragma unroll
        for (int g4 = 0; g4 < 8; ++g4) {
          const float4 w4 = *reinterpret_cast<const float4*>(wq - (32 * cb + 4 * g4));
          pk[2 * g4] = Bits<T>::pack(s[4 * g4] * w4.w, s[4 * g4 + 1] * w4.z);
          pk[2 * g4 + 1] = Bits<T>::pack(s[4 * g4 + 2] * w4.y, s[4 * g4 + 3] * w4.x);
        }
        // P columns [16 cb, 16 cb + 16) lie in S columns this thread has already read
        tc::tmem_st8(sb + (uint32_t)(16 * cb), pk);
        tc::tmem_st8(sb + (uint32_t)(16 * cb + 8), pk + 8);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&sm.p_full[it.g & 1]);
      buf ^= 1;
      it = nx;
      nx.next();
      nx.next();
    }
  } else if (warp >= 12) {
    // ---------------- Q into tensor memory, O out
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint16_t* qb = reinterpret_cast<const uint16_t*>(q);
    uint16_t* ob = reinterpret_cast<uint16_t*>(o);
    auto load_q = [&](const WsIter& s) {
      const int t = s.tt * kT + row;
      uint32_t w[32];
      if (t < L) {
        const uint4* src = reinterpret_cast<const uint4*>(qb + ((size_t)s.b * L + t) * dm + (size_t)s.h * kHD);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 x = src[i];
          w[4 * i] = x.x, w[4 * i + 1] = x.y, w[4 * i + 2] = x.z, w[4 * i + 3] = x.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = 0u;
      }
      const uint32_t qa = tmem + kColQ + 32u * (uint32_t)(s.n & 1) + lane_off;
#pragma unroll
      for (int i = 0; i < 4; ++i) tc::tmem_st8(qa + 8u * i, w + 8 * i);
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&sm.q_full[s.n & 1]);
    };
    if (it.valid()) load_q(it);
    while (it.valid()) {
      WsIter nx = it;
      nx.next_item();
      if (nx.valid()) load_q(nx);  // its buffer was last read by item n - 1, already written out
      const bool ok = wwait(&sm.o_full[it.n & 1], (uint32_t)(it.n >> 1) & 1u);
      if (nbar_or(3, 128, !ok)) break;
      tc::fence_after_sync();
      const uint32_t oa = tmem + kColO + 64u * (uint32_t)(it.n & 1) + lane_off;
      float ov[64];
      tc::tmem_ld16x2_wait(oa, oa + 16u, ov, ov + 16);
      tc::tmem_ld16x2_wait(oa + 32u, oa + 48u, ov + 32, ov + 48);
      tc::fence_before_sync();
      tc::mbar_arrive(&sm.o_empty[it.n & 1]);
      const int t = it.tt * kT + row;
      if (t < L) {
        uint4* dst = reinterpret_cast<uint4*>(ob + ((size_t)it.b * L + t) * dm + (size_t)it.h * kHD);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_uint4(Bits<T>::pack(ov[8 * i], ov[8 * i + 1]), Bits<T>::pack(ov[8 * i + 2], ov[8 * i + 3]),
                              Bits<T>::pack(ov[8 * i + 4], ov[8 * i + 5]), Bits<T>::pack(ov[8 * i + 6], ov[8 * i + 7]));
      }
      it = nx;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (tid == 0 && sm.abort) atomicAdd(&g_mixer_timeouts, 1u);
  if (warp == 1) tc::tmem_dealloc(tmem, kWsCols);
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
  if (L % 8 == 0) {
    // warp-specialised form: K~ and V tiles through tensor maps (rows in groups of 8)
    CUtensorMap kmap, vmap;
    const cuuint64_t dims[5] = {8, 8, (cuuint64_t)(dm / 8), (cuuint64_t)(L / 8), (cuuint64_t)B};
    const cuuint64_t strides[4] = {(cuuint64_t)dm * 2, 16, (cuuint64_t)dm * 16, (cuuint64_t)L * dm * 2};
    const cuuint32_t box[5] = {8, 8, 8, 16, 1};
    if ((e = encode_map_5d_u16(&kmap, kt, dims, strides, box)) != cudaSuccess) return e;
    if ((e = encode_map_5d_u16(&vmap, v, dims, strides, box)) != cudaSuccess) return e;
    const size_t wsmem = sizeof(WsSmem);
    if ((e = smem_optin<h3_mixer_ws_kernel<T>>(wsmem)) != cudaSuccess) return e;
    const long long items = (long long)((L + kT - 1) / kT) * heads * B;
    if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
    const int grid = (int)std::min<long long>(items, (long long)num_sms());
    h3_mixer_ws_kernel<T><<<grid, kWsThr, wsmem, st>>>((const T*)q, f, D, (T*)o, L, heads, B, kmap, vmap);
    return cudaGetLastError();
  }
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
