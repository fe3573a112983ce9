// H3 mixer forward on the 5th-generation tensor cores (fp16 / bf16 I/O).
//
// H3 blog "The Solution, Part 1": O = Q (.) SSM_diag(SSM_shift(K) (.) V); per
// head the diagonal-SSM convolution of the kv outer product, contracted with
// q, is exactly the causal Toeplitz-weighted product
//   o_j[t] = sum_{s<=t} (f_h[t-s] + D_h [s==t]) (q_t . k~_s) v_s[j]
// (H3 summary appendix D.2 "H3 Complexity": matrix multiplications plus the
// SSM convolution).  Per 128-row tile of t and each 128-row step of s <= t:
//   S  = Q_t K~_s^T            tcgen05.mma, M=128 N=128 K=64, fp32 in TMEM
//   P  = S (.) T_f(t-s)        tcgen05.ld, scale, round, tcgen05.st over S
//   O += P V_s                 tcgen05.mma, M=128 N=64 K=128, P from TMEM
// The shift SSM k~[s,c] = sum_j Cshift[c,j] k[s-j,c] runs once, in a small
// elementwise kernel, into a workspace (rounded to the operand type).  The
// mixer itself is one persistent warp-specialised kernel (described below);
// Q, K~ and V tiles arrive by tensor-map copies with the 128-byte swizzle,
// which the tensor cores read directly.
#include <algorithm>

#include "kernels.cuh"
#include "tc100.cuh"
#include "tmap.cuh"

namespace fc {

static __device__ unsigned int g_mixer_timeouts;

namespace {
constexpr int kHD = 64;         // head_dim
constexpr int kT = 128;         // rows per t tile
constexpr int kMaxS = 8;        // shift taps
constexpr uint64_t kWaitNs = 2000000000ull;

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
// one sequence, read in batches of kBatch rows through a register window that
// carries the last S - 1 rows over, so each input row is loaded once per
// segment (plus S - 1 halo rows).  Consecutive threads take consecutive
// channel groups of the same rows: every load and store is a coalesced 16-byte
// access.  The kernel runs as a programmatic dependent of the filter
// generator, whose output it does not read: it lets the mixer launch early,
// does its own work while the generator runs, and waits for the generator only
// before it exits, so its completion implies the generator's.
constexpr int kSeg = 32, kBatch = 16;
template <typename T, int S>
__global__ void __launch_bounds__(128, 3) shift_ssm_kernel(const T* __restrict__ k, const float* __restrict__ Cshift,
                                                        T* __restrict__ kt, int B, int L, int dm) {
  const int ng = dm / 8;
  const int nseg = (L + kSeg - 1) / kSeg;
  asm volatile("griddepcontrol.launch_dependents;");
  const long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= (long long)B * nseg * ng) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }
  const int g = (int)(item % ng);
  const long long bs = item / ng;
  const int seg = (int)(bs % nseg), b = (int)(bs / nseg);
  const int c8 = g * 8;
  const uint16_t* kb = reinterpret_cast<const uint16_t*>(k) + (size_t)b * L * dm + c8;
  uint16_t* ob = reinterpret_cast<uint16_t*>(kt) + (size_t)b * L * dm + c8;
  const int t0 = seg * kSeg;
  float cs[S][8];
#pragma unroll
  for (int j = 0; j < S; ++j)
#pragma unroll
    for (int i = 0; i < 8; ++i) cs[j][i] = __ldg(Cshift + (size_t)(c8 + i) * S + j);
  // w[S - 1 + i] = row t0 + i0 + i of the batch, w[0 .. S - 2] the S - 1 rows before it (zero before 0)
  uint4 w[S - 1 + kBatch];
#pragma unroll
  for (int i = 0; i < S - 1; ++i) {
    const int t = t0 - (S - 1) + i;
    w[i] = t >= 0 ? *reinterpret_cast<const uint4*>(kb + (size_t)t * dm) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll 1
  for (int i0 = 0; i0 < kSeg && t0 + i0 < L; i0 += kBatch) {
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int t = t0 + i0 + i;
      w[S - 1 + i] = t < L ? *reinterpret_cast<const uint4*>(kb + (size_t)t * dm) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int t = t0 + i0 + i;
      float acc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll
      for (int j = 0; j < S; ++j) {  // tap j reads row t - j
        const uint16_t* e = reinterpret_cast<const uint16_t*>(&w[S - 1 + i - j]);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(cs[j][c], Bits<T>::tof(e[c]), acc[c]);
      }
      if (t < L) {
        uint4 out;
        out.x = Bits<T>::pack(acc[0], acc[1]);
        out.y = Bits<T>::pack(acc[2], acc[3]);
        out.z = Bits<T>::pack(acc[4], acc[5]);
        out.w = Bits<T>::pack(acc[6], acc[7]);
        *reinterpret_cast<uint4*>(ob + (size_t)t * dm) = out;
      }
    }
#pragma unroll
    for (int i = 0; i < S - 1; ++i) w[i] = w[kBatch + i];
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Warp-specialised persistent form.  One CTA per SM walks
// a list of (t tile, head, b) items, heaviest tiles first and dealt to the
// CTAs in snake order so the causal work evens out.  Per item, 128-row s
// steps s0 = 0, 128, ..., t0; the roles hand over through mbarriers:
//   warp 0      copies each item's Q tile and each step's K~ and V tiles
//               (5-d tensor-map copies straight into the operand layouts;
//               K~ / V through a 4-stage ring);
//   warp 1      issues S = Q K~^T (M=128 N=128 K=64) into one of three S
//               buffers in tensor memory;
//   warp 2      issues O += P V (M=128 N=64 K=128, P read from the S buffer
//               it overwrote), so S- and O-MMAs of different steps are
//               issued from two threads at once;
//   warps 4-7 / 8-11  weight the S tiles of even / odd steps: P = S (.) f[t-s]
//               (+ D on the diagonal), rounded to the operand type and
//               written back over the same tensor-memory columns;
//   warps 12-15 write each item's O.
// Tensor memory: S/P [0,128), [128,256), [256,384); O [384,448), [448,512).
// An S buffer is reused only after the O-MMA that read its P has completed.
// Every wait is bounded; a role that gives up raises a shared flag the
// others see in their own waits, and the CTA lets its copies and MMAs in
// flight finish before freeing tensor memory.
namespace {
constexpr int kWsS = 128;                   // rows per s step
constexpr int kWsStages = 4;                // K~ / V ring depth
constexpr int kWsThr = 512;
constexpr int kWsSBuf = 3;                  // S / P buffers
constexpr uint32_t kWsTile = 128 * kHD * 2;  // one 128 x 64 16-bit tile
constexpr int kWinStride = 264;             // floats between the four shifted window copies
constexpr uint32_t kColO = 384, kWsCols = 512;

struct WsSmem {
  uint8_t k[kWsStages][kWsTile];
  uint8_t v[kWsStages][kWsTile];
  uint8_t q[2][kWsTile];
  float win[2][2][4 * kWinStride];          // [weighting group][buffer]: window copies shifted by 0..3
  uint64_t k_full[kWsStages], v_full[kWsStages];
  uint64_t o_done[kWsStages];  // O-MMA of step g done: frees ring stage g % 4 and S buffer g % 3
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[kWsSBuf], p_full[kWsSBuf];
  uint64_t o_full[2], o_empty[2], drain[2];
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
__device__ __forceinline__ void nbar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
}  // namespace

template <typename T>
__global__ void __launch_bounds__(kWsThr, 1)
    h3_mixer_ws_kernel(const float* __restrict__ fdiag, const float* __restrict__ D, T* __restrict__ o, int L,
                       int heads, int B, const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  // the swizzled tiles need 1024-byte aligned atoms
  WsSmem& sm = *reinterpret_cast<WsSmem*>(smraw + ((1024u - (tc::smem_u32(smraw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int dm = heads * kHD;
  const int nt = (L + kT - 1) / kT;
  const int nitems = nt * heads * B;
  volatile int* abort_flag = &sm.abort;

  if (tid == 0) {
    for (int i = 0; i < kWsStages; ++i) {
      tc::mbar_init(&sm.k_full[i], 1);
      tc::mbar_init(&sm.v_full[i], 1);
      tc::mbar_init(&sm.o_done[i], 1);
    }
    for (int i = 0; i < kWsSBuf; ++i) {
      tc::mbar_init(&sm.s_full[i], 1);
      tc::mbar_init(&sm.p_full[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sm.q_full[i], 1);
      tc::mbar_init(&sm.q_empty[i], 1);
      tc::mbar_init(&sm.o_full[i], 1);
      tc::mbar_init(&sm.o_empty[i], 128);
      tc::mbar_init(&sm.drain[i], 1);
    }
    sm.abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(&sm.tmem_base, kWsCols);
  // launched as a programmatic dependent of the shift SSM: k~ (and, through it, the
  // filters) are read only after that kernel has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
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
    // ---------------- Q, K~ and V copies (lane 0)
    int last_q = -1;
    bool ok = true;
    for (; it.valid(); it.next()) {
      const int stg = it.g % kWsStages;
      const uint32_t use = (uint32_t)(it.g / kWsStages);
      if (lane == 0) {
        if (it.j == 0) {  // the item's Q tile, once the S-MMAs of item n - 2 are done with its buffer
          if (it.n >= 2) ok = wwait(&sm.q_empty[it.n & 1], (uint32_t)((it.n - 2) >> 1) & 1u);
          if (ok) {
            tc::mbar_expect_tx(&sm.q_full[it.n & 1], kWsTile);
            tc::tma_load_3d(tc::smem_u32(sm.q[it.n & 1]), &qmap, kHD * it.h, it.tt * kT, it.b,
                            &sm.q_full[it.n & 1]);
            last_q = it.n;
          }
        }
        if (ok && use > 0) ok = wwait(&sm.o_done[stg], (use - 1) & 1u);  // O-MMA of step g - 4
        if (ok) {
          const int s0 = it.j * kWsS;
          tc::mbar_expect_tx(&sm.k_full[stg], kWsTile);
          tc::tma_load_3d(tc::smem_u32(sm.k[stg]), &kmap, kHD * it.h, s0, it.b, &sm.k_full[stg]);
          tc::mbar_expect_tx(&sm.v_full[stg], kWsTile);
          tc::tma_load_3d(tc::smem_u32(sm.v[stg]), &vmap, kHD * it.h, s0, it.b, &sm.v_full[stg]);
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
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
      for (int n = last_q - 1; n <= last_q; ++n)
        if (n >= 0) (void)tc::mbar_wait_bounded(&sm.q_full[n & 1], (uint32_t)(n >> 1) & 1u, kWaitNs);
    }
  } else if (warp == 1) {
    // ---------------- S = Q K~^T (lane 0)
    const uint32_t idS = tc::idesc_f16(128, kWsS, Bits<T>::bf16);
    const uint64_t dq = tc::desc_sw128(tc::smem_u32(sm.q[0]), 16, 1024);
    const uint64_t dk = tc::desc_sw128(tc::smem_u32(sm.k[0]), 16, 1024);
    bool ok = true;
    for (; it.valid(); it.next()) {
      const int stg = it.g % kWsStages, sb = it.g % kWsSBuf;
      if (lane == 0) {
        if (it.j == 0) ok = wwait(&sm.q_full[it.n & 1], (uint32_t)(it.n >> 1) & 1u);
        if (ok) ok = wwait(&sm.k_full[stg], (uint32_t)(it.g / kWsStages) & 1u);
        if (ok && it.g >= kWsSBuf) {  // O-MMA of step g - 3 (never two phases behind: step g + 1 needs this S)
          const int gp = it.g - kWsSBuf;
          ok = wwait(&sm.o_done[gp % kWsStages], (uint32_t)(gp / kWsStages) & 1u);
        }
        if (ok) {
          tc::fence_after_sync();
          const uint32_t d = tmem + 128u * (uint32_t)sb;
          // descriptor start addresses advance in 16-byte units in the low bits
          const uint64_t qa = dq + (uint64_t)((it.n & 1) * (kWsTile >> 4)), ka = dk + (uint64_t)(stg * (kWsTile >> 4));
          tc::mma_f16(d, qa, ka, idS, 0u);
#pragma unroll
          for (int kk = 1; kk < kHD / 16; ++kk) tc::mma_f16(d, qa + 2u * kk, ka + 2u * kk, idS, 1u);  // +32 bytes
          tc::mma_commit(&sm.s_full[sb]);
          if (it.j + 1 == it.nst) tc::mma_commit(&sm.q_empty[it.n & 1]);
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    }
    if (lane == 0) {  // everything issued has completed before tensor memory is freed
      tc::mma_commit(&sm.drain[0]);
      (void)tc::mbar_wait_bounded(&sm.drain[0], 0, kWaitNs);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---------------- O += P V (lane 0)
    const uint32_t idO = tc::idesc_f16(128, kHD, Bits<T>::bf16, 0, 1);
    const uint64_t dv = tc::desc_sw128(tc::smem_u32(sm.v[0]), 0, 1024);
    bool ok = true;
    for (; it.valid(); it.next()) {
      const int stg = it.g % kWsStages, sb = it.g % kWsSBuf;
      if (lane == 0) {
        if (it.j == 0 && it.n >= 2) ok = wwait(&sm.o_empty[it.n & 1], (uint32_t)((it.n - 2) >> 1) & 1u);
        if (ok) ok = wwait(&sm.p_full[sb], (uint32_t)(it.g / kWsSBuf) & 1u);
        if (ok) ok = wwait(&sm.v_full[stg], (uint32_t)(it.g / kWsStages) & 1u);
        if (ok) {
          tc::fence_after_sync();
          const uint32_t d = tmem + kColO + 64u * (uint32_t)(it.n & 1), a = tmem + 128u * (uint32_t)sb;
          const uint64_t va = dv + (uint64_t)(stg * (kWsTile >> 4));
          tc::mma_f16_tmem_a(d, a, va, idO, it.j > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < kWsS / 16; ++kk)
            tc::mma_f16_tmem_a(d, a + 8u * kk, va + 128u * kk, idO, 1u);  // +2048 bytes: two K atoms
          tc::mma_commit(&sm.o_done[stg]);
          if (it.j + 1 == it.nst) tc::mma_commit(&sm.o_full[it.n & 1]);
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    }
    if (lane == 0) {
      tc::mma_commit(&sm.drain[1]);
      (void)tc::mbar_wait_bounded(&sm.drain[1], 0, kWaitNs);
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
      const int sb = it.g % kWsSBuf;
      const bool ok = wwait(&sm.s_full[sb], (uint32_t)(it.g / kWsSBuf) & 1u);
      if (nbar_or(1 + wg, 128, !ok)) break;
      tc::fence_after_sync();
      const uint32_t sa = tmem + 128u * (uint32_t)sb + lane_off;
      // weights of columns c .. c+3 (c = 0 mod 4): W[r-c+124 .. r-c+127] = copy (r & 3) at (r - (r & 3)) - c + 124
      const float* wq = wb + (row & 3) * kWinStride + (row - (row & 3)) + 124;
#pragma unroll
      for (int cb = 0; cb < kWsS / 32; ++cb) {
        float s[32];
        tc::tmem_ld16x2_wait(sa + (uint32_t)(32 * cb), sa + (uint32_t)(32 * cb + 16), s, s + 16);
        uint32_t pk[16];
#pragma unroll
        for (int g4 = 0; g4 < 8; ++g4) {
          const float4 w4 = *reinterpret_cast<const float4*>(wq - (32 * cb + 4 * g4));
          pk[2 * g4] = Bits<T>::pack(s[4 * g4] * w4.w, s[4 * g4 + 1] * w4.z);
          pk[2 * g4 + 1] = Bits<T>::pack(s[4 * g4 + 2] * w4.y, s[4 * g4 + 3] * w4.x);
        }
        // P columns [16 cb, 16 cb + 16) lie in S columns this thread has already read
        tc::tmem_st8(sa + (uint32_t)(16 * cb), pk);
        tc::tmem_st8(sa + (uint32_t)(16 * cb + 8), pk + 8);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&sm.p_full[sb]);
      buf ^= 1;
      it = nx;
      nx.next();
      nx.next();
    }
  } else if (warp >= 12) {
    // ---------------- O out
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    uint16_t* ob = reinterpret_cast<uint16_t*>(o);
    while (it.valid()) {
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
      it.next_item();
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
  const unsigned sg = (unsigned)((items + 127) / 128);
  const T* kk = (const T*)k;
  T* ko = (T*)kt;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sg);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e0;
  switch (S) {
    case 1: e0 = cudaLaunchKernelEx(&cfg, shift_ssm_kernel<T, 1>, kk, Cs, ko, B, L, dm); break;
    case 2: e0 = cudaLaunchKernelEx(&cfg, shift_ssm_kernel<T, 2>, kk, Cs, ko, B, L, dm); break;
    case 3: e0 = cudaLaunchKernelEx(&cfg, shift_ssm_kernel<T, 3>, kk, Cs, ko, B, L, dm); break;
    case 4: e0 = cudaLaunchKernelEx(&cfg, shift_ssm_kernel<T, 4>, kk, Cs, ko, B, L, dm); break;
    case 5: e0 = cudaLaunchKernelEx(&cfg, shift_ssm_kernel<T, 5>, kk, Cs, ko, B, L, dm); break;
    case 6: e0 = cudaLaunchKernelEx(&cfg, shift_ssm_kernel<T, 6>, kk, Cs, ko, B, L, dm); break;
    case 7: e0 = cudaLaunchKernelEx(&cfg, shift_ssm_kernel<T, 7>, kk, Cs, ko, B, L, dm); break;
    case 8: e0 = cudaLaunchKernelEx(&cfg, shift_ssm_kernel<T, 8>, kk, Cs, ko, B, L, dm); break;
    default: return cudaErrorInvalidValue;
  }
  if (e0 != cudaSuccess) return e0;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // Q, K~ and V tiles (128 rows x one head's 64 columns) through swizzled tensor maps
  CUtensorMap qmap, kmap, vmap;
  const cuuint64_t dims[3] = {(cuuint64_t)dm, (cuuint64_t)L, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)dm * 2, (cuuint64_t)L * dm * 2};
  const cuuint32_t box[3] = {kHD, kT, 1};
  if ((e = encode_map_3d_u16_sw128(&qmap, q, dims, strides, box)) != cudaSuccess) return e;
  if ((e = encode_map_3d_u16_sw128(&kmap, kt, dims, strides, box)) != cudaSuccess) return e;
  if ((e = encode_map_3d_u16_sw128(&vmap, v, dims, strides, box)) != cudaSuccess) return e;
  const size_t wsmem = sizeof(WsSmem) + 1024;
  if ((e = smem_optin<h3_mixer_ws_kernel<T>>(wsmem)) != cudaSuccess) return e;
  const long long tiles = (long long)((L + kT - 1) / kT) * heads * B;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int grid = (int)std::min<long long>(tiles, (long long)num_sms());
  cudaLaunchConfig_t mcfg = {};
  mcfg.gridDim = dim3(grid);
  mcfg.blockDim = dim3(kWsThr);
  mcfg.dynamicSmemBytes = wsmem;
  mcfg.stream = st;
  mcfg.attrs = attr;
  mcfg.numAttrs = 1;
  return cudaLaunchKernelEx(&mcfg, h3_mixer_ws_kernel<T>, f, D, (T*)o, L, heads, B, qmap, kmap, vmap);
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
