// Shared device helpers: complex arithmetic, I/O dtype conversion and the
// exactly phase-reduced SSM power A^k = exp(k * dt * lambda).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace fc {

// Diagonal-SSM parameters for kernels that generate their filter (dt == nullptr: none).
struct SsmArgs {
  const float* dt;
  const float2* lam;
  const float2* Bp;
  const float2* Cp;
  int N;
};

// ---- per-device launch setup, cached so that repeated calls do not repeat
// runtime queries.  Devices with an ordinal >= 64 are served uncached.
inline int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

// Number of SMs of the current device.
inline int num_sms() {
  static std::atomic<int> cache[64];
  const int d = current_device();
  if (d >= 0 && d < 64) {
    const int c = cache[d].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n < 1) n = 1;
  if (d >= 0 && d < 64) cache[d].store(n, std::memory_order_relaxed);
  return n;
}

// Opt the kernel Kern in to `bytes` of dynamic shared memory once per device
// (one cache per kernel instantiation; requests are monotone per kernel).
template <auto Kern>
cudaError_t smem_optin(size_t bytes) {
  static std::atomic<unsigned long long> done{0};
  static std::atomic<size_t> max_bytes[64];
  const int d = current_device();
  const bool cacheable = d >= 0 && d < 64;
  if (cacheable && (done.load(std::memory_order_acquire) >> d & 1ull) &&
      max_bytes[d].load(std::memory_order_relaxed) >= bytes)
    return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && cacheable) {
    max_bytes[d].store(bytes, std::memory_order_relaxed);
    done.fetch_or(1ull << d, std::memory_order_release);
  }
  return e;
}

// Debug-build bounds checks (-DFC_CHECK): a failed check records
// (site << 48 | index) in a per-file device word and the access is skipped.
#ifdef FC_CHECK
static __device__ unsigned long long g_fc_check;
__device__ __forceinline__ bool fc_ok(int site, long long idx, long long lim) {
  if (idx >= 0 && idx < lim) return true;
  atomicCAS(&g_fc_check, 0ull, ((unsigned long long)site << 48) | ((unsigned long long)idx & 0xffffffffffffull));
  return false;
}
#define FC_OK_IDX(site, idx, lim) ::fc::fc_ok((site), (long long)(idx), (long long)(lim))
#define FC_CHECK_READER(name)                                                        \
  extern "C" __attribute__((visibility("default"))) unsigned long long name() {     \
    unsigned long long v = 0;                                                        \
    cudaMemcpyFromSymbol(&v, ::fc::g_fc_check, sizeof(v));                          \
    return v;                                                                        \
  }
#else
#define FC_OK_IDX(site, idx, lim) true
#define FC_CHECK_READER(name)
#endif

__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
__device__ __forceinline__ float2 cconj(float2 a) { return make_float2(a.x, -a.y); }

// ---- I/O element types --------------------------------------------------------------
template <typename T> struct IO;
template <> struct IO<float> {
  static __device__ __forceinline__ float ld(const float* p) { return __ldg(p); }
  static __device__ __forceinline__ float ldplain(const float* p) { return *p; }
  static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
};
template <> struct IO<__half> {
  static __device__ __forceinline__ float ld(const __half* p) { return __half2float(__ldg(p)); }
  static __device__ __forceinline__ float ldplain(const __half* p) { return __half2float(*p); }
  static __device__ __forceinline__ void st(__half* p, float v) { *p = __float2half_rn(v); }
};
template <> struct IO<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }
  static __device__ __forceinline__ float ldplain(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// ---- SSM powers ------------------------------------------------------------------
// A^k for A = exp(dt * (lr + i li)):  |A^k| = exp(k dt lr), arg = k dt li.
// The phase k*dt*li (radians, up to ~1e7 for long filters with large Im(lambda))
// is formed in double precision (dt*li is exact in double; the product with k has
// relative error 1e-16) and reduced modulo 2*pi there, so the float sine/cosine
// only ever sees |angle| <= pi.  The error of the reduction is |q| times the
// rounding of 2*pi in double (~2.4e-16), i.e. < 1e-9 rad for |phase| < 1e7.
__device__ __forceinline__ float2 ssm_pow(float dt, float lr, float li, double k) {
  const double two_pi = 6.283185307179586476925286766559;
  const double ph = k * ((double)dt * (double)li);
  const double q = rint(ph * (1.0 / two_pi));
  const float red = (float)fma(-q, two_pi, ph);
  float s, c;
  sincosf(red, &s, &c);
  const float mag = expf((float)(k * ((double)dt * (double)lr)));
  return make_float2(mag * c, mag * s);
}

}  // namespace fc
