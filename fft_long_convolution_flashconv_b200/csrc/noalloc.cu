// ssm_conv_fwd_noalloc: filter generation + FFT convolution whose only
// scratch (the H x L filter) lives in a fixed array inside this library, for
// callers that may not allocate device memory (see include/flashconv.h).
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "../../include/flashconv.h"
#include "kernels.cuh"

namespace {

constexpr size_t kNoAllocFilterFloats = (size_t)1 << 20;  // 4 MiB: H * L <= 1,048,576

// One copy per device that loads the library, held until the process exits.
// Host code must not use this name as a device address: its address on the
// current device comes from cudaGetSymbolAddress (noalloc_scratch below).
static __device__ __align__(256) float g_noalloc_filter[kNoAllocFilterFloats];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached.
cudaError_t noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    float* p = nullptr;
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_noalloc_filter);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

thread_local char g_na_err[256] = "";

fc_status na_fail(fc_status s, const char* msg) {
  snprintf(g_na_err, sizeof(g_na_err), "%s", msg);
  return s;
}

bool al(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" {

FC_API size_t ssm_conv_noalloc_max_filter_floats(void) { return kNoAllocFilterFloats; }

FC_API const char* ssm_conv_noalloc_last_error(void) { return g_na_err; }

FC_API fc_status ssm_conv_fwd_noalloc(const void* u, const float* dt, const float* lambda, const float* Bp,
                                      const float* Cp, const float* D, void* y, int B, int H, int L, int N,
                                      fc_dtype dtype, void* stream) {
  g_na_err[0] = 0;
  if (!(dtype == FC_F32 || dtype == FC_F16 || dtype == FC_BF16)) return na_fail(FC_EINVAL, "unknown dtype");
  if (B < 1 || H < 1 || N < 1) return na_fail(FC_EINVAL, "B, H and N must be >= 1");
  if (!u || !y || !dt || !lambda || !Bp || !Cp || !D) return na_fail(FC_EINVAL, "null pointer argument");
  if (!al(u, 16) || !al(y, 16) || !al(dt, 4) || !al(lambda, 8) || !al(Bp, 8) || !al(Cp, 8) || !al(D, 4))
    return na_fail(FC_EINVAL, "misaligned pointer (u, y: 16 bytes; dt, D: 4; complex parameters: 8)");
  if (L < 1 || L > 8192) return na_fail(FC_EUNSUPPORTED, "L must be in [1, 8192]");
  if (N > 1024 || H > 65535) return na_fail(FC_EUNSUPPORTED, "N must be <= 1024 and H <= 65535");
  if (B > (1 << 30)) return na_fail(FC_EUNSUPPORTED, "B must be <= 2^30");
  if ((size_t)H * (size_t)L > kNoAllocFilterFloats)
    return na_fail(FC_EUNSUPPORTED,
                   "H * L exceeds the fixed scratch of ssm_conv_fwd_noalloc (1,048,576 filter values); "
                   "use ssm_conv_fwd with a caller workspace");
  const size_t bytes = (size_t)B * H * L * (dtype == FC_F32 ? 4 : 2);
  const char* pu = (const char*)u;
  const char* py = (const char*)y;
  if (!(pu + bytes <= py || py + bytes <= pu)) return na_fail(FC_EINVAL, "u and y overlap");
  float* f = nullptr;
  cudaError_t e = noalloc_scratch(&f);
  if (e != cudaSuccess) return na_fail(FC_ECUDA, "could not resolve the scratch array on this device");
  // the same kernels as ssm_conv_fwd, with the library array as the filter
  // scratch; the whole H x L filter is rewritten before it is read, so nothing
  // needs clearing
  e = fc::run_ssm_conv(u, dt, lambda, Bp, Cp, D, y, B, H, L, N, f, dtype, (cudaStream_t)stream);
  if (e != cudaSuccess) return na_fail(FC_ECUDA, "launch failed");
  return FC_OK;
}

}  // extern "C"
