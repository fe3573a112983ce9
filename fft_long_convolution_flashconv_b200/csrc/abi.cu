// C ABI of libflashconv_b200.so: argument validation and dispatch.  Every
// check runs on the host before anything is launched; on failure the call
// returns a negative fc_status, writes nothing, and records a message for
// fc_last_error().
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "../../include/flashconv.h"
#include "../../include/flashconv_testing.h"
#include "kernels.cuh"

namespace {

thread_local char g_err[512] = "";

fc_status fail(fc_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

fc_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return FC_OK;
  return fail(FC_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool pow2(long long x) { return x > 0 && (x & (x - 1)) == 0; }
size_t dtype_size(int d) { return d == FC_F32 ? 4 : 2; }
bool dtype_ok(int d) { return d == FC_F32 || d == FC_F16 || d == FC_BF16; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Transform half-length for a convolution of length L: the next power of two
// >= max(L, 16) (rows shorter than it are zero-padded on chip).
int transform_half(int L) {
  int Lc = 16;
  while (Lc < L) Lc <<= 1;
  return Lc;
}

#define FC_REQUIRE(cond, st, ...) \
  do {                            \
    if (!(cond)) return fail(st, __VA_ARGS__); \
  } while (0)

fc_status check_params(const float* dt, const float* lambda, const float* Bp, const float* Cp) {
  FC_REQUIRE(dt && lambda && Bp && Cp, FC_EINVAL, "null SSM parameter pointer");
  FC_REQUIRE(aligned(dt, 4) && aligned(lambda, 8) && aligned(Bp, 8) && aligned(Cp, 8), FC_EINVAL,
             "SSM parameter pointers must be 4-byte (dt) / 8-byte (complex) aligned");
  return FC_OK;
}

}  // namespace

namespace fc {
// Filter generation then the fused convolution; f is H x L floats of scratch
// (unused when the convolution kernel generates the filter itself).  Shared by
// ssm_conv_fwd (caller workspace) and ssm_conv_fwd_noalloc (library array).
cudaError_t run_ssm_conv(const void* u, const float* dt, const float* lambda, const float* Bp, const float* Cp,
                         const float* D, void* y, int B, int H, int L, int N, float* f, int dtype,
                         cudaStream_t st) {
  const SsmArgs none{nullptr, nullptr, nullptr, nullptr, 0};
  cudaError_t e;
  if (fftconv_tc_supported(L, dtype, B)) {  // filter kernel, then the tensor-core convolution
    e = launch_ssm_gen(dt, lambda, Bp, Cp, H, N, L, f, st, true);
    if (e != cudaSuccess) return e;
    return launch_fftconv_tc(u, f, D, y, B, H, L, dtype, true, st);
  }
  if (fftconv_tcl_supported(L, dtype)) {
    e = launch_ssm_gen(dt, lambda, Bp, Cp, H, N, L, f, st, true);
    if (e != cudaSuccess) return e;
    return launch_fftconv_tcl(u, f, L, D, y, B, H, L, L, 1, dtype, true, false, st);
  }
  const int Lc = transform_half(L);
  if (Lc >= 1024 && N > 64) {  // filter generated inside the convolution kernel (no tensor-core generator)
    const SsmArgs sp{dt, (const float2*)lambda, (const float2*)Bp, (const float2*)Cp, N};
    return launch_fftconv(u, nullptr, L, sp, D, y, B, H, L, Lc, 1, dtype, st);
  }
  e = launch_ssm_gen(dt, lambda, Bp, Cp, H, N, L, f, st);
  if (e != cudaSuccess) return e;
  return launch_fftconv(u, f, L, none, D, y, B, H, L, Lc, 1, dtype, st);
}
}  // namespace fc

extern "C" {

FC_API int fc_version(void) { return 100; }

FC_API const char* fc_status_string(int s) {
  switch (s) {
    case FC_OK: return "ok";
    case FC_EINVAL: return "invalid argument";
    case FC_EUNSUPPORTED: return "unsupported configuration";
    case FC_ECUDA: return "CUDA error";
    case FC_ENOMEM: return "out of memory";
    default: return "unknown status";
  }
}

FC_API const char* fc_last_error(void) { return g_err; }

FC_API fc_status ssm_kernel_gen(const float* dt, const float* lambda, const float* Bp, const float* Cp, int H, int N,
                                int L, float* f_out, void* stream) {
  g_err[0] = 0;
  FC_REQUIRE(H >= 1 && N >= 1 && L >= 1, FC_EINVAL, "H, N, L must be >= 1 (got %d, %d, %d)", H, N, L);
  FC_REQUIRE(N <= 1024, FC_EUNSUPPORTED, "N = %d > 1024", N);
  FC_REQUIRE(L <= (1 << 20), FC_EUNSUPPORTED, "L = %d > 1048576", L);
  fc_status s = check_params(dt, lambda, Bp, Cp);
  if (s != FC_OK) return s;
  FC_REQUIRE(f_out && aligned(f_out, 16), FC_EINVAL, "f_out must be non-null and 16-byte aligned");
  FC_REQUIRE(H <= 65535, FC_EUNSUPPORTED, "H = %d > 65535", H);
  return cuda_status(fc::launch_ssm_gen(dt, lambda, Bp, Cp, H, N, L, f_out, (cudaStream_t)stream),
                     "ssm_kernel_gen launch");
}

static fc_status check_conv_io(const void* u, const void* y, int B, int H, long long L, int dtype) {
  FC_REQUIRE(dtype_ok(dtype), FC_EINVAL, "unknown dtype %d", dtype);
  FC_REQUIRE(B >= 1 && H >= 1, FC_EINVAL, "B, H must be >= 1 (got %d, %d)", B, H);
  FC_REQUIRE(B <= (1 << 30), FC_EUNSUPPORTED, "B = %d > 2^30", B);
  FC_REQUIRE(u && y, FC_EINVAL, "null u or y");
  FC_REQUIRE(aligned(u, 16) && aligned(y, 16), FC_EINVAL, "u and y must be 16-byte aligned");
  const size_t bytes = (size_t)B * H * (size_t)L * dtype_size(dtype);
  const char* pu = (const char*)u;
  const char* py = (const char*)y;
  FC_REQUIRE(pu + bytes <= py || py + bytes <= pu, FC_EINVAL, "u and y overlap");
  return FC_OK;
}

FC_API fc_status fftconv_fwd(const void* u, const float* f, const float* D, void* y, int B, int H, int L,
                             fc_dtype dtype, void* stream) {
  g_err[0] = 0;
  fc_status s = check_conv_io(u, y, B, H, L, dtype);
  if (s != FC_OK) return s;
  FC_REQUIRE(f && D, FC_EINVAL, "null f or D");
  FC_REQUIRE(aligned(f, 16) && aligned(D, 4), FC_EINVAL, "f must be 16-byte aligned, D 4-byte aligned");
  FC_REQUIRE(L >= 1 && L <= 8192, FC_EUNSUPPORTED, "fftconv_fwd: L must be in [1, 8192] (got %d)", L);
  if (fc::fftconv_tc_supported(L, dtype, B))
    return cuda_status(fc::launch_fftconv_tc(u, f, D, y, B, H, L, dtype, false, (cudaStream_t)stream),
                       "fftconv_fwd (tensor cores) launch");
  if (fc::fftconv_tcl_supported(L, dtype))
    return cuda_status(fc::launch_fftconv_tcl(u, f, L, D, y, B, H, L, L, 1, dtype, false, false, (cudaStream_t)stream),
                       "fftconv_fwd (tensor cores) launch");
  const fc::SsmArgs none{nullptr, nullptr, nullptr, nullptr, 0};
  return cuda_status(
      fc::launch_fftconv(u, f, L, none, D, y, B, H, L, transform_half(L), 1, dtype, (cudaStream_t)stream),
      "fftconv_fwd launch");
}

FC_API size_t fftconv_long_workspace(int B, int H, int L) {
  if (B < 1 || H < 1 || L <= 8192 || L > 65536) return 0;
  return fc::fftconv_long_workspace_bytes(B, H, L);
}

FC_API fc_status fftconv_long_fwd(const void* u, const float* f, const float* D, void* y, int B, int H, int L,
                                  void* workspace, size_t ws_bytes, fc_dtype dtype, void* stream) {
  g_err[0] = 0;
  FC_REQUIRE(L >= 1 && L <= 65536, FC_EUNSUPPORTED, "fftconv_long_fwd: L must be in [1, 65536] (got %d)", L);
  if (L <= 8192) return fftconv_fwd(u, f, D, y, B, H, L, dtype, stream);
  fc_status s = check_conv_io(u, y, B, H, L, dtype);
  if (s != FC_OK) return s;
  FC_REQUIRE(f && D, FC_EINVAL, "null f or D");
  FC_REQUIRE(aligned(f, 16) && aligned(D, 4), FC_EINVAL, "f must be 16-byte aligned, D 4-byte aligned");
  const long long pairs = (long long)H * ((B + 1) / 2);
  FC_REQUIRE(pairs <= (1LL << 29), FC_EUNSUPPORTED, "H * ceil(B / 2) = %lld > 2^29", pairs);
  FC_REQUIRE(workspace && aligned(workspace, 256), FC_EINVAL, "workspace must be non-null and 256-byte aligned");
  const size_t need = fftconv_long_workspace(B, H, L);
  FC_REQUIRE(ws_bytes >= need, FC_EINVAL, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  return cuda_status(fc::launch_fftconv_long(u, f, D, y, B, H, L, workspace, dtype, (cudaStream_t)stream),
                     "fftconv_long_fwd launch");
}

FC_API fc_status fftconv_bwd(const void* dy, const void* u, const float* f, const float* D, void* du, float* df,
                             float* dD, int B, int H, int L, fc_dtype dtype, void* stream) {
  g_err[0] = 0;
  FC_REQUIRE(du || (df && dD), FC_EINVAL, "nothing to compute: du is null and df / dD are null");
  FC_REQUIRE(L >= 1, FC_EINVAL, "L must be >= 1");
  FC_REQUIRE((df == nullptr) == (dD == nullptr), FC_EINVAL, "df and dD must both be given or both be null");
  FC_REQUIRE(dtype_ok(dtype), FC_EINVAL, "unknown dtype %d", dtype);
  FC_REQUIRE(B >= 1 && H >= 1, FC_EINVAL, "B, H must be >= 1 (got %d, %d)", B, H);
  FC_REQUIRE(B <= (1 << 30), FC_EUNSUPPORTED, "B = %d > 2^30", B);
  FC_REQUIRE(dy && aligned(dy, 16), FC_EINVAL, "dy must be non-null and 16-byte aligned");
  fc_status s = FC_OK;
  if (du) {  // du may not overlap dy
    s = check_conv_io(dy, du, B, H, L, dtype);
    if (s != FC_OK) return s;
  }
  FC_REQUIRE(L >= 1 && L <= 8192, FC_EUNSUPPORTED, "fftconv_bwd: L must be in [1, 8192] (got %d)", L);
  FC_REQUIRE(H <= 65535, FC_EUNSUPPORTED, "H = %d > 65535", H);
  if (du) FC_REQUIRE(f && D && aligned(f, 16) && aligned(D, 4), FC_EINVAL, "du needs f (16-byte aligned) and D");
  if (df)
    FC_REQUIRE(u && aligned(u, 16) && aligned(df, 4) && aligned(dD, 4), FC_EINVAL,
               "df needs u (16-byte aligned); df, dD 4-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  if (du) {
    s = fc::fftconv_tc_supported(L, dtype, B)
            ? cuda_status(fc::launch_fftconv_tc(dy, f, D, du, B, H, L, dtype, false, st, true),
                          "fftconv_bwd: du (tensor cores) launch")
        : fc::fftconv_tcl_supported(L, dtype)
            ? cuda_status(fc::launch_fftconv_tcl(dy, f, L, D, du, B, H, L, L, 1, dtype, false, true, st),
                          "fftconv_bwd: du (tensor cores) launch")
            : cuda_status(fc::launch_fftconv(dy, f, L, fc::SsmArgs{nullptr, nullptr, nullptr, nullptr, 0}, D, du, B,
                                             H, L, transform_half(L), 1, dtype, st, 1),
                          "fftconv_bwd: du launch");
    if (s != FC_OK) return s;
  }
  if (df) {
    s = cuda_status(fc::launch_fftconv_dfilter(dy, u, df, dD, B, H, L, dtype, st), "fftconv_bwd: df launch");
  }
  return s;
}

FC_API size_t ssm_conv_workspace(int H, int L) {
  if (H < 1 || L < 1) return 0;
  return round_up((size_t)H * L * sizeof(float), 256);
}

FC_API fc_status ssm_conv_fwd(const void* u, const float* dt, const float* lambda, const float* Bp, const float* Cp,
                              const float* D, void* y, int B, int H, int L, int N, void* workspace,
                              size_t ws_bytes, fc_dtype dtype, void* stream) {
  g_err[0] = 0;
  fc_status s = check_conv_io(u, y, B, H, L, dtype);
  if (s != FC_OK) return s;
  s = check_params(dt, lambda, Bp, Cp);
  if (s != FC_OK) return s;
  FC_REQUIRE(D && aligned(D, 4), FC_EINVAL, "null or misaligned D");
  FC_REQUIRE(N >= 1 && N <= 1024, FC_EUNSUPPORTED, "N must be in [1, 1024] (got %d)", N);
  FC_REQUIRE(L >= 1 && L <= 8192, FC_EUNSUPPORTED, "ssm_conv_fwd: L must be in [1, 8192] (got %d)", L);
  FC_REQUIRE(H <= 65535, FC_EUNSUPPORTED, "H = %d > 65535", H);
  FC_REQUIRE(workspace && aligned(workspace, 256), FC_EINVAL, "workspace must be non-null and 256-byte aligned");
  FC_REQUIRE(ws_bytes >= ssm_conv_workspace(H, L), FC_EINVAL, "workspace too small: %zu < %zu bytes", ws_bytes,
             ssm_conv_workspace(H, L));
  return cuda_status(fc::run_ssm_conv(u, dt, lambda, Bp, Cp, D, y, B, H, L, N, (float*)workspace, dtype,
                                       (cudaStream_t)stream),
                     "ssm_conv_fwd launch");
}

// The state-passing pipeline on validated arguments: chunk filter, chunk
// convolutions, then end states, carry and initial-state term.
static fc_status statepass_run(const void* u, const float* dt, const float* lambda, const float* Bp, const float* Cp,
                               const float* D, void* y, int B, int H, int L, int N, int chunk, const float* state_in,
                               float* state_out, float* fT, float* s_ws, float* x_ws, int dtype, cudaStream_t st) {
  const int C = L / chunk;
  fc_status s = cuda_status(fc::launch_ssm_gen(dt, lambda, Bp, Cp, H, N, chunk, fT, st,
                                               fc::fftconv_tcl_supported(chunk, dtype)),
                            "statepass: filter launch");
  if (s != FC_OK) return s;
  const fc::SsmArgs none{nullptr, nullptr, nullptr, nullptr, 0};
  s = fc::fftconv_tcl_supported(chunk, dtype)
          ? cuda_status(fc::launch_fftconv_tcl(u, fT, chunk, D, y, B, H, L, chunk, C, dtype, true, false, st),
                        "statepass: chunk conv (tensor cores) launch")
          : cuda_status(fc::launch_fftconv(u, fT, chunk, none, D, y, B, H, L, chunk, C, dtype, st),
                        "statepass: chunk conv launch");
  if (s != FC_OK) return s;
  return cuda_status(fc::launch_statepass_tail(u, dt, lambda, Bp, Cp, y, B, H, L, N, chunk, state_in, state_out,
                                               s_ws, x_ws, dtype, st),
                     "statepass: state launch");
}

// workspace layout: [f_T: H*T floats][s: B*H*C*N complex][x: B*H*C*N complex], each 256-aligned
FC_API size_t fftconv_statepass_workspace(int B, int H, int L, int N, int chunk) {
  if (B < 1 || H < 1 || L < 1 || N < 1 || chunk < 1 || L % chunk) return 0;
  const size_t C = (size_t)(L / chunk);
  const size_t fb = round_up((size_t)H * chunk * sizeof(float), 256);
  const size_t sb = round_up((size_t)B * H * C * N * 2 * sizeof(float), 256);
  return fb + 2 * sb;
}

FC_API fc_status fftconv_statepass(const void* u, const float* dt, const float* lambda, const float* Bp,
                                   const float* Cp, const float* D, void* y, int B, int H, int L, int N, int chunk,
                                   const float* state_in, float* state_out, void* workspace, size_t ws_bytes,
                                   fc_dtype dtype, void* stream) {
  g_err[0] = 0;
  FC_REQUIRE(L >= 1, FC_EINVAL, "L must be >= 1");
  fc_status s = check_conv_io(u, y, B, H, L, dtype);
  if (s != FC_OK) return s;
  s = check_params(dt, lambda, Bp, Cp);
  if (s != FC_OK) return s;
  FC_REQUIRE(D && aligned(D, 4), FC_EINVAL, "null or misaligned D");
  FC_REQUIRE(N >= 1 && N <= 256, FC_EUNSUPPORTED, "N must be in [1, 256] (got %d)", N);
  FC_REQUIRE(pow2(chunk) && chunk >= 16 && chunk <= 8192, FC_EUNSUPPORTED,
             "chunk must be a power of two in [16, 8192] (got %d)", chunk);
  FC_REQUIRE(L % chunk == 0, FC_EINVAL, "L = %d is not a multiple of chunk = %d", L, chunk);
  FC_REQUIRE(H <= 65535 && B <= 65535 && L / chunk <= 2147483647, FC_EUNSUPPORTED, "B or H > 65535");
  FC_REQUIRE(!state_in || aligned(state_in, 8), FC_EINVAL, "state_in must be 8-byte aligned");
  FC_REQUIRE(!state_out || aligned(state_out, 8), FC_EINVAL, "state_out must be 8-byte aligned");
  FC_REQUIRE(workspace && aligned(workspace, 256), FC_EINVAL, "workspace must be non-null and 256-byte aligned");
  const size_t need = fftconv_statepass_workspace(B, H, L, N, chunk);
  FC_REQUIRE(ws_bytes >= need, FC_EINVAL, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  const int C = L / chunk;
  const size_t fb = round_up((size_t)H * chunk * sizeof(float), 256);
  const size_t sb = round_up((size_t)B * H * C * N * 2 * sizeof(float), 256);
  return statepass_run(u, dt, lambda, Bp, Cp, D, y, B, H, L, N, chunk, state_in, state_out, (float*)workspace,
                       (float*)((char*)workspace + fb), (float*)((char*)workspace + fb + sb), dtype,
                       (cudaStream_t)stream);
}

// workspace: [forward workspace][lambda', B', C': 3 x H x N complex][x0': B x H x N complex]
//            [lambda_0: B x H x N complex][dy reversed][du reversed], each 256-aligned
FC_API size_t fftconv_statepass_bwd_workspace(int B, int H, int L, int N, int chunk, fc_dtype dtype) {
  const size_t fw = fftconv_statepass_workspace(B, H, L, N, chunk);
  if (fw == 0 || !dtype_ok(dtype)) return 0;
  const size_t pb = round_up((size_t)H * N * 2 * sizeof(float), 256);
  const size_t xb = round_up((size_t)B * H * N * 2 * sizeof(float), 256);
  const size_t rb = round_up((size_t)B * H * L * dtype_size(dtype), 256);
  return fw + 3 * pb + 2 * xb + 2 * rb;
}

FC_API fc_status fftconv_statepass_bwd(const void* dy, const float* dt, const float* lambda, const float* Bp,
                                       const float* Cp, const float* D, void* du, int B, int H, int L, int N,
                                       int chunk, const float* dstate_out, float* dstate_in, void* workspace,
                                       size_t ws_bytes, fc_dtype dtype, void* stream) {
  g_err[0] = 0;
  FC_REQUIRE(L >= 1, FC_EINVAL, "L must be >= 1");
  fc_status s = check_conv_io(dy, du, B, H, L, dtype);
  if (s != FC_OK) return s;
  s = check_params(dt, lambda, Bp, Cp);
  if (s != FC_OK) return s;
  FC_REQUIRE(D && aligned(D, 4), FC_EINVAL, "null or misaligned D");
  FC_REQUIRE(N >= 1 && N <= 256, FC_EUNSUPPORTED, "N must be in [1, 256] (got %d)", N);
  FC_REQUIRE(pow2(chunk) && chunk >= 16 && chunk <= 8192, FC_EUNSUPPORTED,
             "chunk must be a power of two in [16, 8192] (got %d)", chunk);
  FC_REQUIRE(L % chunk == 0, FC_EINVAL, "L = %d is not a multiple of chunk = %d", L, chunk);
  FC_REQUIRE(H <= 65535 && B <= 65535, FC_EUNSUPPORTED, "B or H > 65535");
  FC_REQUIRE(!dstate_out || aligned(dstate_out, 8), FC_EINVAL, "dstate_out must be 8-byte aligned");
  FC_REQUIRE(!dstate_in || aligned(dstate_in, 8), FC_EINVAL, "dstate_in must be 8-byte aligned");
  FC_REQUIRE(workspace && aligned(workspace, 256), FC_EINVAL, "workspace must be non-null and 256-byte aligned");
  const size_t need = fftconv_statepass_bwd_workspace(B, H, L, N, chunk, dtype);
  FC_REQUIRE(ws_bytes >= need, FC_EINVAL, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  const int C = L / chunk;
  const size_t fb = round_up((size_t)H * chunk * sizeof(float), 256);
  const size_t sb = round_up((size_t)B * H * C * N * 2 * sizeof(float), 256);
  const size_t fw = fftconv_statepass_workspace(B, H, L, N, chunk);
  const size_t pb = round_up((size_t)H * N * 2 * sizeof(float), 256);
  const size_t xb = round_up((size_t)B * H * N * 2 * sizeof(float), 256);
  const size_t rb = round_up((size_t)B * H * L * dtype_size(dtype), 256);
  char* w = (char*)workspace;
  float* lam_a = (float*)(w + fw);
  float* B_a = (float*)(w + fw + pb);
  float* C_a = (float*)(w + fw + 2 * pb);
  float* x0_a = (float*)(w + fw + 3 * pb);
  float* lam0 = (float*)(w + fw + 3 * pb + xb);
  void* dy_rev = w + fw + 3 * pb + 2 * xb;
  void* du_rev = w + fw + 3 * pb + 2 * xb + rb;
  cudaStream_t st = (cudaStream_t)stream;
  s = cuda_status(fc::launch_sp_adjoint_params(dt, lambda, Bp, Cp, dstate_out, lam_a, B_a, C_a, x0_a, B, H, N, st),
                  "statepass_bwd: adjoint parameters launch");
  if (s != FC_OK) return s;
  s = cuda_status(fc::launch_reverse_rows(dy, dy_rev, (long long)B * H, L, dtype, st), "statepass_bwd: reverse dy");
  if (s != FC_OK) return s;
  s = statepass_run(dy_rev, dt, lam_a, B_a, C_a, D, du_rev, B, H, L, N, chunk, dstate_out ? x0_a : nullptr,
                    dstate_in ? lam0 : nullptr, (float*)w, (float*)(w + fb), (float*)(w + fb + sb), dtype, st);
  if (s != FC_OK) return s;
  s = cuda_status(fc::launch_reverse_rows(du_rev, du, (long long)B * H, L, dtype, st), "statepass_bwd: reverse du");
  if (s != FC_OK || !dstate_in) return s;
  return cuda_status(fc::launch_sp_adjoint_state(dt, lambda, lam0, dstate_in, B, H, N, st),
                     "statepass_bwd: initial-state gradient launch");
}

// workspace layout: [f: heads*L floats][k~: B*L*heads*head_dim 16-bit elements], each 256-aligned
FC_API size_t h3_mixer_workspace(int B, int L, int heads, int head_dim, int N) {
  (void)N;
  if (heads < 1 || L < 1 || B < 1 || head_dim < 1) return 0;
  return round_up((size_t)heads * L * sizeof(float), 256) + round_up((size_t)B * L * heads * head_dim * 2, 256);
}

FC_API fc_status h3_mixer_fwd(const void* q, const void* k, const void* v, const float* Cshift, const float* dt,
                              const float* lambda, const float* Bp, const float* Cp, const float* D, void* o, int B,
                              int L, int heads, int head_dim, int N, int shift_len, void* workspace,
                              size_t ws_bytes, fc_dtype dtype, void* stream) {
  g_err[0] = 0;
  FC_REQUIRE(dtype_ok(dtype), FC_EINVAL, "unknown dtype %d", dtype);
  FC_REQUIRE(q && k && v && o, FC_EINVAL, "null q, k, v or o");
  FC_REQUIRE(aligned(q, 16) && aligned(k, 16) && aligned(v, 16) && aligned(o, 16), FC_EINVAL,
             "q, k, v, o must be 16-byte aligned");
  FC_REQUIRE(Cshift && D && aligned(Cshift, 4) && aligned(D, 4), FC_EINVAL, "null or misaligned Cshift / D");
  fc_status s = check_params(dt, lambda, Bp, Cp);
  if (s != FC_OK) return s;
  FC_REQUIRE(B >= 1 && L >= 1 && heads >= 1, FC_EINVAL, "B, L, heads must be >= 1");
  FC_REQUIRE(head_dim == 64, FC_EUNSUPPORTED, "head_dim must be 64 (got %d)", head_dim);
  FC_REQUIRE(shift_len >= 1 && shift_len <= 8, FC_EUNSUPPORTED, "shift_len must be in [1, 8] (got %d)",
             shift_len);
  FC_REQUIRE(L <= 65536, FC_EUNSUPPORTED, "L = %d > 65536", L);
  FC_REQUIRE(N >= 1 && N <= 1024, FC_EUNSUPPORTED, "N must be in [1, 1024]");
  FC_REQUIRE(heads <= 65535 && B <= 65535, FC_EUNSUPPORTED, "B or heads > 65535");
  const size_t bytes = (size_t)B * L * heads * head_dim * dtype_size(dtype);
  const char* po = (const char*)o;
  for (const void* in : {q, k, v}) {
    const char* pi = (const char*)in;
    FC_REQUIRE(po + bytes <= pi || pi + bytes <= po, FC_EINVAL, "o overlaps an input");
  }
  FC_REQUIRE(workspace && aligned(workspace, 256), FC_EINVAL, "workspace must be non-null and 256-byte aligned");
  const size_t need = h3_mixer_workspace(B, L, heads, head_dim, N);
  FC_REQUIRE(ws_bytes >= need, FC_EINVAL, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  float* f = (float*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  s = cuda_status(fc::launch_ssm_gen(dt, lambda, Bp, Cp, heads, N, L, f, st, dtype == FC_F16 || dtype == FC_BF16),
                  "h3_mixer: filter launch");
  if (s != FC_OK) return s;
  if (dtype == FC_F16 || dtype == FC_BF16) {
    void* kt = (char*)workspace + round_up((size_t)heads * L * sizeof(float), 256);
    return cuda_status(fc::launch_h3_mixer_tc(q, k, v, Cshift, f, D, o, kt, B, L, heads, shift_len, dtype, st),
                       "h3_mixer (tensor cores) launch");
  }
  return cuda_status(fc::launch_h3_mixer(q, k, v, Cshift, f, D, o, B, L, heads, shift_len, dtype, st),
                     "h3_mixer launch");
}

FC_API fc_status ssm_decode_step(const void* u, float* x, const float* dt, const float* lambda, const float* Bp,
                                 const float* Cp, const float* D, void* y, int B, int H, int N, int T,
                                 fc_dtype dtype, void* stream) {
  g_err[0] = 0;
  FC_REQUIRE(T >= 1, FC_EINVAL, "T must be >= 1 (got %d)", T);
  fc_status s = check_conv_io(u, y, B, H, T, dtype);
  if (s != FC_OK) return s;
  s = check_params(dt, lambda, Bp, Cp);
  if (s != FC_OK) return s;
  FC_REQUIRE(D && aligned(D, 4), FC_EINVAL, "null or misaligned D");
  FC_REQUIRE(x && aligned(x, 8), FC_EINVAL, "x must be non-null and 8-byte aligned");
  FC_REQUIRE(N >= 1 && N <= 1024, FC_EUNSUPPORTED, "N must be in [1, 1024] (got %d)", N);
  FC_REQUIRE(H <= 65535, FC_EUNSUPPORTED, "H = %d > 65535", H);
  return cuda_status(fc::launch_ssm_decode(u, x, dt, lambda, Bp, Cp, D, y, B, H, N, T, dtype, (cudaStream_t)stream),
                     "ssm_decode_step launch");
}

FC_API size_t h3_decode_state_bytes(int B, int heads, int head_dim, int N) {
  if (B < 1 || heads < 1 || head_dim < 1 || N < 1) return 0;
  return (size_t)B * heads * head_dim * head_dim * N * 2 * sizeof(float);
}

FC_API fc_status h3_mixer_decode_step(const void* q, const void* k, const void* v, void* kring, float* state,
                                      const float* Cshift, const float* dt, const float* lambda, const float* Bp,
                                      const float* Cp, const float* D, void* o, int B, int heads, int head_dim,
                                      int N, int shift_len, long long pos, fc_dtype dtype, void* stream) {
  g_err[0] = 0;
  FC_REQUIRE(dtype_ok(dtype), FC_EINVAL, "unknown dtype %d", dtype);
  FC_REQUIRE(q && k && v && o && state, FC_EINVAL, "null q, k, v, o or state");
  FC_REQUIRE(aligned(q, 16) && aligned(k, 16) && aligned(v, 16) && aligned(o, 16) && aligned(state, 8), FC_EINVAL,
             "q, k, v, o must be 16-byte aligned, state 8-byte aligned");
  FC_REQUIRE(Cshift && D && aligned(Cshift, 4) && aligned(D, 4), FC_EINVAL, "null or misaligned Cshift / D");
  fc_status s = check_params(dt, lambda, Bp, Cp);
  if (s != FC_OK) return s;
  FC_REQUIRE(B >= 1 && heads >= 1 && pos >= 0, FC_EINVAL, "B, heads must be >= 1 and pos >= 0");
  FC_REQUIRE(head_dim >= 1 && head_dim <= 64, FC_EUNSUPPORTED, "head_dim must be in [1, 64] (got %d)", head_dim);
  FC_REQUIRE(shift_len >= 1 && shift_len <= 8, FC_EUNSUPPORTED, "shift_len must be in [1, 8] (got %d)", shift_len);
  FC_REQUIRE(shift_len == 1 || (kring && aligned(kring, 16)), FC_EINVAL, "kring must be non-null and 16-byte aligned");
  FC_REQUIRE(N >= 1 && N <= 1024, FC_EUNSUPPORTED, "N must be in [1, 1024]");
  FC_REQUIRE(heads <= 65535 && B <= 65535, FC_EUNSUPPORTED, "B or heads > 65535");
  return cuda_status(fc::launch_h3_decode(q, k, v, kring, state, Cshift, dt, lambda, Bp, Cp, D, o, B, heads,
                                          head_dim, N, shift_len, pos, dtype, (cudaStream_t)stream),
                     "h3_mixer_decode_step launch");
}

FC_API unsigned int fc_tc_timeouts(void) {
  return fc::mixer_tc_timeouts() + fc::fftconv_tc_timeouts() + fc::fftconv_tcl_timeouts() +
         fc::statepass_tc_timeouts() + fc::gen_tc_timeouts();
}

FC_TEST_API unsigned int fc_debug_tc_timeouts(void) { return fc_tc_timeouts(); }

}  // extern "C"
