// Internal launchers (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

namespace fc {


// ssm_conv_fwd's dispatch: filter generation into f (H x L floats of scratch),
// then the fused convolution (tensor cores where supported).
cudaError_t run_ssm_conv(const void* u, const float* dt, const float* lambda, const float* Bp, const float* Cp,
                         const float* D, void* y, int B, int H, int L, int N, float* f, int dtype,
                         cudaStream_t st);

// hi_only (N <= 64): single fp16 tables, about 11 significant bits, for a filter that a 16-bit
// tensor-core convolution or the 16-bit mixer rounds to its operand type anyway; otherwise the
// tables are split hi + lo (about 22 bits).
cudaError_t launch_ssm_gen(const float* dt, const float* lam, const float* Bp, const float* Cp, int H, int N, int L,
                           float* f, cudaStream_t st, bool hi_only = false);

// dtype: 0 f32, 1 f16, 2 bf16.  Lc = transform half-length (chunk), C chunks per row.
// sp.dt != nullptr: generate the filter from the SSM parameters inside the
// kernel (Lc >= 1024); otherwise read it from f (row stride fstride).
// conj_filter = 1 multiplies by the conjugate filter spectrum: the result is
// then the anti-causal correlation sum_{t>=s} f[t-s] u[t] + D u[s] (the input
// gradient of the convolution); not with generated filters.
cudaError_t launch_fftconv(const void* u, const float* f, int fstride, SsmArgs sp, const float* D, void* y, int B,
                           int H, long long Lrow, int Lc, int C, int dtype, cudaStream_t st, int conj_filter = 0);

cudaError_t launch_statepass_tail(const void* u, const float* dt, const float* lam, const float* Bp,
                                  const float* Cp, void* y, int B, int H, int L, int N, int T,
                                  const float* state_in, float* state_out, float* s_ws, float* x_ws, int dtype,
                                  cudaStream_t st);

// Tensor-core state passing (fp16 / bf16, T in {2048, 4096, 8192}, N <= 64):
// end states into s_ws, and the initial-state correction added into y for
// chunks c >= c_begin (x_ws = state entering each chunk).
bool statepass_tc_supported(int T, int N, int dtype);
cudaError_t launch_sp_state_tc(const void* u, const float* dt, const float* lam, const float* Bp, int B, int H, int L,
                               int N, int T, float* s_ws, int dtype, cudaStream_t st);
cudaError_t launch_sp_corr_tc(void* y, const float* dt, const float* lam, const float* Cp, const float* x_ws, int B,
                              int H, int L, int N, int T, int c_begin, int dtype, cudaStream_t st);
unsigned int statepass_tc_timeouts();

cudaError_t launch_h3_mixer(const void* q, const void* k, const void* v, const float* Cshift, const float* fdiag,
                            const float* D, void* o, int B, int L, int heads, int shift_len, int dtype,
                            cudaStream_t st);

// Tensor-core H3 mixer (fp16 / bf16 I/O, head_dim 64, shift_len <= 8).
// ktilde: scratch of B x L x (heads*64) elements of the I/O type (the shift-SSM output).
cudaError_t launch_h3_mixer_tc(const void* q, const void* k, const void* v, const float* Cshift, const float* fdiag,
                               const float* D, void* o, void* ktilde, int B, int L, int heads, int shift_len,
                               int dtype, cudaStream_t st);
// Number of tensor-core CTAs that gave up waiting for an MMA (0 in normal operation).
unsigned int mixer_tc_timeouts();

// Recurrent view: Tn tokens of x <- A x + B u_t, y_t = 2 Re(C x) + D u_t per
// (b, h) row; u, y: B x H x Tn; x: B x H x N complex, updated in place.
cudaError_t launch_ssm_decode(const void* u, float* x, const float* dt, const float* lam, const float* Bp,
                              const float* Cp, const float* D, void* y, int B, int H, int N, int Tn, int dtype,
                              cudaStream_t st);
// One token of the H3 mixer in recurrent form (state, kring updated in place).
cudaError_t launch_h3_decode(const void* q, const void* k, const void* v, void* kring, float* state, const float* Cs,
                             const float* dt, const float* lam, const float* Bp, const float* Cp, const float* D,
                             void* o, int B, int heads, int hd, int N, int S, long long pos, int dtype,
                             cudaStream_t st);

// State-passing backward helpers: the adjoint SSM's parameters (lambda' =
// conj(lambda), B' = 2 conj(C), C' = conj(B) / 2, x0' = G / conj(A) when G is
// given), row reversal in time, and dstate_in = conj(A) lambda_0.
cudaError_t launch_sp_adjoint_params(const float* dt, const float* lam, const float* Bp, const float* Cp,
                                     const float* G, float* lam_a, float* B_a, float* C_a, float* x0_a, int B, int H,
                                     int N, cudaStream_t st);
cudaError_t launch_reverse_rows(const void* in, void* out, long long rows, int L, int dtype, cudaStream_t st);
cudaError_t launch_sp_adjoint_state(const float* dt, const float* lam, const float* lam0, float* dsin, int B, int H,
                                    int N, cudaStream_t st);

// Tensor-core fused FFT convolution (block-FFT stages as tcgen05 GEMMs).
bool fftconv_tc_supported(int L, int dtype, int B);
// after_filter_kernel: f is written by the kernel launched just before on the
// same stream (ssm_gen), which lets this launch start as its programmatic
// dependent (prologue overlapped; the filter is read only after that kernel
// has completed).
cudaError_t launch_fftconv_tc(const void* u, const float* f, const float* D, void* y, int B, int H, int L, int dtype,
                              bool after_filter_kernel, cudaStream_t st, bool conj_filter = false);

// Gradient of the convolution with respect to the filter and D:
//   df[h,k] = sum_b sum_{t>=k} dy[b,h,t] u[b,h,t-k],  dD[h] = sum_b sum_t dy u
// (CUDA cores, L a power of two in [16, 8192]).
cudaError_t launch_fftconv_dfilter(const void* dy, const void* u, float* df, float* dD, int B, int H, int L,
                                   int dtype, cudaStream_t st);
unsigned int fftconv_tc_timeouts();

// Tensor-core fused FFT convolution for transform half-lengths Lc = 2048,
// 4096, 8192 (16-bit I/O), rows laid out as launch_fftconv (C chunks of Lc
// per row of Lrow).  after_filter_kernel as launch_fftconv_tc; conj_filter as
// launch_fftconv.
bool fftconv_tcl_supported(int Lc, int dtype);
cudaError_t launch_fftconv_tcl(const void* u, const float* f, int fstride, const float* D, void* y, int B, int H,
                               long long Lrow, int Lc, int C, int dtype, bool after_filter_kernel, bool conj_filter,
                               cudaStream_t st);
unsigned int fftconv_tcl_timeouts();

// Causal convolution with an arbitrary filter for L > 8192 (any length up to
// 65536) as one four-step FFT convolution per row pair (fftconv_long.cu); the
// workspace holds the row-pair and filter spectra in complex fp32.
size_t fftconv_long_workspace_bytes(int B, int H, int L);
cudaError_t launch_fftconv_long(const void* u, const float* f, const float* D, void* y, int B, int H, int L,
                                void* workspace, int dtype, cudaStream_t st);
// Tensor-core filter generation CTAs that gave up waiting for an MMA.
unsigned int gen_tc_timeouts();

}  // namespace fc
