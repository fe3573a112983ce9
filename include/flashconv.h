/* flashconv.h -- C ABI of libflashconv_b200.so: the diagonal-SSM long
 * convolution of H3 / FlashConv on B200 (sm_100a).
 *
 * Source of every operation: "Hungry Hungry Hippos: Towards Language Modeling
 * with State Space Models" (arXiv 2212.14052v3) as summarised section by
 * section ("H3 summary") and retold in plain language ("H3 blog").  The
 * pages give no API; arguments follow their problem statement (SSM matrices
 * A, B, C, D, input u, output y).
 *
 * Conventions shared by all entry points
 * --------------------------------------
 *  - Every array pointer is caller-owned DEVICE memory on the current CUDA
 *    device, unless a comment says otherwise.  The library never allocates
 *    device memory; scratch space is passed in as `workspace`.  The one
 *    exception is ssm_conv_fwd_noalloc (below), whose scratch is a fixed
 *    array compiled into the library.
 *  - Sequences are row-major B x H x L (t contiguous); the H3 mixer's q, k, v,
 *    o are B x L x (heads*head_dim) (channel contiguous).
 *  - Complex arrays are interleaved (re, im) float32 pairs.
 *  - SSM parameters and filters are float32 whatever the I/O dtype.
 *  - I/O dtype: FC_F32, FC_F16 or FC_BF16 (u, y, q, k, v, o).  Accumulation
 *    is float32 everywhere.  With FC_F32 I/O every step runs in float32 on
 *    the CUDA cores and the output is rounded once.  With 16-bit I/O some
 *    intermediates are rounded to 16-bit tensor-core operands; each entry
 *    point states which.  All 16-bit outputs are rounded to nearest even.
 *  - u/y/q/k/v/o and filter pointers must be 16-byte aligned; parameter
 *    arrays 4-byte aligned (8-byte for complex).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous on that stream, keep no state between
 *    calls (except ssm_conv_fwd_noalloc's shared array), and may be issued
 *    from several host threads.
 *  - Return value: FC_OK, or a negative fc_status.  Argument errors are found
 *    on the host before anything is launched (nothing is written).  Launch
 *    errors come back as FC_ECUDA; faults during execution surface at the
 *    caller's next synchronisation.  fc_last_error() gives a message for the
 *    last failure on the calling host thread.
 *  - Tensor-core kernels wait on their own matrix-multiply completions with a
 *    bound of two seconds.  A block whose wait runs out (never seen in
 *    normal operation) stops, frees its tensor memory and leaves its part of
 *    the output unwritten; the call has already returned FC_OK.  Such events
 *    are counted on the device; fc_tc_timeouts() reads the count (after the
 *    caller's synchronisation), so a caller can detect an incomplete result.
 */
#ifndef FLASHCONV_B200_H
#define FLASHCONV_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FC_API __attribute__((visibility("default")))
#else
#define FC_API
#endif

typedef enum {
  FC_OK = 0,
  FC_EINVAL = -1,        /* bad argument: null pointer, size, alignment, workspace too small */
  FC_EUNSUPPORTED = -2,  /* valid but outside what is built (e.g. L not a power of two) */
  FC_ECUDA = -3,         /* a CUDA runtime call or kernel launch failed */
  FC_ENOMEM = -4         /* reserved */
} fc_status;

typedef enum { FC_F32 = 0, FC_F16 = 1, FC_BF16 = 2 } fc_dtype;

/* Library version (major*10000 + minor*100 + patch). */
FC_API int fc_version(void);

/* Static text for a status code. */
FC_API const char* fc_status_string(int status);

/* Message describing the last failing call on this host thread ("" if none). */
FC_API const char* fc_last_error(void);

/* Number of tensor-core blocks, over every kernel of the library on the
 * current device since it was loaded, that gave up waiting for a
 * matrix-multiply completion and left their part of an output unwritten
 * (see the conventions above).  0 in normal operation.  Synchronises with
 * the device (it reads a device counter). */
FC_API unsigned int fc_tc_timeouts(void);

/* ssm_kernel_gen -- diagonal-SSM convolution filter (A1).
 * H3 blog "The Convolution Connection": unrolling the recurrence gives the
 * filter f = [CB, CAB, CA^2B, ...]; H3 summary section 2 "Convolutional view".
 *   A[h,n]  = exp(dt[h] * lambda[h,n])
 *   f[h,k]  = 2 Re sum_{n<N} C[h,n] A[h,n]^k B[h,n],   0 <= k < L
 * (2 Re: conjugate-pair convention of the S4D-based diagonal SSM.)
 * Arguments: dt (H floats); lambda, Bp, Cp (H x N complex); f_out (H x L
 * floats, written).  Limits: H >= 1, 1 <= N <= 1024, 1 <= L <= 1048576.
 * A^k is evaluated with its phase k*dt*Im(lambda) reduced modulo 2 pi in
 * double precision, so long, slowly decaying filters keep their phase.
 * Precision: for N <= 64 the sum over modes is a tensor-core GEMM whose
 * operands (tables of powers and of 2 C B A^k) are each split into a 16-bit
 * high part and a 16-bit remainder (about 22 significant bits), summed in
 * float32; for N > 64 it is float32 on the CUDA cores. */
FC_API fc_status ssm_kernel_gen(const float* dt, const float* lambda, const float* Bp, const float* Cp,
                                int H, int N, int L, float* f_out, void* stream);

/* fftconv_fwd -- fused FFT causal convolution (A2-A4).
 * H3 summary section 4 "Short-sequence computation": the FFT, the pointwise
 * multiply and the inverse FFT run fused in one kernel; section 2
 * "Convolutional view": zero initial state gives a linear convolution plus a
 * residual term.
 *   y[b,h,t] = sum_{s<=t} f[h,t-s] u[b,h,s] + D[h] u[b,h,t]
 * evaluated as IFFT_{2L}(FFT_{2L}(pad u) * FFT_{2L}(pad f)) cropped to t < L.
 * u, y: B x H x L in `dtype`; f: H x L floats (any real filter, not only an
 * SSM's); D: H floats.  Limits: 1 <= L <= 8192 (any length; rows whose L is
 * not a power of two >= 16 are zero-padded on chip to the next one, which
 * leaves the causal outputs t < L exact); B, H >= 1.  u and y may not
 * overlap.
 * Precision: FC_F32 and every L without a tensor-core kernel (L < 1024 or
 * not a power of two, or L = 1024 with B <= 2): float32 FFTs on the CUDA
 * cores, one rounding at the store.  16-bit I/O at L = 1024 (B >= 3) and at
 * L = 2048, 4096, 8192 runs the block-FFT stages on the tensor cores: the
 * filter (with D added to its tap 0) is rounded to the I/O type; the DFT-128
 * stages take their data operand in the I/O type (exact for u); at L = 1024
 * the length-16 column DFTs, twiddles and filter product are float32
 * register arithmetic; at L = 2048..8192 the column DFT stages take float16
 * operands scaled so that they stay within 2 max|u| (finite for
 * |u| <= 32752); the inverse stage's input is rounded to the I/O type;
 * accumulation is float32 and y is rounded once at the store. */
FC_API fc_status fftconv_fwd(const void* u, const float* f, const float* D, void* y,
                             int B, int H, int L, fc_dtype dtype, void* stream);

/* fftconv_long_workspace -- device workspace bytes fftconv_long_fwd needs
 * for L > 8192: the complex float32 spectra of H * ceil(B / 2) row pairs
 * and of the H filters at the transform length M = 2^ceil(log2(2L - 1)),
 * i.e. 8 M (H ceil(B / 2) + H) bytes, each part rounded up to 256 bytes.
 * Returns 0 when no workspace is used (L <= 8192) and for arguments the call
 * would reject (B, H < 1, L > 65536). */
FC_API size_t fftconv_long_workspace(int B, int H, int L);

/* fftconv_long_fwd -- y = causal_conv(u, f) + D u for filters as long as the
 * input beyond fftconv_fwd's range, with an arbitrary real filter f.
 * H3 summary, appendix F "Raw speech and EEG": convolutions over 12,000-step
 * EEG clips with filters as long as the clip; §2 "Convolutional view": the
 * causal crop of the linear convolution, y[t] = sum_{s<=t} f[t-s] u[s] + D u[t].
 * u, y: B x H x L in `dtype`; f: H x L floats; D: H floats.  Limits:
 * 1 <= L <= 65536 (any length); H * ceil(B / 2) <= 2^29.  For L <= 8192
 * this is fftconv_fwd (workspace unused, may be null).  For L > 8192:
 * workspace (256-byte aligned, caller-owned, >= fftconv_long_workspace
 * bytes; contents overwritten) holds the spectra of one zero-padded FFT
 * convolution per pair of rows (two real rows of a channel packed as one
 * complex row), the M-point transform split four-step into M / 256 x 256
 * (three passes through the workspace: 256-point DFTs with the twiddle,
 * M / 256-point DFTs with the product by the filter spectrum and their
 * inverses, inverse 256-point DFTs with the crop and + D u).
 * Precision: float32 arithmetic throughout, y rounded once to `dtype`.
 * Errors: as fftconv_fwd, plus FC_EINVAL for a missing, misaligned or too
 * small workspace; nothing is launched then. */
FC_API fc_status fftconv_long_fwd(const void* u, const float* f, const float* D, void* y, int B, int H, int L,
                                  void* workspace, size_t ws_bytes, fc_dtype dtype, void* stream);

/* fftconv_bwd -- backward pass of fftconv_fwd (gradients of a loss with
 * respect to u, f and D, given its gradient dy with respect to y).
 * H3 summary, appendix C.1 "Backward Pass": the backward of the FFT
 * convolution is computed with FFTs too, with conjugate transforms, plus the
 * D u term's gradient.  Differentiating y = f * u + D u:
 *   du[b,h,s] = sum_{t>=s} f[h,t-s] dy[b,h,t] + D[h] dy[b,h,s]   (conj(F^) . DY)
 *   df[h,k]   = sum_b sum_{t>=k} dy[b,h,t] u[b,h,t-k]            (sum_b DY . conj(U))
 *   dD[h]     = sum_b sum_t dy[b,h,t] u[b,h,t]
 * dy, u, du: B x H x L in `dtype`; f: H x L floats; D, dD: H floats; df:
 * H x L floats.  du may be NULL (then f and D may be NULL too); df and dD are
 * given together or both NULL.  df and dD are overwritten, not accumulated.
 * Limits as fftconv_fwd.  Precision: du is fftconv_fwd's kernel (same
 * rounding) with the conjugate filter spectrum; df and dD are float32 FFTs
 * and sums on the CUDA cores. */
FC_API fc_status fftconv_bwd(const void* dy, const void* u, const float* f, const float* D, void* du, float* df,
                             float* dD, int B, int H, int L, fc_dtype dtype, void* stream);

/* ssm_conv_fwd -- ssm_kernel_gen followed by fftconv_fwd in one call (the
 * filter is regenerated on the device every call).  workspace must hold
 * ssm_conv_workspace(H, L) bytes (the H x L filter).  Precision: that of
 * ssm_kernel_gen followed by that of fftconv_fwd, except that when the
 * convolution runs on the tensor cores (16-bit I/O, L = 1024 with B >= 3 or
 * L in {2048, 4096, 8192}) and N <= 64, the filter comes from single fp16
 * tables (about 11 significant bits instead of 22): the convolution rounds
 * f + D to the 16-bit operand type anyway. */
FC_API size_t ssm_conv_workspace(int H, int L);
FC_API fc_status ssm_conv_fwd(const void* u, const float* dt, const float* lambda, const float* Bp,
                              const float* Cp, const float* D, void* y, int B, int H, int L, int N,
                              void* workspace, size_t ws_bytes, fc_dtype dtype, void* stream);

/* fftconv_statepass -- FlashConv state passing for long sequences (A6-A9).
 * H3 summary section 4 "Long-sequence computation" / "Correctness" and
 * appendix C "State Passing"; H3 blog "The Solution, Part 2".  The sequence
 * is split into chunks of T = `chunk`; each chunk is an FFT convolution with
 * the length-T filter plus D u plus the initial-state term, and the state is
 * carried between chunks:
 *   y[cT+t] = (f_T * u_c)[t] + D u_c[t] + 2 Re sum_n C_n A_n^(t+1) x_{c-1,n}
 *   x_c     = A^T x_{c-1} + sum_{i<T} A^(T-1-i) B u_c[i],   x_{-1} = state_in
 * The result equals the unchunked SSM output.
 * u, y: B x H x L in `dtype`; dt: H; lambda, Bp, Cp: H x N complex; D: H.
 * state_in: B x H x N complex or NULL (zero state); state_out: B x H x N
 * complex or NULL (written with x after the last chunk).  A caller can
 * split one sequence over several calls by passing state_out as the next
 * call's state_in.  workspace: at least fftconv_statepass_workspace(...)
 * bytes, 256-byte aligned.  Limits: chunk a power of two, 16 <= chunk <=
 * 8192, L % chunk == 0, 1 <= N <= 256.
 * Precision: the chunk convolutions are stored in the I/O type; the
 * initial-state term is then added to the stored values and the sum rounded
 * again (two roundings for chunks after the first).  They run on the CUDA
 * cores in float32, except with 16-bit I/O and chunk in {2048, 4096, 8192},
 * where they are fftconv_fwd's tensor-core kernel (the chunk filter then
 * comes from single fp16 tables, about 11 significant bits, for N <= 64).
 * With 16-bit I/O, those chunks and N <= 64, the end states and the
 * initial-state term are tensor-core GEMMs with u as an exact 16-bit operand:
 * the end states against a power table split hi/lo into 16-bit parts for
 * bfloat16 u (about 16 significant bits) and a single fp16 table for fp16 u
 * (11 bits); the initial-state term against single fp16 tables (11 bits,
 * below the rounding of y itself). */
FC_API size_t fftconv_statepass_workspace(int B, int H, int L, int N, int chunk);
FC_API fc_status fftconv_statepass(const void* u, const float* dt, const float* lambda, const float* Bp,
                                   const float* Cp, const float* D, void* y, int B, int H, int L, int N,
                                   int chunk, const float* state_in, float* state_out, void* workspace,
                                   size_t ws_bytes, fc_dtype dtype, void* stream);

/* fftconv_statepass_bwd -- backward pass of fftconv_statepass: gradients
 * with respect to u and state_in, given dy (the gradient with respect to y)
 * and optionally dstate_out (the gradient with respect to state_out), so that
 * a sequence split over several calls back-propagates call by call.
 * H3 summary section 4 "Long-sequence computation" and appendix C.1
 * "Backward Pass".  With complex gradients G = dL/dRe + i dL/dIm:
 *   du[t]        = sum_{s>=t} f[s-t] dy[s] + D dy[t] + Re sum_n conj(G_n) A_n^(L-1-t) B_n
 *   dstate_in[n] = sum_t dy[t] 2 conj(C_n A_n^(t+1)) + conj(A_n^L) G_n
 * (f[k] = 2 Re sum_n C_n A_n^k B_n).  It is evaluated as the adjoint SSM, a
 * forward state-passing run over the time-reversed dy with A' = conj(A),
 * B' = 2 conj(C), C' = conj(B) / 2 and initial state G / conj(A) (so A must not
 * underflow to zero where G is given).
 * dy, du: B x H x L in `dtype`; dstate_out, dstate_in: B x H x N complex or
 * NULL (NULL dstate_out: zero; NULL dstate_in: not written).  Parameters,
 * chunk and limits as fftconv_statepass.  workspace: at least
 * fftconv_statepass_bwd_workspace(...) bytes, 256-byte aligned.  Precision:
 * as fftconv_statepass (du is rounded like its y). */
FC_API size_t fftconv_statepass_bwd_workspace(int B, int H, int L, int N, int chunk, fc_dtype dtype);
FC_API fc_status fftconv_statepass_bwd(const void* dy, const float* dt, const float* lambda, const float* Bp,
                                       const float* Cp, const float* D, void* du, int B, int H, int L, int N,
                                       int chunk, const float* dstate_out, float* dstate_in, void* workspace,
                                       size_t ws_bytes, fc_dtype dtype, void* stream);

/* h3_mixer_fwd -- H3 layer core, projections excluded (A10-A11).
 * H3 blog "The Solution, Part 1": O = Q (.) SSM_diag(SSM_shift(K) (.) V);
 * H3 summary section 3 "H3 design" and appendix D.2 "H3 Complexity" (heads).
 * Per head h (channels h*hd .. h*hd+hd-1):
 *   k~[t,c]  = sum_{j<shift_len, j<=t} Cshift[c,j] k[t-j,c]   (tap 0 = current token)
 *   y_ij[t]  = sum_{s<=t} f_h[t-s] k~_i[s] v_j[s] + D_h k~_i[t] v_j[t]
 *   o_j[t]   = sum_i q_i[t] y_ij[t]
 * with f_h the diagonal-SSM filter of head h (as ssm_kernel_gen).
 * q, k, v, o: B x L x (heads*head_dim) in `dtype`; Cshift:
 * (heads*head_dim) x shift_len floats; dt, D: heads floats; lambda, Bp, Cp:
 * heads x N complex.  workspace: at least h3_mixer_workspace(...) bytes
 * (the per-head filters and, for 16-bit I/O, the shift-SSM output k~).
 * Limits: head_dim == 64, 1 <= shift_len <= 8, 1 <= L <= 65536, 1 <= N <= 1024.
 * Precision: FC_F32 runs in float32 on the CUDA cores.  16-bit I/O runs the
 * two GEMMs per tile on the tensor cores: k~ is stored in the I/O type, the
 * Toeplitz-weighted scores (f[t-s] + D [s == t]) (q_t . k~_s) are rounded to
 * the I/O type before they multiply v; accumulation is float32; for N <= 64
 * the filters come from single fp16 tables (about 11 significant bits). */
FC_API size_t h3_mixer_workspace(int B, int L, int heads, int head_dim, int N);
FC_API fc_status h3_mixer_fwd(const void* q, const void* k, const void* v, const float* Cshift,
                              const float* dt, const float* lambda, const float* Bp, const float* Cp,
                              const float* D, void* o, int B, int L, int heads, int head_dim, int N,
                              int shift_len, void* workspace, size_t ws_bytes, fc_dtype dtype,
                              void* stream);

/* ssm_decode_step -- the recurrent view, for generation: T >= 1 tokens of
 *   x <- A x + B u_t,   y_t = 2 Re sum_n C_n x_n + D u_t,   A = exp(dt lambda)
 * H3 summary section 2 "Recurrent view" (each output from the current state
 * and the new input, O(N) per token) and section 5 (generation runs step by
 * step); H3 blog "Background" (x_i from x_{i-1} and u_i).
 * u, y: B x H x T in `dtype` (T = 1 for one generated token); x: B x H x N
 * complex float32 state, read and written in place (zero for an empty
 * history; after a call it is the state after the last token, so calls
 * chain).  Parameters as ssm_kernel_gen, D: H floats.  Limits: N <= 1024,
 * H <= 65535.  Precision: float32 state and arithmetic, y rounded once. */
FC_API fc_status ssm_decode_step(const void* u, float* x, const float* dt, const float* lambda, const float* Bp,
                                 const float* Cp, const float* D, void* y, int B, int H, int N, int T,
                                 fc_dtype dtype, void* stream);

/* h3_mixer_decode_step -- one token of the H3 mixer (h3_mixer_fwd) in
 * recurrent form, for generation.  H3 summary section 2 "Recurrent view" and
 * section 5; H3 blog "The Solution, Part 1".  Per head h and channels i, j:
 *   k~_i   = sum_{s<shift_len, s<=pos} Cshift[i,s] k_{pos-s,i}   (shift SSM)
 *   X_ij  <- A_h X_ij + B_h k~_i v_j                                (N modes)
 *   o_j    = sum_i q_i (2 Re sum_n C_h,n X_ij,n + D_h k~_i v_j)
 * q, k, v, o: B x (heads*head_dim) in `dtype`, the token at position pos.
 * kring: B x (shift_len-1) x (heads*head_dim) in `dtype`, the keys of the
 * previous shift_len-1 tokens (slot p % (shift_len-1) holds position p; read
 * only for positions >= 0, so it needs no initialisation; the call stores
 * this token's keys into it; NULL allowed when shift_len == 1).  state:
 * h3_decode_state_bytes(...) bytes = B x heads x head_dim x head_dim x N
 * complex float32 ([b][head][i][j][n]), zero before position 0, updated in
 * place.  Other parameters as h3_mixer_fwd.  Calls for consecutive positions
 * must be ordered (same stream).  Limits: head_dim <= 64, shift_len <= 8,
 * N <= 1024.  Precision: float32 state and arithmetic, o rounded once. */
FC_API size_t h3_decode_state_bytes(int B, int heads, int head_dim, int N);
FC_API fc_status h3_mixer_decode_step(const void* q, const void* k, const void* v, void* kring, float* state,
                                      const float* Cshift, const float* dt, const float* lambda, const float* Bp,
                                      const float* Cp, const float* D, void* o, int B, int heads, int head_dim,
                                      int N, int shift_len, long long pos, fc_dtype dtype, void* stream);

/* ssm_conv_fwd_noalloc -- ssm_conv_fwd for callers that cannot allocate
 * device memory.  The pages have no counterpart to this call.
 *
 * Some callers cannot call cudaMalloc or lend the library a workspace: code
 * embedded in a host application whose memory manager owns every byte of
 * device memory, or a latency-critical path where an allocation is not
 * allowed.  This variant keeps its only scratch, the H x L float filter, in a
 * fixed 4 MiB array compiled into the library, so it takes no workspace and
 * allocates nothing.  Every GPU that loads the library holds one copy of that
 * array until the process exits.
 *  - The first call on a device looks up the array's device address with
 *    cudaGetSymbolAddress (that device current) and caches it; make that
 *    first call on each device before any stream capture.
 *  - Limit: H * L <= ssm_conv_noalloc_max_filter_floats() (1,048,576);
 *    larger sizes return FC_EUNSUPPORTED and launch nothing.
 *  - All calls share the one array and it keeps the last call's contents.
 *    Each call rewrites the whole filter it then reads, so nothing of an
 *    earlier call reaches a result, but calls that can overlap on the GPU
 *    (different streams with no ordering between them) race on the array and
 *    must not be issued that way.
 *  - Arguments, other limits, kernels and results as ssm_conv_fwd: the same
 *    filter kernel and the same convolution kernel (the tensor-core one for
 *    16-bit I/O at L = 1024, as in ssm_conv_fwd), so the two entry points
 *    return identical bits.  On failure the message is in
 *    ssm_conv_noalloc_last_error() (per host thread).
 *  - Like every tensor-core call, a block whose completion wait runs out
 *    leaves its part of y unwritten (fc_tc_timeouts() counts it); such a y
 *    may then hold an earlier call's values. */
FC_API fc_status ssm_conv_fwd_noalloc(const void* u, const float* dt, const float* lambda, const float* Bp,
                                      const float* Cp, const float* D, void* y, int B, int H, int L, int N,
                                      fc_dtype dtype, void* stream);
FC_API size_t ssm_conv_noalloc_max_filter_floats(void);
FC_API const char* ssm_conv_noalloc_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* FLASHCONV_B200_H */
