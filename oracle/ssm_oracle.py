"""CPU fp64 oracle for the SSM long convolution (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
arm may import or run anything under ``oracle/``; the product path never does.
This code shares nothing with the CUDA library: no kernels, headers, tables or
helpers.  It is plain, slow and written to be checked by eye against the
definitions on the pages.

Sources (the pages hold prose only -- no code, no equations typeset, no
printed example values):
  * "H3 summary"  = the section-by-section summary of "Hungry Hungry Hippos:
    Towards Language Modeling with State Space Models" (arXiv 2212.14052v3).
  * "H3 blog"     = the plain-language retelling of the same paper
    ("Background: What Are State Space Models?", "The Convolution
    Connection", "The Solution, Part 1/2").

Conventions the oracle fixes where the pages are silent (each one is listed
with its reason in the design notes):
  * A complex diagonal SSM driven by real u produces a real output through
    2*Re(C x) (conjugate-pair convention of the S4D-based diagonal SSM,
    H3 blog "The Solution, Part 1", bullet "Diagonal SSM").
  * Discretisation A = exp(dt * lambda), B used as given (no ZOH factor).
  * The state x_t already contains u_t (H3 blog "Background": x_i is updated
    from x_{i-1} using u_i), so f[0] = 2 Re(C B) and an initial state x_{-1}
    reaches y_t through A^(t+1).
  * Shift SSM filter = the C_shift taps j = 0..len-1 with tap 0 = the current
    token, no D term.

parity unpinned: none -- every function below is pinned by tests in
``tests/test_oracle_pins.py`` against closed forms, special cases, brute
force or an independent formulation.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "as_complex", "discretize", "ssm_powers", "ssm_filter", "ssm_filter_from_A",
    "causal_conv_direct", "ssm_recurrence", "statepass_chunked",
    "shift_ssm", "h3_mixer_outer", "h3_mixer_toeplitz", "row_rel_err",
    "causal_conv_bwd", "h3_mixer_recurrent", "statepass_bwd",
]


def as_complex(p) -> np.ndarray:
    """(..., 2) float array of (re, im) pairs -> complex128 (exact promotion)."""
    p = np.asarray(p)
    if np.iscomplexobj(p):
        return p.astype(np.complex128)
    p = p.astype(np.float64)
    return p[..., 0] + 1j * p[..., 1]


def discretize(dt, lam) -> np.ndarray:
    """A[h, n] = exp(dt[h] * lambda[h, n]) in fp64.

    H3 summary, section 2 "State space models": the discrete-time SSM maps
    u to y through a state with matrices A, B, C, D; the diagonal SSM is
    S4D-based (H3 blog, "The Solution, Part 1").  dt and lambda are the
    float32 inputs promoted exactly to float64.
    """
    dt = np.asarray(dt, dtype=np.float64)
    lam = as_complex(lam)
    return np.exp(dt[:, None] * lam)


def ssm_powers(dt, lam, ks) -> np.ndarray:
    """A[h, n]^k for k in ``ks`` as exp(k * dt * lambda) (shape H x N x K).

    Computed from the exponent rather than by repeated multiplication so that
    it is independent of the recurrence below.
    """
    dt = np.asarray(dt, dtype=np.float64)
    lam = as_complex(lam)
    ks = np.asarray(ks, dtype=np.float64)
    return np.exp((dt[:, None] * lam)[:, :, None] * ks[None, None, :])


def ssm_filter(dt, lam, Bp, Cp, L: int) -> np.ndarray:
    """Convolution filter f[h, k] = 2 Re sum_n C[h,n] A[h,n]^k B[h,n], k < L.

    H3 blog, "The Convolution Connection": unrolling the recurrence gives
    y = f * u with f = [CB, CAB, CA^2B, ...]; the 2 Re(.) is the conjugate
    pair convention for a complex diagonal A with real u.
    """
    Bc = as_complex(Bp)
    Cc = as_complex(Cp)
    H = Bc.shape[0]
    f = np.empty((H, L), dtype=np.float64)
    ks = np.arange(L)
    for h in range(H):  # one channel at a time keeps memory small
        P = ssm_powers(np.asarray(dt)[h:h + 1], np.asarray(lam)[h:h + 1], ks)[0]  # N x L
        f[h] = 2.0 * np.real(np.sum((Cc[h] * Bc[h])[:, None] * P, axis=0))
    return f


def ssm_filter_from_A(A, Bc, Cc, L: int) -> np.ndarray:
    """Same filter for a discrete complex A given directly (reaches the A = 0
    and real-a special cases that exp(dt*lambda) cannot express exactly).
    Powers by repeated multiplication."""
    A = np.asarray(A, dtype=np.complex128)
    w = np.asarray(Cc, dtype=np.complex128) * np.asarray(Bc, dtype=np.complex128)
    H, N = A.shape
    f = np.empty((H, L), dtype=np.float64)
    p = np.ones((H, N), dtype=np.complex128)
    for k in range(L):
        f[:, k] = 2.0 * np.real(np.sum(w * p, axis=1))
        p = p * A
    return f


def causal_conv_direct(u, f, D) -> np.ndarray:
    """y[b, h, t] = sum_{s <= t} f[h, t-s] u[b, h, s] + D[h] u[b, h, t].

    H3 summary, section 2 "Convolutional view": with zero initial state the
    output is exactly a linear convolution of the input with the filter plus
    a residual (D) term.  This is the O(L^2) definition; numpy.convolve is the
    direct (non-FFT) sum, truncated to the first L outputs (causal).
    """
    u = np.asarray(u, dtype=np.float64)
    f = np.asarray(f, dtype=np.float64)
    D = np.asarray(D, dtype=np.float64)
    B, H, L = u.shape
    y = np.empty_like(u)
    for b in range(B):
        for h in range(H):
            y[b, h] = np.convolve(u[b, h], f[h, :L])[:L] + D[h] * u[b, h]
    return y


def ssm_recurrence(u, A, Bc, Cc, D, x0=None):
    """Explicit recurrence x_t = A x_{t-1} + B u_t, y_t = 2 Re(C x_t) + D u_t.

    H3 summary, section 2 "State space models" (y_i = C x_i + D u_i) and
    "Recurrent view"; H3 blog "Background" (x_i from x_{i-1} and u_i).
    u: (B, H, L); A, Bc, Cc: (H, N) complex; D: (H,); x0: (B, H, N) complex
    or None (zero state).  Returns (y, x_last) with x_last the state after
    the last step.
    """
    u = np.asarray(u, dtype=np.float64)
    A = np.asarray(A, dtype=np.complex128)
    Bc = np.asarray(Bc, dtype=np.complex128)
    Cc = np.asarray(Cc, dtype=np.complex128)
    D = np.asarray(D, dtype=np.float64)
    Bn, H, L = u.shape
    x = np.zeros((Bn, H, A.shape[1]), dtype=np.complex128) if x0 is None \
        else np.array(x0, dtype=np.complex128)
    y = np.empty_like(u)
    for t in range(L):
        x = A[None] * x + Bc[None] * u[:, :, t, None]
        y[:, :, t] = 2.0 * np.real(np.sum(Cc[None] * x, axis=2)) + D[None] * u[:, :, t]
    return y, x


def statepass_chunked(u, A, Bc, Cc, D, chunk: int, x0=None, f_chunk=None):
    """FlashConv state passing, in the order the pages give it.

    H3 summary, section 4 "Long-sequence computation": split the sequence into
    chunks; each chunk is an FFT convolution with the chunk-length filter, and
    an end-state carried between chunks initialises the next one; section 4
    "Correctness": the result equals the unchunked SSM output.  H3 summary,
    appendix C "State Passing": the chunk-input -> end-state map M_ux has the
    columns A^(T-1) B, ..., A B, B.  H3 summary, section 2 "Convolutional
    view": a chunk's output is its convolution plus the initial-state term.

    Per chunk c (length T): y_c = conv(u_c, f[:T]) + D u_c
                                  + 2 Re sum_n C_n A_n^(t+1) x_{c-1,n};
                            x_c = A^T x_{c-1} + M_ux u_c.
    Here the chunk convolution is the direct sum (the FFT is only how the
    fast path evaluates it).  Returns (y, x_last).
    """
    u = np.asarray(u, dtype=np.float64)
    A = np.asarray(A, dtype=np.complex128)
    Bc = np.asarray(Bc, dtype=np.complex128)
    Cc = np.asarray(Cc, dtype=np.complex128)
    Bn, H, L = u.shape
    T = int(chunk)
    if L % T:
        raise ValueError("L must be a multiple of the chunk length")
    if f_chunk is None:
        f_chunk = ssm_filter_from_A(A, Bc, Cc, T)
    x = np.zeros((Bn, H, A.shape[1]), dtype=np.complex128) if x0 is None \
        else np.array(x0, dtype=np.complex128)
    t1 = np.arange(1, T + 1)
    # A^(t+1), t < T  and  M_ux columns A^(T-1-i) B, i < T
    Apow_out = A[:, :, None] ** t1[None, None, :]                    # H x N x T
    Mux = (A[:, :, None] ** (T - 1 - np.arange(T))[None, None, :]) * Bc[:, :, None]
    AT = A ** T
    y = np.empty_like(u)
    for c in range(L // T):
        uc = u[:, :, c * T:(c + 1) * T]
        y_loc = causal_conv_direct(uc, f_chunk, D)
        corr = 2.0 * np.real(np.einsum("hn,hnt,bhn->bht", Cc, Apow_out, x))
        y[:, :, c * T:(c + 1) * T] = y_loc + corr
        x = AT[None] * x + np.einsum("hni,bhi->bhn", Mux, uc)
    return y, x


def shift_ssm(k, Cshift) -> np.ndarray:
    """Shift SSM on K: k~[b, t, c] = sum_{j < S, j <= t} Cshift[c, j] k[b, t-j, c].

    H3 blog, "The Solution, Part 1", bullet "Shift SSM": A is the shift
    matrix, so the state is the last few inputs and the filter is C itself
    (tap 0 = current token, tap 1 = the one just before, ...).  No D term.
    k: (B, L, C) ; Cshift: (C, S).
    """
    k = np.asarray(k, dtype=np.float64)
    Cs = np.asarray(Cshift, dtype=np.float64)
    Bn, L, C = k.shape
    out = np.zeros_like(k)
    for j in range(Cs.shape[1]):
        if j >= L:
            break
        out[:, j:, :] += Cs[None, None, :, j] * k[:, :L - j, :]
    return out


def h3_mixer_outer(q, k, v, Cshift, f, D, heads: int) -> np.ndarray:
    """H3 mixer, literal form (tiny shapes only; O(B * heads * hd^2 * L^2)).

    H3 blog "The Solution, Part 1": O = Q (.) SSM_diag(SSM_shift(K) (.) V);
    H3 summary section 3 "H3 design" and appendix D.2 "H3 Complexity"
    (multi-head, head dimension O(1)).  Per head h with channels i, j < hd:
      kv_ij[t] = k~_i[t] v_j[t]
      y_ij     = conv(kv_ij, f_h) + D_h kv_ij
      o_j[t]   = sum_i q_i[t] y_ij[t]
    f: (heads, L) diagonal-SSM filters; D: (heads,).
    """
    q = np.asarray(q, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    kt = shift_ssm(k, Cshift)
    Bn, L, dm = q.shape
    hd = dm // heads
    o = np.zeros_like(q)
    for b in range(Bn):
        for h in range(heads):
            sl = slice(h * hd, (h + 1) * hd)
            Q, K, V = q[b, :, sl], kt[b, :, sl], v[b, :, sl]
            for i in range(hd):
                for j in range(hd):
                    kv = K[:, i] * V[:, j]
                    y = np.convolve(kv, f[h])[:L] + D[h] * kv
                    o[b, :, h * hd + j] += Q[:, i] * y
    return o


def h3_mixer_toeplitz(q, k, v, Cshift, f, D, heads: int, rows=None, ts=None) -> np.ndarray:
    """Same mixer rearranged (exact in real arithmetic): for each head,
      o_j[t] = sum_{s <= t} (f_h[t-s] + D_h [s == t]) (q_t . k~_s) v_s[j].
    The sum over i of q_i[t] k~_i[s] is pulled inside the convolution.
    ``rows`` = list of (b, head) pairs and ``ts`` = time indices to evaluate
    (defaults: all).  Returns the full o array with only the requested
    entries filled (others NaN) when subsets are given.
    """
    q = np.asarray(q, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    kt = shift_ssm(k, Cshift)
    Bn, L, dm = q.shape
    hd = dm // heads
    if rows is None:
        rows = [(b, h) for b in range(Bn) for h in range(heads)]
    if ts is None:
        ts = np.arange(L)
    o = np.full_like(q, np.nan)
    for (b, h) in rows:
        sl = slice(h * hd, (h + 1) * hd)
        Q, K, V = q[b, :, sl], kt[b, :, sl], v[b, :, sl]
        for t in ts:
            s = np.arange(t + 1)
            w = f[h, t - s] * (K[: t + 1] @ Q[t])
            w[t] += D[h] * (K[t] @ Q[t])
            o[b, t, sl] = w @ V[: t + 1]
    return o


def row_rel_err(y, ref, axis=-1) -> float:
    """Max over rows of max|y - ref| / max|ref| along ``axis`` (the error metric
    for parity: per-row max-norm relative error)."""
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.max(np.abs(y - ref), axis=axis)
    den = np.max(np.abs(ref), axis=axis)
    den = np.where(den == 0, 1.0, den)
    return float(np.max(num / den))


def causal_conv_bwd(dy, u, f, D):
    """Gradients of the causal convolution y = f * u + D u (all fp64).

    H3 summary, appendix C.1 "Backward Pass": the backward pass of the FFT
    convolution is again a convolution (with the conjugate transform), plus
    the gradient of the D u term.  For a loss whose gradient with respect to
    y is dy, differentiating y[b,h,t] = sum_{s<=t} f[h,t-s] u[b,h,s] + D[h]
    u[b,h,t] term by term gives
      du[b,h,s] = sum_{t>=s} f[h,t-s] dy[b,h,t] + D[h] dy[b,h,s]   (anti-causal)
      df[h,k]   = sum_b sum_{t>=k} dy[b,h,t] u[b,h,t-k]             (k < L)
      dD[h]     = sum_b sum_t dy[b,h,t] u[b,h,t]
    written out here as the plain sums (numpy.correlate is the direct sum).
    Returns (du, df, dD).
    """
    dy = np.asarray(dy, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    f = np.asarray(f, dtype=np.float64)
    D = np.asarray(D, dtype=np.float64)
    B, H, L = u.shape
    du = np.empty_like(u)
    df = np.zeros((H, L), dtype=np.float64)
    dD = np.zeros(H, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            # du[s] = sum_k f[k] dy[s + k]  (k = t - s >= 0, s + k < L)
            du[b, h] = np.correlate(dy[b, h], f[h, :L], mode="full")[L - 1:] + D[h] * dy[b, h]
            # df[k] = sum_t dy[t] u[t - k]
            df[h] += np.correlate(dy[b, h], u[b, h], mode="full")[L - 1:]
            dD[h] += float(np.dot(dy[b, h], u[b, h]))
    return du, df, dD


def h3_mixer_recurrent(q, k, v, Cshift, A, Bc, Cc, D, heads: int) -> np.ndarray:
    """H3 mixer evaluated token by token in its recurrent form (tiny shapes).

    H3 summary, section 2 "Recurrent view" (each output from the current state;
    generation runs step by step) with the H3 layer of the H3 blog, "The
    Solution, Part 1".  Per token t, per head h, channels i, j < hd:
      k~_t      = sum_{j<S} Cshift[:, j] k_{t-j}          (shift SSM: its state is
                                                          the last S-1 inputs)
      X_ij,t    = A_h X_ij,t-1 + B_h k~_i,t v_j,t          (N complex modes)
      y_ij,t    = 2 Re(sum_n C_h,n X_ij,t,n) + D_h k~_i,t v_j,t
      o_j,t     = sum_i q_i,t y_ij,t
    A, Bc, Cc: (heads, N) complex; D: (heads,).  Returns o (B, L, heads*hd).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Cs = np.asarray(Cshift, dtype=np.float64)
    A = np.asarray(A, dtype=np.complex128)
    Bc = np.asarray(Bc, dtype=np.complex128)
    Cc = np.asarray(Cc, dtype=np.complex128)
    D = np.asarray(D, dtype=np.float64)
    Bn, L, dm = q.shape
    hd = dm // heads
    S = Cs.shape[1]
    N = A.shape[1]
    o = np.zeros_like(q)
    for b in range(Bn):
        hist = np.zeros((S, dm))                      # hist[j] = k_{t-j}
        X = np.zeros((heads, hd, hd, N), dtype=np.complex128)
        for t in range(L):
            hist = np.roll(hist, 1, axis=0)
            hist[0] = k[b, t]
            kt = np.sum(Cs.T * hist, axis=0)          # sum_j Cs[c, j] k_{t-j}[c]
            for h in range(heads):
                sl = slice(h * hd, (h + 1) * hd)
                kv = np.outer(kt[sl], v[b, t, sl])    # kv[i, j]
                X[h] = A[h][None, None, :] * X[h] + Bc[h][None, None, :] * kv[:, :, None]
                y = 2.0 * np.real(np.sum(Cc[h][None, None, :] * X[h], axis=2)) + D[h] * kv
                o[b, t, sl] = q[b, t, sl] @ y
    return o


def statepass_bwd(dy, A, Bc, Cc, D, dstate_out=None):
    """Gradients of the long-sequence SSM (state passing) with respect to u
    and the initial state.

    H3 summary, section 4 "Long-sequence computation" with appendix C.1
    "Backward Pass": the forward y_t = 2 Re(C x_t) + D u_t, x_t = A x_{t-1} +
    B u_t over the whole sequence (x_{-1} = state_in, state_out = x_{L-1});
    chunking does not change it.  For a real loss with dL/dy = dy and
    dL/d(state_out) = G (complex convention: G = dL/dRe + i dL/dIm), the
    derivatives of those sums are
      du[t]        = sum_{s>=t} f[s-t] dy[s] + D dy[t] + Re sum_n conj(G_n) A_n^(L-1-t) B_n
      dstate_in[n] = sum_t dy[t] 2 conj(C_n A_n^(t+1)) + conj(A_n^L) G_n
    with f[k] = 2 Re sum_n C_n A_n^k B_n, written here as plain sums.
    dy: (B, H, L); A, Bc, Cc: (H, N) complex; D: (H,); dstate_out:
    (B, H, N) complex or None.  Returns (du, dstate_in)."""
    dy = np.asarray(dy, dtype=np.float64)
    A = np.asarray(A, dtype=np.complex128)
    Bc = np.asarray(Bc, dtype=np.complex128)
    Cc = np.asarray(Cc, dtype=np.complex128)
    D = np.asarray(D, dtype=np.float64)
    Bn, H, L = dy.shape
    N = A.shape[1]
    G = np.zeros((Bn, H, N), dtype=np.complex128) if dstate_out is None \
        else np.asarray(dstate_out, dtype=np.complex128)
    k = np.arange(L)
    P = A[:, :, None] ** k[None, None, :]                       # H x N x L: A^k
    f = 2.0 * np.real(np.sum((Cc * Bc)[:, :, None] * P, axis=1))  # H x L
    du = np.empty_like(dy)
    dsin = np.empty((Bn, H, N), dtype=np.complex128)
    for b in range(Bn):
        for h in range(H):
            for t in range(L):
                du[b, h, t] = np.dot(f[h, :L - t], dy[b, h, t:]) + D[h] * dy[b, h, t] + \
                    np.real(np.sum(np.conj(G[b, h]) * P[h, :, L - 1 - t] * Bc[h]))
            CA = Cc[h][:, None] * (A[h][:, None] ** (k[None, :] + 1))   # N x L: C A^(t+1)
            dsin[b, h] = 2.0 * np.sum(dy[b, h][None, :] * np.conj(CA), axis=1) + np.conj(A[h] ** L) * G[b, h]
    return du, dsin
