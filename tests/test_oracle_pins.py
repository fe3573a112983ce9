"""Pins for the fp64 oracle: each check ties it to something other than itself
(hand-worked values, closed forms, special cases, an independent formulation,
a library FFT), chosen so that a dropped term, a wrong sign or index, or a
transposed operand fails at least one.  CPU only."""
import numpy as np
import pytest

from oracle import ssm_oracle as O
from oracle import cref
from fft_long_convolution_flashconv_b200 import workloads as W


def _cplx(pair):
    return complex(pair[0], pair[1])


# ---------------------------------------------------------------- hand-worked fixtures
def test_golden_real_n1(golden):
    g = golden("hand_worked_real_n1.txt")
    A = np.array([[g["a"][0]]], dtype=np.complex128)
    Bc = np.array([[_cplx(g["B"])]])
    Cc = np.array([[_cplx(g["C"])]])
    D = np.array(g["D"])
    u = np.array(g["u"]).reshape(1, 1, -1)
    L = u.shape[-1]
    f = O.ssm_filter_from_A(A, Bc, Cc, L)
    assert np.array_equal(f[0], np.array(g["f"]))
    y = O.causal_conv_direct(u, f, D)
    assert np.allclose(y[0, 0], g["y"], rtol=0, atol=1e-15)
    y2, x = O.ssm_recurrence(u, A, Bc, Cc, D)
    assert np.allclose(y2[0, 0], g["y"], rtol=0, atol=1e-15)
    assert abs(x[0, 0, 0] - _cplx(g["x_last"])) < 1e-15
    yc = cref.causal_conv(u, f, D)
    assert np.allclose(yc[0, 0], g["y"], rtol=0, atol=1e-15)
    yr, xr = cref.ssm_recurrence(u, A, Bc, Cc, D)
    assert np.allclose(yr[0, 0], g["y"], rtol=0, atol=1e-15)
    assert abs(xr[0, 0, 0] - _cplx(g["x_last"])) < 1e-15


def test_golden_complex_rotation(golden):
    g = golden("hand_worked_complex_rotation.txt")
    A = np.array([[_cplx(g["A"])]])
    f = O.ssm_filter_from_A(A, np.array([[_cplx(g["B"])]]), np.array([[_cplx(g["C"])]]), 8)
    assert np.allclose(f[0], g["f"], atol=1e-14)
    # the exp(dt*lambda) form reaches the same A with dt = 1, lambda = i*pi/2
    lam = np.array([[[0.0, np.pi / 2]]])
    f2 = O.ssm_filter(np.array([1.0]), lam, np.array([[[1.0, 0.0]]]), np.array([[g["C"]]]), 8)
    assert np.allclose(f2[0], g["f"], atol=1e-12)


def test_golden_shift_ssm(golden):
    g = golden("hand_worked_shift_ssm.txt")
    k = np.array(g["k"]).reshape(1, -1, 1)
    Cs = np.array(g["Cshift"]).reshape(1, -1)
    out = O.shift_ssm(k, Cs)
    assert np.array_equal(out[0, :, 0], np.array(g["ktilde"]))


def test_golden_h3_mixer(golden):
    g = golden("hand_worked_h3_mixer.txt")
    q = np.array(g["q"]).reshape(1, 2, 2)
    k = np.array(g["k"]).reshape(1, 2, 2)
    v = np.array(g["v"]).reshape(1, 2, 2)
    Cs = np.array([[1.0, 0, 0, 0], [1.0, 0, 0, 0]])
    f = np.array(g["f"]).reshape(1, 2)
    D = np.array(g["D"])
    o1 = O.h3_mixer_outer(q, k, v, Cs, f, D, heads=1)
    o2 = O.h3_mixer_toeplitz(q, k, v, Cs, f, D, heads=1)
    want = np.array(g["o"]).reshape(1, 2, 2)
    assert np.allclose(o1, want, atol=1e-14)
    assert np.allclose(o2, want, atol=1e-14)


# ---------------------------------------------------------------- closed forms / invariants
def _small(seed=11, B=2, H=3, L=64, N=8, dt=("loguniform", -3.0, -1.0)):
    wl = W.make_conv(B=B, H=H, L=L, N=N, dtype="f32", seed=seed, dt_range=dt)
    A = O.discretize(wl.dt, wl.lam)
    return wl, A, O.as_complex(wl.Bp), O.as_complex(wl.Cp)


def test_filter_exp_form_vs_repeated_product():
    wl, A, Bc, Cc = _small(L=300)
    f1 = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, wl.L)
    f2 = O.ssm_filter_from_A(A, Bc, Cc, wl.L)
    assert O.row_rel_err(f1, f2) < 1e-11


def test_filter_spectrum_closed_form():
    """FFT_{2L} of the zero-padded filter equals the finite geometric sum
    sum_n c_n (1 - A^L z^-L)/(1 - A z^-1) + conj pair, z = exp(2 pi i m / 2L)."""
    wl, A, Bc, Cc = _small(L=128, N=6)
    L = wl.L
    f = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, L)
    M = 2 * L
    F = np.fft.fft(np.concatenate([f, np.zeros_like(f)], axis=1), axis=1)
    zinv = np.exp(-2j * np.pi * np.arange(M) / M)
    c = Cc * Bc
    for h in range(wl.H):
        a = A[h][:, None]
        term = c[h][:, None] * (1 - a ** L * zinv[None] ** L) / (1 - a * zinv[None])
        ac = np.conj(A[h])[:, None]
        term2 = np.conj(c[h])[:, None] * (1 - ac ** L * zinv[None] ** L) / (1 - ac * zinv[None])
        closed = np.sum(term + term2, axis=0)
        assert np.max(np.abs(F[h] - closed)) < 1e-9 * np.max(np.abs(closed))


def test_special_cases():
    wl, A, Bc, Cc = _small(L=50)
    u = wl.u
    f0 = O.ssm_filter(wl.dt, wl.lam, wl.Bp, np.zeros_like(wl.Cp), wl.L)
    assert np.all(f0 == 0)
    y = O.causal_conv_direct(u, f0, wl.D)
    assert np.array_equal(y, wl.D.astype(np.float64)[None, :, None] * u)  # C = 0 -> y = D u
    # A = 0 -> f = [2 Re(CB), 0, 0, ...]
    fz = O.ssm_filter_from_A(np.zeros_like(A), Bc, Cc, 10)
    assert np.allclose(fz[:, 0], 2 * np.real(np.sum(Cc * Bc, axis=1)), atol=1e-15)
    assert np.all(fz[:, 1:] == 0)
    # N = 1, real a: f = 2 a^k
    a = 0.93
    fr = O.ssm_filter_from_A(np.array([[a + 0j]]), np.array([[1 + 0j]]), np.array([[1 + 0j]]), 40)
    assert np.allclose(fr[0], 2 * a ** np.arange(40), rtol=1e-13)


def test_impulse_response_equals_filter():
    wl, A, Bc, Cc = _small(L=200)
    u = np.zeros((1, wl.H, wl.L))
    u[0, :, 0] = 1.0
    f = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, wl.L)
    y, _ = O.ssm_recurrence(u, A, Bc, Cc, wl.D)
    want = f.copy()
    want[:, 0] += wl.D
    assert O.row_rel_err(y[0], want) < 1e-12
    yc, _ = cref.ssm_recurrence(u, A, Bc, Cc, wl.D)
    assert O.row_rel_err(yc[0], want) < 1e-12


def test_conv_equals_recurrence():
    for dt in [("loguniform", -3.0, -1.0), ("split", (-3.0, -2.9), (-1.1, -1.0))]:
        wl, A, Bc, Cc = _small(L=512, H=4, dt=dt)
        f = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, wl.L)
        y1 = O.causal_conv_direct(wl.u, f, wl.D)
        y2, _ = O.ssm_recurrence(wl.u, A, Bc, Cc, wl.D)
        assert O.row_rel_err(y1, y2) < 1e-10
        y3 = cref.causal_conv(wl.u, f, wl.D)
        assert O.row_rel_err(y3, y1) < 1e-13


def test_linearity():
    wl, A, Bc, Cc = _small(L=128)
    f = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, wl.L)
    rng = np.random.default_rng(5)
    u1 = rng.normal(size=wl.u.shape)
    u2 = rng.normal(size=wl.u.shape)
    al, be = 0.7, -1.3
    lhs = O.causal_conv_direct(al * u1 + be * u2, f, wl.D)
    rhs = al * O.causal_conv_direct(u1, f, wl.D) + be * O.causal_conv_direct(u2, f, wl.D)
    assert O.row_rel_err(lhs, rhs) < 1e-12


def test_shift_equivariance_bit_exact_zeros():
    wl, A, Bc, Cc = _small(L=96, B=1)
    f = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, wl.L)
    s = 17
    u = np.zeros((1, wl.H, wl.L))
    u[0, :, s:] = wl.u[0, :, : wl.L - s]
    y = O.causal_conv_direct(u, f, wl.D)
    assert np.all(y[0, :, :s] == 0.0)
    y0 = O.causal_conv_direct(wl.u, f, wl.D)
    assert O.row_rel_err(y[0, :, s:], y0[0, :, : wl.L - s]) < 1e-13
    # delayed impulse: output is f shifted by s
    d = np.zeros((1, wl.H, wl.L))
    d[0, :, s] = 1.0
    yd = O.causal_conv_direct(d, f, np.zeros(wl.H))
    assert np.all(yd[0, :, :s] == 0.0)
    assert np.array_equal(yd[0, :, s:], f[:, : wl.L - s])


def test_library_fft_crosscheck():
    wl, A, Bc, Cc = _small(L=256)
    f = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, wl.L)
    L = wl.L
    U = np.fft.rfft(wl.u, n=2 * L, axis=-1)
    F = np.fft.rfft(f, n=2 * L, axis=-1)
    yf = np.fft.irfft(U * F[None], n=2 * L, axis=-1)[..., :L] + wl.D[None, :, None] * wl.u
    y = O.causal_conv_direct(wl.u, f, wl.D)
    assert O.row_rel_err(yf, y) < 1e-12


def test_statepass_equals_unchunked():
    wl, A, Bc, Cc = _small(L=256, H=3, B=2)
    y_ref, x_ref = O.ssm_recurrence(wl.u, A, Bc, Cc, wl.D)
    for T in (16, 64, 256):
        y, x = O.statepass_chunked(wl.u, A, Bc, Cc, wl.D, T)
        assert O.row_rel_err(y, y_ref) < 1e-10, T
        assert np.max(np.abs(x - x_ref)) < 1e-10 * np.max(np.abs(x_ref))
    # chunk = L reduces to the plain convolution
    f = O.ssm_filter_from_A(A, Bc, Cc, wl.L)
    yT, _ = O.statepass_chunked(wl.u, A, Bc, Cc, wl.D, wl.L)
    assert O.row_rel_err(yT, O.causal_conv_direct(wl.u, f, wl.D)) < 1e-12
    # state_out of call 1 fed as state_in of call 2 == one call on the concatenation
    h = wl.L // 2
    y1, x1 = O.statepass_chunked(wl.u[..., :h], A, Bc, Cc, wl.D, 32)
    y2, x2 = O.statepass_chunked(wl.u[..., h:], A, Bc, Cc, wl.D, 32, x0=x1)
    assert O.row_rel_err(np.concatenate([y1, y2], -1), y_ref) < 1e-10
    assert np.max(np.abs(x2 - x_ref)) < 1e-10 * np.max(np.abs(x_ref))
    # a nonzero initial state reaches y through A^(t+1): compare with the recurrence
    x0 = np.random.default_rng(3).normal(size=x_ref.shape) + 1j
    y3, _ = O.statepass_chunked(wl.u, A, Bc, Cc, wl.D, 64, x0=x0)
    y4, _ = O.ssm_recurrence(wl.u, A, Bc, Cc, wl.D, x0=x0)
    assert O.row_rel_err(y3, y4) < 1e-10
    y5, _ = cref.ssm_recurrence(wl.u, A, Bc, Cc, wl.D, x0=x0)
    assert O.row_rel_err(y5, y4) < 1e-12


def test_shift_ssm_impulse_gives_taps():
    rng = np.random.default_rng(2)
    Cs = rng.normal(size=(5, 4))
    k = np.zeros((1, 10, 5))
    k[0, 3, :] = 1.0
    out = O.shift_ssm(k, Cs)
    assert np.all(out[0, :3] == 0)
    assert np.array_equal(out[0, 3:7].T, Cs)
    assert np.all(out[0, 7:] == 0)


def _mixer_small(hd=3, heads=2, L=12, B=2, seed=9):
    mw = W.make_mixer(B=B, L=L, heads=heads, head_dim=hd, N=4, shift_len=4, dtype="f32", seed=seed)
    f = O.ssm_filter(mw.dt, mw.lam, mw.Bp, mw.Cp, L)
    return mw, f


def test_mixer_forms_agree():
    mw, f = _mixer_small()
    o1 = O.h3_mixer_outer(mw.q, mw.k, mw.v, mw.Cshift, f, mw.D, mw.heads)
    o2 = O.h3_mixer_toeplitz(mw.q, mw.k, mw.v, mw.Cshift, f, mw.D, mw.heads)
    assert np.max(np.abs(o1 - o2)) < 1e-12 * np.max(np.abs(o1))


def test_mixer_hd1_reduces_to_gated_conv():
    mw, f = _mixer_small(hd=1, heads=3)
    o = O.h3_mixer_outer(mw.q, mw.k, mw.v, mw.Cshift, f, mw.D, mw.heads)
    kt = O.shift_ssm(mw.k, mw.Cshift)
    x = np.transpose(kt * mw.v, (0, 2, 1))                       # B x C x L
    y = O.causal_conv_direct(x, f, mw.D)
    want = mw.q * np.transpose(y, (0, 2, 1))
    assert np.max(np.abs(o - want)) < 1e-13 * np.max(np.abs(want))


def test_mixer_delta_filter():
    """f = delta (A = 0, C B = 1/2) -> o_j = (D + 1) (q . k~) v_j."""
    mw, _ = _mixer_small()
    heads, L = mw.heads, mw.L
    A = np.zeros((heads, 1), dtype=np.complex128)
    f = O.ssm_filter_from_A(A, np.ones((heads, 1)), 0.5 * np.ones((heads, 1)), L)
    assert np.all(f[:, 0] == 1.0) and np.all(f[:, 1:] == 0)
    o = O.h3_mixer_outer(mw.q, mw.k, mw.v, mw.Cshift, f, mw.D, heads)
    kt = O.shift_ssm(mw.k, mw.Cshift)
    hd = mw.head_dim
    for h in range(heads):
        sl = slice(h * hd, (h + 1) * hd)
        qk = np.sum(mw.q[:, :, sl] * kt[:, :, sl], axis=-1, keepdims=True)
        want = (np.float64(mw.D[h]) + 1.0) * qk * mw.v[:, :, sl]
        assert np.max(np.abs(o[:, :, sl] - want)) < 1e-13 * np.max(np.abs(want))


# ---------------------------------------------------------------- parity metric
def test_golden_row_rel_err(golden):
    """The parity metric against hand-worked values: per-row max-norm, max over rows."""
    g = golden("hand_worked_row_rel_err.txt")
    ref = np.array(g["ref"]).reshape(3, 3)
    y = np.array(g["y"]).reshape(3, 3)
    for r in range(3):
        assert O.row_rel_err(y[r:r + 1], ref[r:r + 1]) == pytest.approx(g["row_err"][r], rel=1e-15)
    assert O.row_rel_err(y, ref) == pytest.approx(g["metric"][0], rel=1e-15)
    assert O.row_rel_err(y[2:], ref[2:]) == pytest.approx(g["zero_row_only"][0], rel=1e-15)
    # 3-d arrays (B x H x L) reduce along the last axis the same way
    assert O.row_rel_err(y.reshape(1, 3, 3), ref.reshape(1, 3, 3)) == pytest.approx(g["metric"][0], rel=1e-15)
    # a tolerance check built on it must separate the rows: scaling one row's error up
    # by 10x moves the metric, scaling the quiet row does not
    y2 = y.copy()
    y2[1, 1] = 20.0
    assert O.row_rel_err(y2, ref) == pytest.approx(0.2, rel=1e-15)


def test_row_rel_err_planted_mistakes(golden):
    """Plausible mistakes in the metric (made here, on copies) must miss the golden value."""
    g = golden("hand_worked_row_rel_err.txt")
    ref = np.array(g["ref"]).reshape(3, 3)
    y = np.array(g["y"]).reshape(3, 3)
    want = g["metric"][0]
    global_den = float(np.max(np.abs(y - ref)) / np.max(np.abs(ref)))
    wrong_axis = float(np.max(np.max(np.abs(y - ref), axis=0) / np.maximum(np.max(np.abs(ref), axis=0), 1e-300)))
    per_row = np.max(np.abs(y - ref), axis=-1) / np.where(np.max(np.abs(ref), axis=-1) == 0, 1.0,
                                                         np.max(np.abs(ref), axis=-1))
    mean_rows = float(np.mean(per_row))
    for bad in (global_den, wrong_axis, mean_rows):
        assert abs(bad - want) > 1e-3, bad
    assert O.row_rel_err(y, ref) == pytest.approx(want, rel=1e-15)


# ---------------------------------------------------------------- backward pass
def test_golden_conv_bwd(golden):
    g = golden("hand_worked_conv_bwd.txt")
    u = np.array(g["u"]).reshape(1, 1, -1)
    f = np.array(g["f"]).reshape(1, -1)
    D = np.array(g["D"])
    dy = np.array(g["dy"]).reshape(1, 1, -1)
    assert np.allclose(O.causal_conv_direct(u, f, D)[0, 0], g["y"], rtol=0, atol=1e-15)
    du, df, dD = O.causal_conv_bwd(dy, u, f, D)
    assert np.array_equal(du[0, 0], np.array(g["du"]))
    assert np.array_equal(df[0], np.array(g["df"]))
    assert dD[0] == g["dD"][0]


def test_conv_bwd_by_linearity_brute_force():
    """y is linear in u and jointly linear in (f, D), so each gradient entry is
    exactly <dy, y(basis vector)>: brute force over every entry on a tiny case."""
    rng = np.random.default_rng(11)
    B, H, L = 2, 2, 7
    u = rng.normal(size=(B, H, L))
    f = rng.normal(size=(H, L))
    D = rng.normal(size=H)
    dy = rng.normal(size=(B, H, L))
    du, df, dD = O.causal_conv_bwd(dy, u, f, D)
    for b in range(B):
        for h in range(H):
            for s in range(L):
                e = np.zeros_like(u)
                e[b, h, s] = 1.0
                assert abs(np.sum(dy * O.causal_conv_direct(e, f, D)) - du[b, h, s]) < 1e-12
    for h in range(H):
        for k in range(L):
            e = np.zeros_like(f)
            e[h, k] = 1.0
            assert abs(np.sum(dy * O.causal_conv_direct(u, e, np.zeros(H))) - df[h, k]) < 1e-12
        e = np.zeros(H)
        e[h] = 1.0
        assert abs(np.sum(dy * O.causal_conv_direct(u, np.zeros_like(f), e)) - dD[h]) < 1e-12


def test_conv_bwd_adjoint_and_fft_route():
    rng = np.random.default_rng(12)
    B, H, L = 3, 4, 64
    u = rng.normal(size=(B, H, L))
    f = rng.normal(size=(H, L)) * np.exp(-np.arange(L) / 9.0)
    D = rng.normal(size=H)
    dy = rng.normal(size=(B, H, L))
    du, df, dD = O.causal_conv_bwd(dy, u, f, D)
    lhs = np.sum(dy * O.causal_conv_direct(u, f, D))
    assert abs(lhs - np.sum(du * u)) < 1e-10 * abs(lhs)
    assert abs(lhs - (np.sum(df * f) + np.sum(dD * D))) < 1e-10 * abs(lhs)
    # library route: with 2L zero padding, du is the circular correlation
    # irfft(conj(F) DY) and df the batch sum of irfft(DY conj(U)), cropped to L
    M = 2 * L
    F = np.fft.rfft(f, M)
    U = np.fft.rfft(u, M)
    DY = np.fft.rfft(dy, M)
    du_fft = np.fft.irfft(np.conj(F)[None] * DY, M)[..., :L] + D[None, :, None] * dy
    df_fft = np.sum(np.fft.irfft(DY * np.conj(U), M)[..., :L], axis=0)
    assert np.max(np.abs(du_fft - du)) < 1e-12 * np.max(np.abs(du))
    assert np.max(np.abs(df_fft - df)) < 1e-12 * np.max(np.abs(df))


def test_conv_bwd_planted_mistakes(golden):
    g = golden("hand_worked_conv_bwd.txt")
    u = np.array(g["u"])
    f = np.array(g["f"])
    dy = np.array(g["dy"])
    D = g["D"][0]
    L = len(u)
    # causal instead of anti-causal du
    du_causal = np.convolve(dy, f)[:L] + D * dy
    assert not np.allclose(du_causal, g["du"])
    # D term dropped from du
    du_noD = np.correlate(dy, f, mode="full")[L - 1:]
    assert not np.allclose(du_noD, g["du"])
    # df with the lag sign flipped (u leading dy)
    df_flip = np.correlate(u, dy, mode="full")[L - 1:]
    assert not np.allclose(df_flip, g["df"])


def test_mixer_recurrent_equals_outer_form():
    """The token-by-token recurrent mixer (the decode path) equals the
    convolutional outer-product form, whose filter is f = 2 Re(C A^k B)."""
    rng = np.random.default_rng(13)
    Bn, L, heads, hd, N, S = 2, 9, 2, 3, 4, 3
    q, k, v = (rng.normal(size=(Bn, L, heads * hd)) for _ in range(3))
    Cs = rng.normal(size=(heads * hd, S))
    A = 0.9 * np.exp(1j * rng.uniform(0, np.pi, size=(heads, N)))
    Bc = rng.normal(size=(heads, N)) + 1j * rng.normal(size=(heads, N))
    Cc = rng.normal(size=(heads, N)) + 1j * rng.normal(size=(heads, N))
    D = rng.normal(size=heads)
    o_rec = O.h3_mixer_recurrent(q, k, v, Cs, A, Bc, Cc, D, heads)
    f = O.ssm_filter_from_A(A, Bc, Cc, L)
    o_conv = O.h3_mixer_outer(q, k, v, Cs, f, D, heads)
    assert np.max(np.abs(o_rec - o_conv)) < 1e-12 * np.max(np.abs(o_conv))
    # planted: read the output before the state update (x_{t-1} instead of x_t)
    o_lag = O.h3_mixer_outer(q, k, v, Cs, np.concatenate([np.zeros((heads, 1)), f[:, :-1]], 1), D, heads)
    assert np.max(np.abs(o_lag - o_conv)) > 1e-3 * np.max(np.abs(o_conv))


def test_statepass_bwd_by_linearity_brute_force():
    """The loss <dy, y> + Re<G, state_out> is linear in (u, state_in): every
    gradient entry is the loss at a basis vector (through the pinned
    recurrence), including the imaginary directions of the state."""
    rng = np.random.default_rng(21)
    B, H, L, N = 1, 2, 9, 3
    A = 0.9 * np.exp(1j * rng.uniform(0, np.pi, size=(H, N)))
    Bc = rng.normal(size=(H, N)) + 1j * rng.normal(size=(H, N))
    Cc = rng.normal(size=(H, N)) + 1j * rng.normal(size=(H, N))
    D = rng.normal(size=H)
    dy = rng.normal(size=(B, H, L))
    G = rng.normal(size=(B, H, N)) + 1j * rng.normal(size=(B, H, N))
    du, dsin = O.statepass_bwd(dy, A, Bc, Cc, D, dstate_out=G)

    def loss(u, x0):
        y, x = O.ssm_recurrence(u, A, Bc, Cc, D, x0=x0)
        return np.sum(dy * y) + np.sum(np.real(np.conj(G) * x))
    zero_u = np.zeros((B, H, L))
    zero_x = np.zeros((B, H, N), dtype=np.complex128)
    for h in range(H):
        for t in range(L):
            e = zero_u.copy()
            e[0, h, t] = 1.0
            assert abs(loss(e, zero_x) - du[0, h, t]) < 1e-12
        for n in range(N):
            for unit, part in ((1.0, "re"), (1j, "im")):
                x0 = zero_x.copy()
                x0[0, h, n] = unit
                want = dsin[0, h, n].real if part == "re" else dsin[0, h, n].imag
                assert abs(loss(zero_u, x0) - want) < 1e-12


def test_statepass_bwd_without_state_grad_is_conv_bwd():
    """With no gradient on the final state, du is the convolution's input
    gradient (anti-causal correlation with f plus D dy)."""
    rng = np.random.default_rng(22)
    wl, A, Bc, Cc = _small(L=48, H=3, B=2)
    dy = rng.normal(size=wl.u.shape)
    du, _ = O.statepass_bwd(dy, A, Bc, Cc, wl.D)
    f = O.ssm_filter_from_A(A, Bc, Cc, wl.L)
    du2, _, _ = O.causal_conv_bwd(dy, wl.u, f, wl.D)
    assert np.max(np.abs(du - du2)) < 1e-10 * np.max(np.abs(du2))


# ---------------------------------------------------------------- planted mistakes
def test_pins_catch_planted_mistakes(golden):
    """Mutated copies of oracle steps (made here, on the CPU) must fail a pin."""
    g = golden("hand_worked_real_n1.txt")
    u = np.array(g["u"]).reshape(1, 1, -1)
    f = np.array(g["f"]).reshape(1, -1)
    # 1. dropped D term
    y_noD = O.causal_conv_direct(u, f, np.zeros(1))
    assert not np.allclose(y_noD[0, 0], g["y"])
    # 2. off-by-one causal index (y[t] uses u up to t-1)
    y_shift = np.concatenate([[0.0], O.causal_conv_direct(u, f, np.zeros(1))[0, 0, :-1]]) + 0.25 * u[0, 0]
    assert not np.allclose(y_shift, g["y"])
    # 3. conj(C) instead of C in the filter
    gr = golden("hand_worked_complex_rotation.txt")
    A = np.array([[_cplx(gr["A"])]])
    fbad = O.ssm_filter_from_A(A, np.array([[1 + 0j]]), np.conj(np.array([[_cplx(gr["C"])]])), 8)
    assert not np.allclose(fbad[0], gr["f"])
    # 4. state correction through A^t instead of A^(t+1)
    wl, A, Bc, Cc = _small(L=64, H=2, B=1)
    y_ref, _ = O.ssm_recurrence(wl.u, A, Bc, Cc, wl.D)
    T = 16
    fT = O.ssm_filter_from_A(A, Bc, Cc, T)
    x = np.zeros((1, wl.H, A.shape[1]), dtype=np.complex128)
    yb = np.empty_like(wl.u)
    for c in range(wl.L // T):
        uc = wl.u[:, :, c * T:(c + 1) * T]
        p = A[:, :, None] ** np.arange(T)[None, None, :]            # wrong: A^t
        yb[:, :, c * T:(c + 1) * T] = O.causal_conv_direct(uc, fT, wl.D) + \
            2 * np.real(np.einsum("hn,hnt,bhn->bht", Cc, p, x))
        Mux = (A[:, :, None] ** (T - 1 - np.arange(T))[None, None, :]) * Bc[:, :, None]
        x = (A ** T)[None] * x + np.einsum("hni,bhi->bhn", Mux, uc)
    assert O.row_rel_err(yb, y_ref) > 1e-3
    # 5. shift taps reversed
    gs = golden("hand_worked_shift_ssm.txt")
    out = O.shift_ssm(np.array(gs["k"]).reshape(1, -1, 1), np.array(gs["Cshift"])[::-1].reshape(1, -1))
    assert not np.array_equal(out[0, :, 0], np.array(gs["ktilde"]))
    # 6. q and k~ swapped in the mixer (q is not shifted; k is)
    gm = golden("hand_worked_h3_mixer.txt")
    q = np.array(gm["q"]).reshape(1, 2, 2)
    k = np.array(gm["k"]).reshape(1, 2, 2)
    v = np.array(gm["v"]).reshape(1, 2, 2)
    Cs = np.array([[1.0, 0, 0, 0]] * 2)
    obad = O.h3_mixer_outer(k, q, v, Cs, np.array([gm["f"]]), np.array(gm["D"]), 1)
    assert not np.allclose(obad.ravel(), gm["o"])


# ---------------------------------------------------------------- input module sanity
def test_workload_rounding_matches_torch():
    import torch
    x = np.random.default_rng(0).normal(size=10000) * 3
    for dt, td in (("f16", torch.float16), ("bf16", torch.bfloat16), ("f32", torch.float32)):
        want = torch.tensor(x, dtype=torch.float64).to(torch.float32).to(td).to(torch.float64).numpy()
        assert np.array_equal(W.round_to(x, dt), want), dt


def test_workloads_deterministic():
    a = W.make("cfg1_conv_f32_B1_H4_L256")
    b = W.make("cfg1_conv_f32_B1_H4_L256")
    assert np.array_equal(a.u, b.u) and np.array_equal(a.dt, b.dt)
    assert a.u.shape == (1, 4, 256) and a.N == 32
    assert np.all((a.dt >= 1e-3 * 0.999) & (a.dt <= 1e-1 * 1.001))
    c3 = W.make("cfg3_conv_bf16_B4_H1024_L8192", B=1, L=16)
    assert np.all(c3.dt[:512] < 1.3e-3) and np.all(c3.dt[512:] > 0.079)
