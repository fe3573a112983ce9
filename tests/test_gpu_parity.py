"""GPU parity: the CUDA path (called through the C ABI) against the fp64 oracle
on the same seeded inputs.

Tolerance (per-row max-norm relative error, max over rows): 1e-4 for fp32
I/O, 2e-2 for fp16 / bf16 I/O with fp32 accumulation.  Every expected value
comes from ``oracle/``; filters passed to ``fftconv_fwd`` are the oracle's
fp64 filters rounded to fp32 (that rounded array is the input both sides see).
"""
import numpy as np
import pytest
import torch

from fft_long_convolution_flashconv_b200 import api
from fft_long_convolution_flashconv_b200 import workloads as W
from oracle import cref
from oracle import ssm_oracle as O

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "f16": 2e-2, "bf16": 2e-2}
TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def dev(x, dtype="f32"):
    return torch.tensor(np.asarray(x), dtype=torch.float64).to(TORCH_DT[dtype]).cuda().contiguous()


def host(t):
    return t.detach().to(torch.float64).cpu().numpy()


def params(wl):
    return (dev(wl.dt), dev(wl.lam), dev(wl.Bp), dev(wl.Cp), dev(wl.D))


def oracle_A(wl, hs=None):
    hs = slice(None) if hs is None else hs
    return (O.discretize(wl.dt[hs], wl.lam[hs]), O.as_complex(wl.Bp[hs]), O.as_complex(wl.Cp[hs]))


# ------------------------------------------------------------------ A1 filter generation
@pytest.mark.parametrize("H,N,L,dt", [
    (4, 32, 256, ("loguniform", -3.0, -1.0)),
    (5, 64, 3000, ("loguniform", -3.0, -1.0)),          # ragged: 2 tiles, partial 64-block
    (6, 64, 8192, ("split", (-3.0, -2.9), (-1.1, -1.0))),
    (3, 64, 65536, ("loguniform", -3.0, -2.5)),         # long, slowly decaying: phase reduction
    (2, 1, 100, ("loguniform", -1.0, -1.0)),            # N = 1 (real A for n = 0)
    (3, 64, 1001, ("loguniform", -3.0, -1.0)),          # L % 16 != 0: ragged last row, scalar stores
    (2, 96, 3000, ("loguniform", -3.0, -1.0)),          # N > 64: CUDA-core generator
    (3, 64, 12345, ("loguniform", -3.0, -1.0)),         # 64-tap rows: two units, ragged, scalar stores
    (2, 32, 20000, ("loguniform", -3.0, -2.0)),         # 64-tap rows: three units over two CTAs
    (4, 64, 4100, ("loguniform", -3.0, -1.0)),          # 64-tap rows: one partial unit
    (2, 1, 5000, ("loguniform", -2.0, -1.0)),           # 64-tap rows, N = 1
])
def test_ssm_kernel_gen(H, N, L, dt):
    wl = W.make_conv(B=1, H=H, L=8, N=N, dtype="f32", seed=7, dt_range=dt)
    dtt, lam, Bp, Cp, _ = params(wl)
    f = host(api.ssm_kernel_gen(dtt, lam, Bp, Cp, L))
    ref = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, L)
    assert O.row_rel_err(f, ref) < 1e-5


# ------------------------------------------------------------------ A2-A4 fused conv, all plans
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("L", [16, 32, 64, 128, 256, 512, 1024, 2048, 4096, 8192])
def test_fftconv_all_sizes(L, dtype):
    B, H = 3, 5  # odd B: one row has no partner; H = 5: partial channel groups
    wl = W.make_conv(B=B, H=H, L=L, N=16, dtype=dtype, seed=L, dt_range=("loguniform", -3.0, -1.0))
    f32 = W.round_to(O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, L), "f32")
    u = dev(wl.u, dtype)
    y = host(api.fftconv_fwd(u, dev(f32), dev(wl.D)))
    ref = cref.causal_conv(wl.u, f32, wl.D.astype(np.float64))
    err = O.row_rel_err(y.reshape(B * H, L), ref.reshape(B * H, L))
    assert err < TOL[dtype], err


@pytest.mark.parametrize("B,H,dtype", [(10, 3, "f16"), (3, 4, "bf16"), (4, 300, "f16"), (7, 2, "bf16"),
                                       (5, 1, "f16"), (2, 5, "bf16")])
def test_fftconv_tensor_core_batches(B, H, dtype):
    """L = 1024 fp16/bf16 with B >= 3 runs the tensor-core block FFT (rounds of
    three row pairs that may span two channels): several pairs per channel
    (B = 10), odd B (a pair without its second row), more rounds than SMs
    (H = 300), a single channel; B = 2 takes the CUDA-core path."""
    L = 1024
    wl = W.make_conv(B=B, H=H, L=L, N=16, dtype=dtype, seed=B * 1000 + H, dt_range=("loguniform", -3.0, -1.0))
    f32 = W.round_to(O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, L), "f32")
    y = host(api.fftconv_fwd(dev(wl.u, dtype), dev(f32), dev(wl.D)))
    ref = cref.causal_conv(wl.u, f32, wl.D.astype(np.float64))
    assert O.row_rel_err(y.reshape(B * H, L), ref.reshape(B * H, L)) < TOL[dtype]


def test_fftconv_arbitrary_filter_and_impulse_alignment():
    """A non-SSM filter; impulses at several offsets land exactly where the
    causal index bookkeeping says (argmax position is an integer check)."""
    L, H = 1024, 3
    rng = np.random.default_rng(0)
    f = rng.normal(size=(H, L)) * np.exp(-np.arange(L) / 300.0)[None]
    f = W.round_to(f, "f32")
    shifts = [0, 1, 17, 511, 1023]
    u = np.zeros((len(shifts), H, L))
    for i, s in enumerate(shifts):
        u[i, :, s] = 1.0
    D = np.zeros(H)
    y = host(api.fftconv_fwd(dev(u), dev(f), dev(D)))
    for i, s in enumerate(shifts):
        for h in range(H):
            want = np.zeros(L)
            want[s:] = f[h, : L - s]
            assert np.max(np.abs(y[i, h] - want)) < 1e-5 * np.max(np.abs(f[h]))
            assert int(np.argmax(np.abs(y[i, h]))) == s + int(np.argmax(np.abs(f[h, : L - s])))
            assert np.max(np.abs(y[i, h, :s])) < 1e-5 * np.max(np.abs(f[h])) if s else True


@pytest.mark.parametrize("L,N,dtype", [(1024, 65, "f32"), (2048, 40, "f16"), (4096, 17, "bf16"), (8192, 70, "f32"),
                                       (512, 64, "f16")])
def test_ssm_conv_fused_generation(L, N, dtype):
    """ssm_conv_fwd: for L >= 1024 and N > 64 the filter is generated inside
    the convolution kernel (several mode blocks, odd B, channels split across
    CTAs); otherwise the tensor-core generator runs first."""
    B, H = 3, 7
    wl = W.make_conv(B=B, H=H, L=L, N=N, dtype=dtype, seed=N + L, dt_range=("loguniform", -3.0, -1.0))
    dtt, lam, Bp, Cp, D = params(wl)
    y = host(api.ssm_conv_fwd(dev(wl.u, dtype), dtt, lam, Bp, Cp, D))
    f = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, L)
    ref = cref.causal_conv(wl.u, f, wl.D.astype(np.float64))
    assert O.row_rel_err(y.reshape(-1, L), ref.reshape(-1, L)) < TOL[dtype]


def test_ssm_conv_cfg1_full():
    wl = W.make("cfg1_conv_f32_B1_H4_L256")
    dtt, lam, Bp, Cp, D = params(wl)
    y = host(api.ssm_conv_fwd(dev(wl.u), dtt, lam, Bp, Cp, D))
    f = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, wl.L)
    ref = O.causal_conv_direct(wl.u, f, wl.D)
    assert O.row_rel_err(y.reshape(-1, wl.L), ref.reshape(-1, wl.L)) < 1e-4
    A, Bc, Cc = oracle_A(wl)
    ref2, _ = O.ssm_recurrence(wl.u, A, Bc, Cc, wl.D)
    assert O.row_rel_err(y.reshape(-1, wl.L), ref2.reshape(-1, wl.L)) < 1e-4


def test_ssm_conv_cfg2_full_all_rows():
    """Full 8 x 768 x 1024 fp16 workload, filter generated on the device each
    call; every row checked against the C oracle."""
    wl = W.make("cfg2_conv_f16_B8_H768_L1024")
    dtt, lam, Bp, Cp, D = params(wl)
    u = dev(wl.u, "f16")
    y1 = api.ssm_conv_fwd(u, dtt, lam, Bp, Cp, D)
    y2 = api.ssm_conv_fwd(u, dtt, lam, Bp, Cp, D)   # a second call gives the same bits
    assert torch.equal(y1, y2)
    y = host(y1)
    f = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, wl.L)
    ref = cref.causal_conv(wl.u, f, wl.D.astype(np.float64))
    assert O.row_rel_err(y.reshape(-1, wl.L), ref.reshape(-1, wl.L)) < 2e-2


def test_ssm_conv_cfg3_full_sampled_rows():
    wl = W.make("cfg3_conv_bf16_B4_H1024_L8192")
    dtt, lam, Bp, Cp, D = params(wl)
    y = api.ssm_conv_fwd(dev(wl.u, "bf16"), dtt, lam, Bp, Cp, D)
    rng = np.random.default_rng(123)
    hs = np.unique(np.concatenate([rng.choice(512, 12, replace=False), 512 + rng.choice(512, 12, replace=False),
                                   [0, 511, 512, 1023]]))
    bs = rng.integers(0, wl.B, size=len(hs))
    f = O.ssm_filter(wl.dt[hs], wl.lam[hs], wl.Bp[hs], wl.Cp[hs], wl.L)
    u_s = wl.u[bs, hs][:, None, :]                                         # rows x 1 x L
    yh = host(y[torch.as_tensor(bs).cuda(), torch.as_tensor(hs).cuda()])
    err = 0.0
    for i in range(len(hs)):
        ref = cref.causal_conv(u_s[i:i + 1], f[i:i + 1], wl.D[hs[i]:hs[i] + 1].astype(np.float64))
        err = max(err, O.row_rel_err(yh[i], ref[0, 0]))
    assert err < 2e-2, err


# ------------------------------------------------------------------ A6-A9 state passing
@pytest.mark.parametrize("B,H,L,T,N,dtype", [
    (2, 3, 512, 64, 16, "f32"),
    (1, 3, 192, 64, 16, "f32"),     # odd number of chunk-rows (unpaired chunk)
    (2, 2, 256, 256, 8, "f32"),     # chunk == L
    (1, 2, 256, 16, 8, "f32"),      # smallest chunk
    (2, 3, 1024, 256, 32, "f16"),     # 16-bit I/O on the CUDA-core tail, 4 chunks
    # tensor-core tail (16-bit I/O, T in {2048, 4096, 8192}, N <= 64)
    (1, 2, 16384, 8192, 64, "bf16"),
    (2, 3, 8192, 2048, 33, "f16"),      # ragged mode count, 4 chunks
    (1, 2, 16384, 4096, 64, "bf16"),
    (1, 3, 2048, 2048, 1, "bf16"),      # one chunk, one mode: correction from state_in only
    (2, 2, 8192, 2048, 64, "f16-nox0"),  # no initial state: the first chunk is not corrected
])
def test_statepass_small(B, H, L, T, N, dtype):
    with_x0 = not dtype.endswith("-nox0")
    dtype = dtype.replace("-nox0", "")
    wl = W.make_conv(B=B, H=H, L=L, N=N, dtype=dtype, seed=L + T, dt_range=("loguniform", -3.0, -1.0))
    dtt, lam, Bp, Cp, D = params(wl)
    rng = np.random.default_rng(1)
    x0 = rng.normal(size=(B, H, N)) + 1j * rng.normal(size=(B, H, N))
    if not with_x0:
        x0 = np.zeros_like(x0)
    x0_t = torch.view_as_real(torch.tensor(x0.astype(np.complex64))).cuda().contiguous()
    y, xs = api.fftconv_statepass(dev(wl.u, dtype), dtt, lam, Bp, Cp, D, T, state_in=x0_t if with_x0 else None,
                                  return_state=True)
    A, Bc, Cc = oracle_A(wl)
    x0_r = x0.astype(np.complex64).astype(np.complex128)
    ref, xref = cref.ssm_recurrence(wl.u, A, Bc, Cc, wl.D.astype(np.float64), x0=x0_r)
    assert O.row_rel_err(host(y).reshape(-1, L), ref.reshape(-1, L)) < TOL[dtype]
    xg = host(xs)
    xg = xg[..., 0] + 1j * xg[..., 1]
    tol = 1e-4 if dtype == "f32" else 5e-3
    assert np.max(np.abs(xg - xref)) < tol * np.max(np.abs(xref))


def test_statepass_state_composition():
    """state_out of call 1 fed as state_in of call 2 == one call on the whole."""
    B, H, L, T, N = 2, 3, 1024, 128, 16
    wl = W.make_conv(B=B, H=H, L=L, N=N, dtype="f32", seed=5)
    dtt, lam, Bp, Cp, D = params(wl)
    u = dev(wl.u)
    y_all, x_all = api.fftconv_statepass(u, dtt, lam, Bp, Cp, D, T, return_state=True)
    h = L // 2
    y1, x1 = api.fftconv_statepass(u[..., :h].contiguous(), dtt, lam, Bp, Cp, D, T, return_state=True)
    y2, x2 = api.fftconv_statepass(u[..., h:].contiguous(), dtt, lam, Bp, Cp, D, T, state_in=x1,
                                   return_state=True)
    yc = torch.cat([y1, y2], -1)
    assert O.row_rel_err(host(yc).reshape(-1, L), host(y_all).reshape(-1, L)) < 1e-5
    assert torch.allclose(x2, x_all, rtol=1e-4, atol=1e-5 * float(x_all.abs().max()))


def test_statepass_cfg4_full_sampled_rows():
    """Full B=1, H=2560, L=65536, T=8192 fp16; sampled rows against the
    unchunked recurrence."""
    wl = W.make("cfg4_statepass_f16_B1_H2560_L65536_T8192")
    dtt, lam, Bp, Cp, D = params(wl)
    y = api.fftconv_statepass(dev(wl.u, "f16"), dtt, lam, Bp, Cp, D, wl.chunk)
    rng = np.random.default_rng(321)
    hs = np.unique(np.concatenate([rng.choice(wl.H, 14, replace=False), [0, wl.H - 1]]))
    A, Bc, Cc = oracle_A(wl, hs)
    ref, _ = cref.ssm_recurrence(wl.u[:, hs], A, Bc, Cc, wl.D[hs].astype(np.float64))
    yh = host(y[:, torch.as_tensor(hs).cuda()])
    assert O.row_rel_err(yh.reshape(-1, wl.L), ref.reshape(-1, wl.L)) < 2e-2


# ------------------------------------------------------------------ A10-A11 H3 mixer
def _mixer_ref(mw, rows=None, ts=None):
    f = O.ssm_filter(mw.dt, mw.lam, mw.Bp, mw.Cp, mw.L)
    return O.h3_mixer_toeplitz(mw.q, mw.k, mw.v, mw.Cshift, f, mw.D, mw.heads, rows=rows, ts=ts)


def _mixer_gpu(mw):
    return host(api.h3_mixer_fwd(dev(mw.q, mw.dtype), dev(mw.k, mw.dtype), dev(mw.v, mw.dtype), dev(mw.Cshift),
                                 dev(mw.dt), dev(mw.lam), dev(mw.Bp), dev(mw.Cp), dev(mw.D), mw.heads))


def _head_err(o, ref, mw, rows, ts):
    hd = mw.head_dim
    err = 0.0
    for (b, h) in rows:
        a = o[b][ts][:, h * hd:(h + 1) * hd]
        r = ref[b][ts][:, h * hd:(h + 1) * hd]
        err = max(err, float(np.max(np.abs(a - r)) / np.max(np.abs(r))))
    return err


@pytest.mark.parametrize("dtype,L,S,heads", [("f32", 200, 4, 2), ("f16", 130, 4, 2), ("f32", 64, 1, 2),
                                             ("bf16", 96, 3, 2), ("f16", 256, 8, 3), ("bf16", 129, 1, 1),
                                             ("f16", 300, 2, 2), ("f16", 1000, 4, 3), ("bf16", 512, 2, 5),
                                             ("f16", 1024, 1, 1), ("f16", 1, 4, 1), ("bf16", 7, 8, 2),
                                             ("f16", 2048, 3, 1)])
def test_h3_mixer_small(dtype, L, S, heads):
    """fp32 I/O runs the CUDA-core kernel, fp16/bf16 the tensor-core ones
    (128-row tiles: ragged, exact and multi-tile lengths; L a multiple of 8
    takes the warp-specialised kernel, other L the one-tile-per-CTA kernel)."""
    mw = W.make_mixer(B=2, L=L, heads=heads, head_dim=64, N=8, shift_len=S, dtype=dtype, seed=L)
    o = _mixer_gpu(mw)
    ref = _mixer_ref(mw)
    rows = [(b, h) for b in range(2) for h in range(heads)]
    assert _head_err(o, ref, mw, rows, np.arange(L)) < TOL[dtype]


def test_tensor_core_waits_never_timed_out():
    import ctypes
    from fft_long_convolution_flashconv_b200 import _lib
    lib = _lib.load()
    lib.fc_debug_tc_timeouts.restype = ctypes.c_uint
    torch.cuda.synchronize()
    assert lib.fc_debug_tc_timeouts() == 0


def test_h3_mixer_cfg5_full_sampled():
    mw = W.make("cfg5_h3mixer_f16_B8_L2048_d768")
    o = _mixer_gpu(mw)
    rng = np.random.default_rng(77)
    rows = [(0, 0), (7, 11), (3, 5), (int(rng.integers(8)), int(rng.integers(12)))]
    ts = np.unique(np.concatenate([[0, 1, 3, 63, 64, 65, 1023, 2047], rng.choice(2048, 40, replace=False)]))
    ref = _mixer_ref(mw, rows=rows, ts=ts)
    assert _head_err(o, ref, mw, rows, ts) < 2e-2


# ------------------------------------------------------------------ (f)1 backward pass
@pytest.mark.parametrize("B,H,L,dtype", [
    (3, 5, 16, "f32"), (2, 3, 256, "f32"), (3, 4, 1024, "f32"), (2, 3, 8192, "f32"),
    (3, 5, 1024, "f16"), (5, 6, 1024, "bf16"),          # du on the tensor-core conv
    (2, 3, 512, "f16"), (2, 4, 4096, "bf16"), (1, 3, 8192, "f16"),
])
def test_fftconv_bwd(B, H, L, dtype):
    """du, df, dD against the oracle's gradient sums (per-row max-norm; df per
    channel, dD over channels)."""
    wl = W.make_conv(B=B, H=H, L=L, N=16, dtype=dtype, seed=L + B, dt_range=("loguniform", -3.0, -1.0))
    f32 = W.round_to(O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, L), "f32")
    dy = W.round_to(np.random.default_rng(L).normal(size=(B, H, L)), dtype)
    du, df, dD = api.fftconv_bwd(dev(dy, dtype), dev(wl.u, dtype), dev(f32), dev(wl.D))
    rdu, rdf, rdD = O.causal_conv_bwd(dy, wl.u, f32, wl.D)
    assert O.row_rel_err(host(du).reshape(-1, L), rdu.reshape(-1, L)) < TOL[dtype]
    # df and dD come from the 16-bit inputs exactly and are float32 sums: fp32 tolerance
    # scaled by the summation length
    assert O.row_rel_err(host(df), rdf) < 1e-4 * max(1.0, np.log2(L * B) / 4)
    assert np.max(np.abs(host(dD) - rdD)) < 1e-4 * np.max(np.abs(rdD)) * max(1.0, np.log2(L * B) / 4)


def test_fftconv_bwd_parts_and_impulse():
    """du alone and df alone give the same values as the full call; an impulse
    dy at t0 gives du = f reversed in time up to t0 (bit-exact zeros after t0
    are not required: the FFT leaves rounding noise) and df[k] = u[t0 - k]."""
    B, H, L = 2, 3, 512
    wl = W.make_conv(B=B, H=H, L=L, N=16, dtype="f32", seed=77)
    f32 = W.round_to(O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, L), "f32")
    dy = np.zeros((B, H, L))
    t0 = 300
    dy[:, :, t0] = 1.0
    du, df, dD = api.fftconv_bwd(dev(dy), dev(wl.u), dev(f32), dev(wl.D))
    du1, n1, n2 = api.fftconv_bwd(dev(dy), dev(wl.u), dev(f32), dev(wl.D), need_dfilter=False)
    assert n1 is None and n2 is None
    n3, df2, dD2 = api.fftconv_bwd(dev(dy), dev(wl.u), dev(f32), dev(wl.D), need_du=False)
    assert n3 is None
    assert torch.equal(du, du1) and torch.equal(df, df2) and torch.equal(dD, dD2)
    want_du = np.zeros((B, H, L))
    for s in range(t0 + 1):
        want_du[:, :, s] = f32[None, :, t0 - s]
    want_du[:, :, t0] += wl.D[None, :]
    assert np.max(np.abs(host(du) - want_du)) < 1e-5 * np.max(np.abs(want_du))
    want_df = np.zeros((H, L))
    for k in range(t0 + 1):
        want_df[:, k] = wl.u[:, :, t0 - k].sum(0)
    # df is a float32 FFT correlation summed over rows: rounding ~1e-5 relative per transform
    assert np.max(np.abs(host(df) - want_df)) < 1e-4 * np.max(np.abs(want_df))


# ------------------------------------------------------------------ (f)2 recurrent decode
@pytest.mark.parametrize("B,H,N,dtype", [(2, 3, 16, "f32"), (3, 5, 64, "f32"), (2, 3, 200, "f32"),
                                         (1, 2, 700, "f32"), (2, 4, 64, "f16"), (3, 2, 33, "bf16")])
def test_ssm_decode_matches_recurrence(B, H, N, dtype):
    """T tokens in one call, then single tokens chained through the state,
    against the oracle recurrence over the whole sequence (outputs and the
    final state)."""
    L1, L2 = 37, 5
    wl = W.make_conv(B=B, H=H, L=L1 + L2, N=N, dtype=dtype, seed=N + B)
    dtt, lam, Bp, Cp, D = params(wl)
    u = dev(wl.u, dtype)
    x = torch.zeros((B, H, N, 2), dtype=torch.float32, device="cuda")
    ys = [api.ssm_decode_step(u[..., :L1].contiguous(), x, dtt, lam, Bp, Cp, D)]
    for t in range(L1, L1 + L2):
        ys.append(api.ssm_decode_step(u[..., t:t + 1].contiguous(), x, dtt, lam, Bp, Cp, D))
    y = host(torch.cat(ys, -1))
    A, Bc, Cc = oracle_A(wl)
    ref, xref = cref.ssm_recurrence(wl.u, A, Bc, Cc, wl.D.astype(np.float64))
    assert O.row_rel_err(y.reshape(-1, L1 + L2), ref.reshape(-1, L1 + L2)) < TOL[dtype]
    xg = host(x)
    xg = xg[..., 0] + 1j * xg[..., 1]
    assert np.max(np.abs(xg - xref)) < 1e-4 * np.max(np.abs(xref))


@pytest.mark.parametrize("S,dtype", [(4, "f32"), (1, "f32"), (3, "f16"), (8, "bf16")])
def test_h3_mixer_decode_matches_parallel_form(S, dtype):
    """Token-by-token decode of the H3 mixer against the oracle's recurrent
    form (pinned to the convolutional form) on every position."""
    B, L, heads, hd, N = 2, 20, 2, 64, 8
    mw = W.make_mixer(B=B, L=L, heads=heads, head_dim=hd, N=N, shift_len=S, dtype=dtype, seed=40 + S)
    q, k, v = dev(mw.q, dtype), dev(mw.k, dtype), dev(mw.v, dtype)
    Cs, dtt, lam, Bp, Cp, D = dev(mw.Cshift), dev(mw.dt), dev(mw.lam), dev(mw.Bp), dev(mw.Cp), dev(mw.D)
    state = api.h3_decode_state(B, heads, hd, N, "cuda")
    kring = torch.zeros((B, max(S - 1, 1), heads * hd), dtype=q.dtype, device="cuda")
    outs = []
    for t in range(L):
        outs.append(api.h3_mixer_decode_step(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(),
                                             kring, state, Cs, dtt, lam, Bp, Cp, D, heads, t))
    o = host(torch.stack(outs, 1))
    A = O.discretize(mw.dt, mw.lam)
    ref = O.h3_mixer_recurrent(mw.q, mw.k, mw.v, mw.Cshift, A, O.as_complex(mw.Bp), O.as_complex(mw.Cp), mw.D,
                               heads)
    err = 0.0
    for b in range(B):
        for h in range(heads):
            sl = slice(h * hd, (h + 1) * hd)
            err = max(err, float(np.max(np.abs(o[b, :, sl] - ref[b, :, sl])) / np.max(np.abs(ref[b, :, sl]))))
    assert err < TOL[dtype], err


# ------------------------------------------------------------------ tensor-core conv: layout and range edges
@pytest.mark.parametrize("B,H,L,dtype", [(1, 200, 8192, "bf16"), (3, 300, 2048, "f16"), (2, 7, 4096, "bf16"),
                                         (5, 160, 4096, "f16"), (2, 151, 8192, "f16")])
def test_fftconv_tensor_core_long(B, H, L, dtype):
    """L = 2048..8192 block-FFT conv: odd B, B = 1, and more channels than SMs
    (CTA item ranges that start and end inside a channel)."""
    wl = W.make_conv(B=B, H=H, L=L, N=16, dtype=dtype, seed=H + L, dt_range=("loguniform", -3.0, -1.0))
    f32 = W.round_to(O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, L), "f32")
    y = host(api.fftconv_fwd(dev(wl.u, dtype), dev(f32), dev(wl.D)))
    rng = np.random.default_rng(H)
    hs = np.unique(np.concatenate([rng.choice(H, min(H, 24), replace=False), [0, H - 1]]))
    ref = cref.causal_conv(wl.u[:, hs], f32[hs], wl.D[hs].astype(np.float64))
    assert O.row_rel_err(y[:, hs].reshape(-1, L), ref.reshape(-1, L)) < TOL[dtype]


@pytest.mark.parametrize("L,dtype", [(1024, "f16"), (1024, "bf16"), (2048, "bf16"), (8192, "f16")])
def test_fftconv_tensor_core_impulse_alignment(L, dtype):
    """Impulses through the tensor-core paths (odd B, so one row has no pair
    partner): u = delta at t0 gives y = f shifted by t0 plus D delta; the
    argmax of |y - D delta| sits at t0 + argmax|f| and y is ~0 before t0."""
    B, H = 3, 2
    t0s = [0, 1, 15, 16, 511, L - 1]
    rng = np.random.default_rng(L)
    f = np.zeros((H, L))
    f[:, :40] = rng.normal(size=(H, 40))
    f[:, 7] = 5.0  # a unique peak at lag 7
    f32 = W.round_to(f, "f32")
    D = np.array([0.5, -0.25])
    for t0 in t0s:
        u = np.zeros((B, H, L))
        u[:, :, t0] = 1.0
        y = host(api.fftconv_fwd(dev(u, dtype), dev(f32), dev(D)))
        for b in range(B):
            for h in range(H):
                want = np.zeros(L)
                n = L - t0
                want[t0:] = f32[h, :n]
                want[t0] += D[h]
                assert np.max(np.abs(y[b, h] - want)) < 2e-2 * 5.0, (t0, b, h)
                if t0 + 7 < L:
                    assert int(np.argmax(np.abs(y[b, h] - D[h] * u[b, h]))) == t0 + 7
                if t0 > 0:
                    assert np.max(np.abs(y[b, h, :t0])) < 2e-2 * 5.0


@pytest.mark.parametrize("L", [1024, 8192])
def test_fftconv_fp16_slow_filters_constant_step_and_large_inputs(L):
    """fp16 I/O on the tensor-core paths with slow filters (dt ~ 1e-3): a
    constant input, a step input and a random input near the |u| limit
    (scaled so the outputs stay within fp16 range), against the oracle."""
    B, H = 2, 4
    wl = W.make_conv(B=B, H=H, L=L, N=64, dtype="f16", seed=3, dt_range=("loguniform", -3.0, -2.9))
    f32 = W.round_to(O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, L), "f32")
    gain = np.max(np.sum(np.abs(f32), axis=1)) + np.max(np.abs(wl.D))
    amp = min(30000.0, 30000.0 / gain)
    cases = {
        "constant": np.full((B, H, L), amp),
        "step": np.where(np.arange(L)[None, None, :] >= L // 3, amp, -0.5 * amp) * np.ones((B, H, 1)),
        "large random": np.clip(np.random.default_rng(5).normal(size=(B, H, L)) * amp / 3, -amp, amp),
    }
    for name, u in cases.items():
        u16 = W.round_to(u, "f16")
        y = host(api.fftconv_fwd(dev(u16, "f16"), dev(f32), dev(wl.D)))
        ref = cref.causal_conv(u16, f32, wl.D.astype(np.float64))
        assert np.all(np.isfinite(y)), name
        assert O.row_rel_err(y.reshape(-1, L), ref.reshape(-1, L)) < 2e-2, name


# ------------------------------------------------------------------ (f)4 any length
@pytest.mark.parametrize("L,dtype", [(1, "f32"), (7, "f32"), (100, "f16"), (1000, "bf16"), (1500, "f32"),
                                     (3000, "f16"), (5000, "bf16"), (8191, "f32")])
def test_fftconv_any_length(L, dtype):
    """Lengths that are not powers of two (EEG-clip-like lengths): zero padding
    to the next power of two on chip, causal outputs exact up to rounding."""
    B, H = 3, 5
    rng = np.random.default_rng(L)
    u = W.round_to(rng.normal(size=(B, H, L)), dtype)
    f = W.round_to(rng.normal(size=(H, L)) * np.exp(-np.arange(L) / max(1.0, L / 7.0)), "f32")  # arbitrary filters
    D = rng.normal(size=H)
    y = host(api.fftconv_fwd(dev(u, dtype), dev(f), dev(D)))
    ref = cref.causal_conv(u, f, D)
    assert O.row_rel_err(y.reshape(-1, L), ref.reshape(-1, L)) < TOL[dtype]
    dy = W.round_to(rng.normal(size=(B, H, L)), dtype)
    du, df, dD = api.fftconv_bwd(dev(dy, dtype), dev(u, dtype), dev(f), dev(D))
    rdu, rdf, rdD = O.causal_conv_bwd(dy, u, f, D)
    assert O.row_rel_err(host(du).reshape(-1, L), rdu.reshape(-1, L)) < TOL[dtype]
    assert O.row_rel_err(host(df), rdf) < 1e-4 * max(1.0, np.log2(L * B + 1) / 4)


@pytest.mark.parametrize("B,H,L,dtype", [(2, 3, 12000, "f32"), (3, 2, 9001, "bf16"), (1, 2, 20000, "f16"),
                                         (2, 2, 8193, "f32"), (1, 1, 65536, "f32"), (5, 2, 40000, "f32"),
                                         (2, 1, 32769, "bf16")])
def test_fftconv_long_matches_oracle(B, H, L, dtype):
    """Filters as long as the input past 8192 (12,000-step EEG-clip length,
    non-powers of two, the first length past 8192, the maximum; transform
    lengths 32768, 65536 and 131072, i.e. every four-step split; odd B
    leaves a pair with one row): against the direct fp64 convolution."""
    rng = np.random.default_rng(L + B)
    u = W.round_to(rng.normal(size=(B, H, L)), dtype)
    f = W.round_to(rng.normal(size=(H, L)) * np.exp(-np.arange(L) / (L / 3.0)), "f32")  # arbitrary, long-reaching
    D = rng.normal(size=H)
    y = host(api.fftconv_long_fwd(dev(u, dtype), dev(f), dev(D)))
    ref = cref.causal_conv(u, f, D)
    assert O.row_rel_err(y.reshape(-1, L), ref.reshape(-1, L)) < TOL[dtype]


def test_fftconv_long_bench_size_sampled_rows():
    """The EEG-length bench shape (B=8, H=256, L=12000, fp32) in the launch
    configuration the bench times; sampled rows (first, last, a row whose pair
    partner is the other half of its pair, channels at both ends) against the
    direct fp64 convolution one row at a time."""
    B, H, L = 8, 256, 12000
    rng = np.random.default_rng(12000)
    u = rng.normal(size=(B, H, L)).astype(np.float32)
    f = (rng.normal(size=(H, L)) * np.exp(-np.arange(L) / 4000.0)).astype(np.float32)
    D = rng.normal(size=H).astype(np.float32)
    y = host(api.fftconv_long_fwd(dev(u), dev(f), dev(D)))
    for b, h in [(0, 0), (1, 0), (7, 255), (6, 255), (3, 128), (4, 17)]:
        ref = cref.causal_conv(u[b:b + 1, h:h + 1].astype(np.float64), f[h:h + 1], D[h:h + 1])
        assert O.row_rel_err(y[b, h][None], ref.reshape(1, L)) < TOL["f32"], (b, h)


@pytest.mark.parametrize("L", [8193, 12000, 40000, 65536])
def test_fftconv_long_shift_filters_are_exact(L):
    """A filter that is a unit impulse at tap s shifts the input by s: y[t] =
    u[t - s] + D u[t] for t >= s, D u[t] before.  Taps at both ends of the
    four-step index split (s = 0, 1, 255, 256, M1 - 1, L - 1) land on exactly the
    right outputs; with an integer-valued u the results are exact up to the
    fp32 rounding of the transforms."""
    M = 1 << int(np.ceil(np.log2(2 * L - 1)))
    M1 = M // 256
    shifts = [0, 1, 255, 256, M1 - 1, L - 1]
    H, B = len(shifts), 3
    rng = np.random.default_rng(L)
    u = rng.integers(-4, 5, size=(B, H, L)).astype(np.float32)
    f = np.zeros((H, L), np.float32)
    for h, s in enumerate(shifts):
        f[h, s] = 1.0
    D = np.full(H, 0.5, np.float32)
    y = host(api.fftconv_long_fwd(dev(u), dev(f), dev(D)))
    for h, s in enumerate(shifts):
        want = 0.5 * u[:, h].astype(np.float64)
        want[:, s:] += u[:, h, :L - s]
        assert np.max(np.abs(y[:, h] - want)) < 1e-3, (L, s)


def test_fftconv_long_short_lengths_are_fftconv_fwd():
    B, H, L = 3, 4, 5000
    rng = np.random.default_rng(5)
    u = dev(W.round_to(rng.normal(size=(B, H, L)), "f16"), "f16")
    f = dev(rng.normal(size=(H, L)) * np.exp(-np.arange(L) / 900.0))
    D = dev(rng.normal(size=H))
    assert np.array_equal(host(api.fftconv_long_fwd(u, f, D)), host(api.fftconv_fwd(u, f, D)))


def test_ssm_conv_any_length():
    wl = W.make_conv(B=2, H=6, L=1234, N=80, dtype="f32", seed=9)  # N > 64: fused generation path
    y = host(api.ssm_conv_fwd(dev(wl.u), *params(wl)))
    f = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, wl.L)
    ref = cref.causal_conv(wl.u, f, wl.D.astype(np.float64))
    assert O.row_rel_err(y.reshape(-1, wl.L), ref.reshape(-1, wl.L)) < 1e-4


# ------------------------------------------------------------------ (f)3 state-passing backward
@pytest.mark.parametrize("B,H,L,T,N,dtype,with_g", [
    (2, 3, 256, 64, 8, "f32", True), (1, 2, 512, 128, 16, "f32", False), (2, 2, 1024, 256, 33, "f32", True),
    (1, 3, 8192, 2048, 16, "f16", True), (1, 2, 16384, 8192, 64, "bf16", False),
])
def test_statepass_bwd(B, H, L, T, N, dtype, with_g):
    """du and dstate_in against the oracle's gradient sums; with a gradient on
    the final state and without."""
    wl = W.make_conv(B=B, H=H, L=L, N=N, dtype=dtype, seed=L + N, dt_range=("loguniform", -3.0, -1.0))
    dtt, lam, Bp, Cp, D = params(wl)
    rng = np.random.default_rng(T)
    dy = W.round_to(rng.normal(size=(B, H, L)), dtype)
    G = (rng.normal(size=(B, H, N)) + 1j * rng.normal(size=(B, H, N))) if with_g else None
    g_t = torch.view_as_real(torch.tensor(G.astype(np.complex64))).cuda().contiguous() if with_g else None
    du, dsin = api.fftconv_statepass_bwd(dev(dy, dtype), dtt, lam, Bp, Cp, D, T, dstate_out=g_t, need_dstate_in=True)
    A, Bc, Cc = oracle_A(wl)
    G64 = G.astype(np.complex64).astype(np.complex128) if with_g else None
    rdu, rdsin = O.statepass_bwd(dy, A, Bc, Cc, wl.D.astype(np.float64), dstate_out=G64)
    assert O.row_rel_err(host(du).reshape(-1, L), rdu.reshape(-1, L)) < TOL[dtype]
    g = host(dsin)
    g = g[..., 0] + 1j * g[..., 1]
    tol = 1e-4 if dtype == "f32" else 5e-3
    assert np.max(np.abs(g - rdsin)) < tol * np.max(np.abs(rdsin))
