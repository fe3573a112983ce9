"""C ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before launching
anything (each call below carries at least one argument that validation
rejects, so no kernel is ever launched with the fake pointers used here)."""
import ctypes
import os
import re

import pytest

from fft_long_convolution_flashconv_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flashconv.h")

P = 0x10000000  # fake, 256-byte aligned "device" address: never dereferenced
P2 = 0x20000000
P3 = 0x30000000


def declared_symbols():
    txt = open(HEADER).read()
    return re.findall(r"FC_API\s+[\w\s\*]+?\b(\w+)\s*\(", txt)


def test_header_declares_expected_entry_points():
    syms = set(declared_symbols())
    for s in ("ssm_kernel_gen", "fftconv_fwd", "fftconv_statepass", "h3_mixer_fwd",
              "fftconv_statepass_workspace", "h3_mixer_workspace", "ssm_conv_fwd", "ssm_conv_workspace",
              "fc_last_error", "fc_status_string", "fc_version", "fftconv_bwd", "fc_tc_timeouts",
              "ssm_decode_step", "h3_mixer_decode_step", "h3_decode_state_bytes",
              "fftconv_statepass_bwd", "fftconv_statepass_bwd_workspace", "fftconv_long_fwd",
              "fftconv_long_workspace"):
        assert s in syms


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    for s in declared_symbols():
        assert hasattr(lib, s), s
        assert s in _lib.SIGNATURES, s


def test_nvcc_target_is_sm100a():
    from fft_long_convolution_flashconv_b200 import build
    assert "arch=compute_100a,code=sm_100a" in build.NVCC_FLAGS


def _err():
    return _lib.load().fc_last_error().decode()


def test_fftconv_rejects_bad_arguments():
    lib = _lib.load()
    # L too large (any L in [1, 8192] is accepted, powers of two or not)
    assert lib.fftconv_fwd(P, P2, P3, P + (1 << 26), 2, 3, 16384, 1, None) == _lib.FC_EUNSUPPORTED
    assert "[1, 8192]" in _err()
    assert lib.fftconv_fwd(P, P2, P3, P + (1 << 26), 2, 3, 8193, 1, None) == _lib.FC_EUNSUPPORTED
    # null pointers
    assert lib.fftconv_fwd(None, P2, P3, P, 2, 3, 64, 1, None) == _lib.FC_EINVAL
    assert lib.fftconv_fwd(P, None, P3, P + (1 << 26), 2, 3, 64, 1, None) == _lib.FC_EINVAL
    # misaligned u
    assert lib.fftconv_fwd(P + 2, P2, P3, P + (1 << 26), 2, 3, 64, 1, None) == _lib.FC_EINVAL
    assert "aligned" in _err()
    # overlapping u / y
    assert lib.fftconv_fwd(P, P2, P3, P + 64, 2, 3, 64, 1, None) == _lib.FC_EINVAL
    assert "overlap" in _err()
    # bad dtype, bad sizes
    assert lib.fftconv_fwd(P, P2, P3, P + (1 << 26), 2, 3, 64, 7, None) == _lib.FC_EINVAL
    assert lib.fftconv_fwd(P, P2, P3, P + (1 << 26), 0, 3, 64, 1, None) == _lib.FC_EINVAL


def test_ssm_gen_rejects_bad_arguments():
    lib = _lib.load()
    assert lib.ssm_kernel_gen(P, P2, P3, P, 4, 0, 256, P2, None) == _lib.FC_EINVAL
    assert lib.ssm_kernel_gen(P, P2, P3, P, 4, 2000, 256, P2, None) == _lib.FC_EUNSUPPORTED
    assert lib.ssm_kernel_gen(P, None, P3, P, 4, 64, 256, P2, None) == _lib.FC_EINVAL
    assert lib.ssm_kernel_gen(P, P2, P3, P, 4, 64, 256, P2 + 4, None) == _lib.FC_EINVAL


def test_statepass_rejects_bad_arguments():
    lib = _lib.load()
    B, H, L, N, T = 1, 4, 1024, 64, 256
    ws = lib.fftconv_statepass_workspace(B, H, L, N, T)
    assert ws > 0
    y = P + (1 << 26)
    # L not a multiple of chunk
    assert lib.fftconv_statepass(P, P2, P3, P, P2, P3, y, B, H, 1000, N, T, None, None, P3, ws, 1, None) \
        == _lib.FC_EINVAL
    # chunk not a power of two / too big
    assert lib.fftconv_statepass(P, P2, P3, P, P2, P3, y, B, H, 3 * 300, N, 300, None, None, P3, ws, 1, None) \
        == _lib.FC_EUNSUPPORTED
    assert lib.fftconv_statepass(P, P2, P3, P, P2, P3, y, B, H, 32768, N, 16384, None, None, P3, ws, 1, None) \
        == _lib.FC_EUNSUPPORTED
    # workspace too small / misaligned
    assert lib.fftconv_statepass(P, P2, P3, P, P2, P3, y, B, H, L, N, T, None, None, P3, ws - 1, 1, None) \
        == _lib.FC_EINVAL
    assert "workspace too small" in _err()
    assert lib.fftconv_statepass(P, P2, P3, P, P2, P3, y, B, H, L, N, T, None, None, P3 + 16, ws, 1, None) \
        == _lib.FC_EINVAL
    # N too large
    assert lib.fftconv_statepass(P, P2, P3, P, P2, P3, y, B, H, L, 300, T, None, None, P3, ws, 1, None) \
        == _lib.FC_EUNSUPPORTED
    assert lib.fftconv_statepass_workspace(B, H, 1000, N, T) == 0


def test_mixer_rejects_bad_arguments():
    lib = _lib.load()
    B, L, heads, hd, N = 2, 128, 2, 64, 8
    ws = lib.h3_mixer_workspace(B, L, heads, hd, N)
    o = P + (1 << 26)
    args = lambda **kw: dict(q=P, k=P2, v=P3, Cs=P, dt=P, lam=P2, Bp=P3, Cp=P, D=P, o=o, B=B, L=L,
                             heads=heads, hd=hd, N=N, S=4, ws=P2, wsb=ws, dtype=1, **kw)

    def call(a):
        return lib.h3_mixer_fwd(a["q"], a["k"], a["v"], a["Cs"], a["dt"], a["lam"], a["Bp"], a["Cp"], a["D"],
                                a["o"], a["B"], a["L"], a["heads"], a["hd"], a["N"], a["S"], a["ws"], a["wsb"],
                                a["dtype"], None)
    a = args(); a["hd"] = 32
    assert call(a) == _lib.FC_EUNSUPPORTED
    a = args(); a["S"] = 9
    assert call(a) == _lib.FC_EUNSUPPORTED
    a = args(); a["wsb"] = ws - 1
    assert call(a) == _lib.FC_EINVAL
    a = args(); a["o"] = P2 + 128
    assert call(a) == _lib.FC_EINVAL and "overlap" in _err()
    a = args(); a["k"] = None
    assert call(a) == _lib.FC_EINVAL


def test_error_message_is_per_call():
    lib = _lib.load()
    assert lib.fftconv_fwd(P, P2, P3, P + (1 << 26), 2, 3, 16384, 1, None) != 0
    assert _err()
    assert lib.fc_status_string(0) == b"ok"


def test_noalloc_rejects_oversize_before_any_launch():
    lib = _lib.load()
    assert lib.ssm_conv_noalloc_max_filter_floats() == 1 << 20
    # H * L = 2^21 > the fixed scratch: refused on the host, nothing launched
    y = P + (1 << 28)
    assert lib.ssm_conv_fwd_noalloc(P, P2, P3, P, P2, P3, y, 1, 256, 8192, 64, 1, None) == _lib.FC_EUNSUPPORTED
    assert b"fixed scratch" in lib.ssm_conv_noalloc_last_error()
    assert lib.ssm_conv_fwd_noalloc(P, P2, P3, P, P2, P3, y, 1, 4, 10000, 64, 1, None) == _lib.FC_EUNSUPPORTED
    assert lib.ssm_conv_fwd_noalloc(None, P2, P3, P, P2, P3, y, 1, 4, 1024, 64, 1, None) == _lib.FC_EINVAL


def test_backward_and_decode_reject_bad_arguments():
    lib = _lib.load()
    du = P + (1 << 26)
    # nothing requested, df without dD, L out of range, overlap of dy and du
    assert lib.fftconv_bwd(P, P2, P3, P, None, None, None, 2, 3, 64, 1, None) == _lib.FC_EINVAL
    assert lib.fftconv_bwd(P, P2, P3, P, None, P2, None, 2, 3, 64, 1, None) == _lib.FC_EINVAL
    assert lib.fftconv_bwd(P, P2, P3, P, du, None, None, 2, 3, 9000, 1, None) == _lib.FC_EUNSUPPORTED
    assert lib.fftconv_bwd(P, P2, P3, P, P + 64, None, None, 2, 3, 64, 1, None) == _lib.FC_EINVAL
    # du requested without f
    assert lib.fftconv_bwd(P, P2, None, P, du, None, None, 2, 3, 64, 1, None) == _lib.FC_EINVAL
    # decode: T < 1, N too large, misaligned state
    y = P + (1 << 26)
    assert lib.ssm_decode_step(P, P2, P, P2, P3, P, P, y, 2, 3, 16, 0, 1, None) == _lib.FC_EINVAL
    assert lib.ssm_decode_step(P, P2, P, P2, P3, P, P, y, 2, 3, 2000, 1, 1, None) == _lib.FC_EUNSUPPORTED
    assert lib.ssm_decode_step(P, P2 + 4, P, P2, P3, P, P, y, 2, 3, 16, 1, 1, None) == _lib.FC_EINVAL
    # mixer decode: head_dim too large, shift_len out of range, negative position
    o = P + (1 << 26)
    assert lib.h3_mixer_decode_step(P, P, P, P, P2, P, P, P2, P3, P, P, o, 1, 2, 65, 8, 4, 0, 1,
                                    None) == _lib.FC_EUNSUPPORTED
    assert lib.h3_mixer_decode_step(P, P, P, P, P2, P, P, P2, P3, P, P, o, 1, 2, 64, 8, 9, 0, 1,
                                    None) == _lib.FC_EUNSUPPORTED
    assert lib.h3_mixer_decode_step(P, P, P, P, P2, P, P, P2, P3, P, P, o, 1, 2, 64, 8, 4, -1, 1,
                                    None) == _lib.FC_EINVAL
    assert lib.h3_decode_state_bytes(2, 3, 64, 8) == 2 * 3 * 64 * 64 * 8 * 8


def test_long_conv_rejects_bad_arguments():
    lib = _lib.load()
    y = P + (1 << 28)
    ws = lib.fftconv_long_workspace(2, 3, 12000)
    assert ws >= 4 * 2 * 3 * 16384 * 4
    assert lib.fftconv_long_workspace(2, 3, 8192) == 0 and lib.fftconv_long_workspace(2, 3, 70000) == 0
    # L out of range, missing / misaligned / small workspace, overlap
    assert lib.fftconv_long_fwd(P, P2, P3, y, 2, 3, 70000, P3, ws, 0, None) == _lib.FC_EUNSUPPORTED
    assert lib.fftconv_long_fwd(P, P2, P3, y, 2, 3, 12000, None, ws, 0, None) == _lib.FC_EINVAL
    assert lib.fftconv_long_fwd(P, P2, P3, y, 2, 3, 12000, P3 + 16, ws, 0, None) == _lib.FC_EINVAL
    assert lib.fftconv_long_fwd(P, P2, P3, y, 2, 3, 12000, P3, ws - 1, 0, None) == _lib.FC_EINVAL
    assert "workspace too small" in _err()
    assert lib.fftconv_long_fwd(P, P2, P3, P + 64, 2, 3, 12000, P3, ws, 0, None) == _lib.FC_EINVAL
    # L <= 8192 goes through fftconv_fwd's validation
    assert lib.fftconv_long_fwd(P, P2, P3, y, 2, 3, 4096, None, 0, 7, None) == _lib.FC_EINVAL
    # more row pairs than the pass grids index
    far = P + (1 << 50)  # an output that cannot overlap the (fake) input of this size
    assert lib.fftconv_long_fwd(P, P2, P3, far, 2, (1 << 29) + 1, 9000, P3, 1 << 62, 0, None) == _lib.FC_EUNSUPPORTED
    assert "2^29" in _err()


@pytest.mark.parametrize("B,H,L,M", [(2, 3, 12000, 32768), (3, 2, 8193, 32768), (5, 7, 20000, 65536),
                                     (1, 1, 32768, 65536), (1, 1, 32769, 131072), (4, 2, 65536, 131072)])
def test_long_conv_workspace_holds_pair_and_filter_spectra(B, H, L, M):
    """The workspace of the four-step long convolution: the complex fp32
    spectra of the H * ceil(B / 2) row pairs and of the H filters at the
    transform length M = 2^ceil(log2(2L - 1)), each part rounded up to 256
    bytes."""
    lib = _lib.load()
    r256 = lambda b: (b + 255) // 256 * 256
    pairs = H * ((B + 1) // 2)
    assert lib.fftconv_long_workspace(B, H, L) == r256(pairs * M * 8) + r256(H * M * 8)
