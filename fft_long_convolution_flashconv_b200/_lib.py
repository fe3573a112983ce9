"""ctypes binding of libflashconv_b200.so (argument marshalling only).

Every entry point declared in include/flashconv.h is bound here with the same
name.  There is no fallback: if the shared library is missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libflashconv_b200.so")

FC_OK, FC_EINVAL, FC_EUNSUPPORTED, FC_ECUDA, FC_ENOMEM = 0, -1, -2, -3, -4
FC_F32, FC_F16, FC_BF16 = 0, 1, 2

# name -> (restype, argtypes)
_vp, _fp, _i, _sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "fc_version": (ctypes.c_int, []),
    "fc_status_string": (ctypes.c_char_p, [_i]),
    "fc_last_error": (ctypes.c_char_p, []),
    "fc_tc_timeouts": (ctypes.c_uint, []),
    "ssm_kernel_gen": (_i, [_fp, _fp, _fp, _fp, _i, _i, _i, _fp, _vp]),
    "fftconv_fwd": (_i, [_vp, _fp, _fp, _vp, _i, _i, _i, _i, _vp]),
    "fftconv_long_workspace": (_sz, [_i, _i, _i]),
    "fftconv_long_fwd": (_i, [_vp, _fp, _fp, _vp, _i, _i, _i, _vp, _sz, _i, _vp]),
    "fftconv_bwd": (_i, [_vp, _vp, _fp, _fp, _vp, _fp, _fp, _i, _i, _i, _i, _vp]),
    "ssm_conv_workspace": (_sz, [_i, _i]),
    "ssm_decode_step": (_i, [_vp, _fp, _fp, _fp, _fp, _fp, _fp, _vp, _i, _i, _i, _i, _i, _vp]),
    "h3_decode_state_bytes": (_sz, [_i, _i, _i, _i]),
    "h3_mixer_decode_step": (_i, [_vp, _vp, _vp, _vp, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _vp, _i, _i, _i, _i, _i,
                                  ctypes.c_longlong, _i, _vp]),
    "ssm_conv_fwd": (_i, [_vp, _fp, _fp, _fp, _fp, _fp, _vp, _i, _i, _i, _i, _vp, _sz, _i, _vp]),
    "fftconv_statepass_workspace": (_sz, [_i, _i, _i, _i, _i]),
    "fftconv_statepass": (_i, [_vp, _fp, _fp, _fp, _fp, _fp, _vp, _i, _i, _i, _i, _i, _fp, _fp, _vp, _sz,
                               _i, _vp]),
    "fftconv_statepass_bwd_workspace": (_sz, [_i, _i, _i, _i, _i, _i]),
    "fftconv_statepass_bwd": (_i, [_vp, _fp, _fp, _fp, _fp, _fp, _vp, _i, _i, _i, _i, _i, _fp, _fp, _vp, _sz,
                                   _i, _vp]),
    "ssm_conv_fwd_noalloc": (_i, [_vp, _fp, _fp, _fp, _fp, _fp, _vp, _i, _i, _i, _i, _i, _vp]),
    "ssm_conv_noalloc_max_filter_floats": (_sz, []),
    "ssm_conv_noalloc_last_error": (ctypes.c_char_p, []),
    "h3_mixer_workspace": (_sz, [_i, _i, _i, _i, _i]),
    "h3_mixer_fwd": (_i, [_vp, _vp, _vp, _fp, _fp, _fp, _fp, _fp, _fp, _vp, _i, _i, _i, _i, _i, _i, _vp, _sz,
                          _i, _vp]),
}

_lib = None


class FlashConvError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: status {status}: {msg}")
        self.status = status


def load(path: str = None) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built).  FC_LIB_PATH
    selects another build of it (e.g. the bounds-checked debug variant)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or os.environ.get("FC_LIB_PATH") or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m fft_long_convolution_flashconv_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(status: int, where: str) -> None:
    if status != FC_OK:
        msg = load().fc_last_error().decode(errors="replace")
        raise FlashConvError(status, where, msg)
