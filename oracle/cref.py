"""ctypes loader for the plain-C fp64 oracle (TEST INFRASTRUCTURE ONLY; see
``oracle/conv_ref.c``).  ``build()`` compiles it with gcc -O2 -fopenmp."""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "conv_ref.c")
_SO = os.path.join(_HERE, "libconv_ref.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               _SRC, "-o", _SO, "-lm"])
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        dp = ctypes.POINTER(ctypes.c_double)
        L.oracle_causal_conv.argtypes = [dp, dp, dp, dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
        L.oracle_causal_conv.restype = None
        L.oracle_ssm_recurrence.argtypes = [dp, dp, dp, dp, dp, ctypes.c_void_p, dp, ctypes.c_void_p,
                                            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
        L.oracle_ssm_recurrence.restype = None
        L.oracle_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def causal_conv(u, f, D) -> np.ndarray:
    """C version of ``ssm_oracle.causal_conv_direct`` (u: B x H x L)."""
    u = np.ascontiguousarray(u, dtype=np.float64)
    B, H, L = u.shape
    f = np.ascontiguousarray(np.asarray(f, dtype=np.float64)[:, :L])
    D = np.ascontiguousarray(D, dtype=np.float64)
    y = np.empty_like(u)
    lib().oracle_causal_conv(_p(u), _p(f), _p(D), _p(y), B * H, H, L)
    return y


def ssm_recurrence(u, A, Bc, Cc, D, x0=None):
    """C version of ``ssm_oracle.ssm_recurrence``; returns (y, x_last)."""
    u = np.ascontiguousarray(u, dtype=np.float64)
    B, H, L = u.shape
    N = np.asarray(A).shape[1]
    if N > 1024:
        raise ValueError("N > 1024")

    def cplx(a):
        a = np.asarray(a, dtype=np.complex128)
        return np.ascontiguousarray(np.stack([a.real, a.imag], axis=-1))
    Ai, Bi, Ci = cplx(A), cplx(Bc), cplx(Cc)
    D = np.ascontiguousarray(D, dtype=np.float64)
    y = np.empty_like(u)
    xo = np.empty((B, H, N, 2), dtype=np.float64)
    x0p = None
    if x0 is not None:
        x0i = cplx(x0)
        x0p = x0i.ctypes.data_as(ctypes.c_void_p)
    lib().oracle_ssm_recurrence(_p(u), _p(Ai), _p(Bi), _p(Ci), _p(D), x0p, _p(y),
                                xo.ctypes.data_as(ctypes.c_void_p), B * H, H, N, L)
    return y, xo[..., 0] + 1j * xo[..., 1]
