"""Seeded synthetic workloads for the SSM long convolution.

This module only draws random numbers and fixes shapes; it holds none of the
method's arithmetic (no discretisation, no filter, no convolution).  Both the
CPU oracle and the CUDA path consume the arrays it returns.

Workload shapes follow the H3 / FlashConv pages ("Hungry Hungry Hippos",
section 2 "State space models" / "Convolutional view", section 3 "H3 design",
section 4 "FlashConv"): a diagonal SSM per channel with the S4D-Lin
initialisation lambda_n = -0.5 + i*pi*n, B_n = 1, C complex normal, D normal,
and u standard normal.  Floating inputs that the GPU reads in 16-bit form are
rounded to that dtype here (round-to-nearest-even), and the rounded values are
what every consumer sees.

Draw order from ``numpy.random.default_rng(seed)`` (fixed, so any consumer can
reproduce a case):
  * convolution workloads: dt, C.re, C.im, D, u
  * H3 mixer workload:     q, k, v, C_shift, dt, C.re, C.im, D
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = [
    "ConvWorkload", "MixerWorkload", "CONFIGS", "make_conv", "make_mixer",
    "round_to", "s4d_lin_lambda", "np_dtype_name",
]

DTYPES = ("f32", "f16", "bf16")


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to ``dtype`` with round-to-nearest-even and return
    them as float64 again (the exact values a 16/32-bit buffer holds)."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "f16":
        return x.astype(np.float16).astype(np.float64)
    if dtype == "bf16":
        # float64 -> float32 is RNE; float32 -> bfloat16 by RNE on the bit
        # pattern.  The double rounding cannot differ from a direct RNE for
        # normal N(0,1) data except in astronomically rare ties; the value
        # stored is whatever this function returns, and both sides use it.
        f = x.astype(np.float32)
        b = f.view(np.uint32).astype(np.uint64)
        lsb = (b >> 16) & 1
        b = (b + 0x7FFF + lsb) & 0xFFFF0000
        return b.astype(np.uint32).view(np.float32).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Return the raw storage array for ``dtype`` (float32, float16, or the
    bfloat16 bit pattern as uint16) holding the rounded values of ``x``."""
    r = round_to(x, dtype)
    if dtype == "f32":
        return r.astype(np.float32)
    if dtype == "f16":
        return r.astype(np.float16)
    if dtype == "bf16":
        return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    raise ValueError(dtype)


def np_dtype_name(dtype: str) -> str:
    return {"f32": "float32", "f16": "float16", "bf16": "bfloat16"}[dtype]


def s4d_lin_lambda(H: int, N: int) -> np.ndarray:
    """S4D-Lin continuous-time eigenvalues lambda_n = -0.5 + i*pi*n, stored as
    float32 real/imag parts (shape H x N x 2) -- these float32 values are the
    input; consumers promote them exactly."""
    lam = np.zeros((H, N, 2), dtype=np.float32)
    lam[:, :, 0] = np.float32(-0.5)
    lam[:, :, 1] = (np.pi * np.arange(N, dtype=np.float64)).astype(np.float32)[None, :]
    return lam


@dataclasses.dataclass
class ConvWorkload:
    name: str
    B: int
    H: int
    L: int
    N: int
    dtype: str
    seed: int
    chunk: Optional[int]
    dt: np.ndarray        # (H,) float32
    lam: np.ndarray       # (H, N, 2) float32 (re, im)
    Bp: np.ndarray        # (H, N, 2) float32
    Cp: np.ndarray        # (H, N, 2) float32
    D: np.ndarray         # (H,) float32
    u: np.ndarray         # (B, H, L) float64 holding dtype-rounded values

    def u_storage(self) -> np.ndarray:
        return to_storage(self.u, self.dtype)


@dataclasses.dataclass
class MixerWorkload:
    name: str
    B: int
    L: int
    heads: int
    head_dim: int
    N: int
    shift_len: int
    dtype: str
    seed: int
    q: np.ndarray         # (B, L, heads*head_dim) float64 holding rounded values
    k: np.ndarray
    v: np.ndarray
    Cshift: np.ndarray    # (heads*head_dim, shift_len) float32
    dt: np.ndarray        # (heads,) float32
    lam: np.ndarray       # (heads, N, 2) float32
    Bp: np.ndarray        # (heads, N, 2) float32
    Cp: np.ndarray        # (heads, N, 2) float32
    D: np.ndarray         # (heads,) float32


# name -> keyword arguments.  cfg1..cfg5 are the five published workloads;
# the "small_*" entries are reduced shapes with the same recipe that the
# oracle finishes in seconds while still spanning several tiles and a tail.
CONFIGS = {
    "cfg1_conv_f32_B1_H4_L256": dict(kind="conv", B=1, H=4, L=256, N=32, dtype="f32", seed=0,
                                     dt_range=("loguniform", -3.0, -1.0)),
    "cfg2_conv_f16_B8_H768_L1024": dict(kind="conv", B=8, H=768, L=1024, N=64, dtype="f16", seed=1,
                                        dt_range=("loguniform", -3.0, -1.0)),
    "cfg3_conv_bf16_B4_H1024_L8192": dict(kind="conv", B=4, H=1024, L=8192, N=64, dtype="bf16", seed=2,
                                          dt_range=("split", (-3.0, -2.9), (-1.1, -1.0))),
    "cfg4_statepass_f16_B1_H2560_L65536_T8192": dict(kind="conv", B=1, H=2560, L=65536, N=64, dtype="f16",
                                                     seed=3, chunk=8192,
                                                     dt_range=("loguniform", -3.0, -1.0)),
    "cfg5_h3mixer_f16_B8_L2048_d768": dict(kind="mixer", B=8, L=2048, heads=12, head_dim=64, N=64,
                                           shift_len=4, dtype="f16", seed=4),
}


def _draw_dt(rng: np.random.Generator, H: int, spec) -> np.ndarray:
    kind = spec[0]
    if kind == "loguniform":
        lo, hi = spec[1], spec[2]
        return (10.0 ** rng.uniform(lo, hi, H)).astype(np.float32)
    if kind == "split":
        (lo1, hi1), (lo2, hi2) = spec[1], spec[2]
        h1 = H // 2
        a = 10.0 ** rng.uniform(lo1, hi1, h1)
        b = 10.0 ** rng.uniform(lo2, hi2, H - h1)
        return np.concatenate([a, b]).astype(np.float32)
    raise ValueError(spec)


def make_conv(B: int, H: int, L: int, N: int, dtype: str, seed: int,
              dt_range=("loguniform", -3.0, -1.0), chunk: Optional[int] = None,
              name: str = "custom", u_override: Optional[np.ndarray] = None) -> ConvWorkload:
    """Seeded diagonal-SSM convolution workload (see module docstring for the
    draw order)."""
    if dtype not in DTYPES:
        raise ValueError(dtype)
    rng = np.random.default_rng(seed)
    dt = _draw_dt(rng, H, dt_range)
    c_re = rng.normal(0.0, np.sqrt(0.5), (H, N))
    c_im = rng.normal(0.0, np.sqrt(0.5), (H, N))
    D = rng.normal(0.0, 1.0, H).astype(np.float32)
    if u_override is None:
        u = rng.normal(0.0, 1.0, (B, H, L))
    else:
        u = np.asarray(u_override, dtype=np.float64).reshape(B, H, L)
    Cp = np.stack([c_re, c_im], axis=-1).astype(np.float32)
    Bp = np.zeros((H, N, 2), dtype=np.float32)
    Bp[:, :, 0] = 1.0
    return ConvWorkload(name=name, B=B, H=H, L=L, N=N, dtype=dtype, seed=seed, chunk=chunk,
                        dt=dt, lam=s4d_lin_lambda(H, N), Bp=Bp, Cp=Cp, D=D,
                        u=round_to(u, dtype))


def make_mixer(B: int, L: int, heads: int, head_dim: int, N: int, shift_len: int, dtype: str,
               seed: int, name: str = "custom") -> MixerWorkload:
    """Seeded H3 mixer workload: q, k, v ~ N(0, 1/d_model), C_shift ~ N(0, 1),
    per-head diagonal SSM with the S4D-Lin init, D ~ N(0, 1)."""
    rng = np.random.default_rng(seed)
    dm = heads * head_dim
    sd = np.sqrt(1.0 / dm)
    q = rng.normal(0.0, sd, (B, L, dm))
    k = rng.normal(0.0, sd, (B, L, dm))
    v = rng.normal(0.0, sd, (B, L, dm))
    Cshift = rng.normal(0.0, 1.0, (dm, shift_len)).astype(np.float32)
    dt = (10.0 ** rng.uniform(-3.0, -1.0, heads)).astype(np.float32)
    c_re = rng.normal(0.0, np.sqrt(0.5), (heads, N))
    c_im = rng.normal(0.0, np.sqrt(0.5), (heads, N))
    D = rng.normal(0.0, 1.0, heads).astype(np.float32)
    Cp = np.stack([c_re, c_im], axis=-1).astype(np.float32)
    Bp = np.zeros((heads, N, 2), dtype=np.float32)
    Bp[:, :, 0] = 1.0
    return MixerWorkload(name=name, B=B, L=L, heads=heads, head_dim=head_dim, N=N,
                         shift_len=shift_len, dtype=dtype, seed=seed,
                         q=round_to(q, dtype), k=round_to(k, dtype), v=round_to(v, dtype),
                         Cshift=Cshift, dt=dt, lam=s4d_lin_lambda(heads, N), Bp=Bp, Cp=Cp, D=D)


def make(name: str, **overrides):
    """Build one of CONFIGS by name (keyword overrides change shape fields)."""
    spec = dict(CONFIGS[name])
    spec.update(overrides)
    kind = spec.pop("kind")
    if kind == "conv":
        return make_conv(name=name, **spec)
    return make_mixer(name=name, **spec)
