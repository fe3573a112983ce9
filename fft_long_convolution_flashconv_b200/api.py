"""PyTorch-facing wrappers over the C ABI (argument marshalling only: every
step runs in the CUDA library; torch only provides device memory and the
current stream).

Complex SSM parameters are float32 tensors of shape (..., 2) (re, im) or
complex64 tensors.  I/O tensors are float32, float16 or bfloat16 CUDA tensors.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib
from ._lib import check

_DT = {torch.float32: _lib.FC_F32, torch.float16: _lib.FC_F16, torch.bfloat16: _lib.FC_BF16}


def _stream():
    return ctypes_void(torch.cuda.current_stream().cuda_stream)


def ctypes_void(x):
    import ctypes
    return ctypes.c_void_p(x)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _cpx(t: torch.Tensor) -> torch.Tensor:
    if t.is_complex():
        t = torch.view_as_real(t)
    if t.dtype != torch.float32 or t.shape[-1] != 2:
        raise ValueError("complex parameters must be complex64 or float32 (..., 2)")
    return t.contiguous()


def _f32(t: torch.Tensor) -> torch.Tensor:
    if t.dtype != torch.float32:
        raise ValueError("parameters must be float32")
    return t.contiguous()


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return _DT[t.dtype]


def _alloc_ws(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns >= 256-byte aligned blocks
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


def tc_timeouts() -> int:
    """Tensor-core blocks that gave up waiting on a matrix-multiply completion
    (their part of an output is unwritten); 0 in normal operation."""
    return int(_lib.load().fc_tc_timeouts())


def ssm_kernel_gen(dt, lam, Bp, Cp, L: int, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """f[h, k] = 2 Re sum_n C B A^k, A = exp(dt lambda); returns H x L float32."""
    lib = _lib.load()
    dt, lam, Bp, Cp = _f32(dt), _cpx(lam), _cpx(Bp), _cpx(Cp)
    H, N = lam.shape[0], lam.shape[1]
    if out is None:
        out = torch.empty((H, L), dtype=torch.float32, device=dt.device)
    check(lib.ssm_kernel_gen(_ptr(dt), _ptr(lam), _ptr(Bp), _ptr(Cp), H, N, L, _ptr(out), _stream()),
          "ssm_kernel_gen")
    return out


def fftconv_fwd(u: torch.Tensor, f: torch.Tensor, D: torch.Tensor,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = causal_conv(u, f) + D u via the fused FFT kernel; u: B x H x L."""
    lib = _lib.load()
    B, H, L = u.shape
    f, D = _f32(f), _f32(D)
    if out is None:
        out = torch.empty_like(u)
    check(lib.fftconv_fwd(_ptr(u), _ptr(f), _ptr(D), _ptr(out), B, H, L, _dtype(u), _stream()), "fftconv_fwd")
    return out


def long_conv_workspace_bytes(B: int, H: int, L: int) -> int:
    return int(_lib.load().fftconv_long_workspace(B, H, L))


def fftconv_long_fwd(u: torch.Tensor, f: torch.Tensor, D: torch.Tensor, out: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = causal_conv(u, f) + D u for L up to 65536 (arbitrary filter); u: B x H x L."""
    lib = _lib.load()
    B, H, L = u.shape
    f, D = _f32(f), _f32(D)
    if out is None:
        out = torch.empty_like(u)
    need = int(lib.fftconv_long_workspace(B, H, L))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=u.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    check(lib.fftconv_long_fwd(_ptr(u), _ptr(f), _ptr(D), _ptr(out), B, H, L, _ptr(workspace), ws_bytes,
                               _dtype(u), _stream()), "fftconv_long_fwd")
    return out


def fftconv_bwd(dy: torch.Tensor, u: torch.Tensor, f: torch.Tensor, D: torch.Tensor, need_du: bool = True,
                need_dfilter: bool = True):
    """Gradients of y = causal_conv(u, f) + D u given dy; returns (du, df, dD)
    (None for the parts not requested)."""
    lib = _lib.load()
    B, H, L = dy.shape
    f, D = _f32(f), _f32(D)
    du = torch.empty_like(dy) if need_du else None
    df = torch.empty((H, L), dtype=torch.float32, device=dy.device) if need_dfilter else None
    dD = torch.empty((H,), dtype=torch.float32, device=dy.device) if need_dfilter else None
    check(lib.fftconv_bwd(_ptr(dy), _ptr(u), _ptr(f), _ptr(D), _ptr(du), _ptr(df), _ptr(dD), B, H, L, _dtype(dy),
                          _stream()), "fftconv_bwd")
    return du, df, dD


def ssm_decode_step(u, x, dt, lam, Bp, Cp, D, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """T tokens of the recurrent view; u: B x H x T; x: B x H x N x 2 float32
    state, updated in place.  Returns y (B x H x T)."""
    lib = _lib.load()
    B, H, Tn = u.shape
    dt, lam, Bp, Cp, D = _f32(dt), _cpx(lam), _cpx(Bp), _cpx(Cp), _f32(D)
    N = lam.shape[1]
    if x.dtype != torch.float32 or tuple(x.shape) != (B, H, N, 2) or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 B x H x N x 2 tensor")
    if out is None:
        out = torch.empty_like(u)
    check(lib.ssm_decode_step(_ptr(u), _ptr(x), _ptr(dt), _ptr(lam), _ptr(Bp), _ptr(Cp), _ptr(D), _ptr(out), B, H,
                              N, Tn, _dtype(u), _stream()), "ssm_decode_step")
    return out


def h3_decode_state(B, heads, head_dim, N, device) -> torch.Tensor:
    """Zeroed recurrent state of the H3 mixer (B x heads x hd x hd x N x 2 float32)."""
    return torch.zeros((B, heads, head_dim, head_dim, N, 2), dtype=torch.float32, device=device)


def h3_mixer_decode_step(q, k, v, kring, state, Cshift, dt, lam, Bp, Cp, D, heads: int, pos: int,
                         out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One token (q, k, v: B x d_model) of the H3 mixer in recurrent form."""
    lib = _lib.load()
    B, dm = q.shape
    hd = dm // heads
    Cshift, dt, lam, Bp, Cp, D = _f32(Cshift), _f32(dt), _cpx(lam), _cpx(Bp), _cpx(Cp), _f32(D)
    N = lam.shape[1]
    S = Cshift.shape[1]
    if out is None:
        out = torch.empty_like(q)
    check(lib.h3_mixer_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(kring), _ptr(state), _ptr(Cshift), _ptr(dt),
                                   _ptr(lam), _ptr(Bp), _ptr(Cp), _ptr(D), _ptr(out), B, heads, hd, N, S, pos,
                                   _dtype(q), _stream()), "h3_mixer_decode_step")
    return out


def ssm_conv_workspace_bytes(H: int, L: int) -> int:
    return int(_lib.load().ssm_conv_workspace(H, L))


def ssm_conv_fwd(u, dt, lam, Bp, Cp, D, workspace: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Filter generation + fused FFT convolution in one call."""
    lib = _lib.load()
    B, H, L = u.shape
    dt, lam, Bp, Cp, D = _f32(dt), _cpx(lam), _cpx(Bp), _cpx(Cp), _f32(D)
    N = lam.shape[1]
    need = int(lib.ssm_conv_workspace(H, L))
    if workspace is None:
        workspace = _alloc_ws(need, u.device)
    if out is None:
        out = torch.empty_like(u)
    check(lib.ssm_conv_fwd(_ptr(u), _ptr(dt), _ptr(lam), _ptr(Bp), _ptr(Cp), _ptr(D), _ptr(out), B, H, L, N,
                           _ptr(workspace), workspace.numel() * workspace.element_size(), _dtype(u), _stream()),
          "ssm_conv_fwd")
    return out


def ssm_conv_fwd_noalloc(u, dt, lam, Bp, Cp, D, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """ssm_conv_fwd without a workspace: the filter goes to a fixed scratch
    array inside the library (H * L <= ssm_conv_noalloc_max_filter_floats())."""
    lib = _lib.load()
    B, H, L = u.shape
    dt, lam, Bp, Cp, D = _f32(dt), _cpx(lam), _cpx(Bp), _cpx(Cp), _f32(D)
    N = lam.shape[1]
    if out is None:
        out = torch.empty_like(u)
    st = lib.ssm_conv_fwd_noalloc(_ptr(u), _ptr(dt), _ptr(lam), _ptr(Bp), _ptr(Cp), _ptr(D), _ptr(out), B, H, L, N,
                                  _dtype(u), _stream())
    if st != _lib.FC_OK:
        raise _lib.FlashConvError(st, "ssm_conv_fwd_noalloc", lib.ssm_conv_noalloc_last_error().decode())
    return out


def statepass_workspace_bytes(B, H, L, N, chunk) -> int:
    return int(_lib.load().fftconv_statepass_workspace(B, H, L, N, chunk))


def fftconv_statepass(u, dt, lam, Bp, Cp, D, chunk: int, state_in: Optional[torch.Tensor] = None,
                      return_state: bool = False, workspace: Optional[torch.Tensor] = None,
                      out: Optional[torch.Tensor] = None):
    """Chunked state passing; returns y (and the final state B x H x N x 2 if
    return_state)."""
    lib = _lib.load()
    B, H, L = u.shape
    dt, lam, Bp, Cp, D = _f32(dt), _cpx(lam), _cpx(Bp), _cpx(Cp), _f32(D)
    N = lam.shape[1]
    need = int(lib.fftconv_statepass_workspace(B, H, L, N, chunk))
    if workspace is None:
        workspace = _alloc_ws(need, u.device)
    if out is None:
        out = torch.empty_like(u)
    sin = _cpx(state_in) if state_in is not None else None
    sout = torch.empty((B, H, N, 2), dtype=torch.float32, device=u.device) if return_state else None
    check(lib.fftconv_statepass(_ptr(u), _ptr(dt), _ptr(lam), _ptr(Bp), _ptr(Cp), _ptr(D), _ptr(out), B, H, L,
                                N, chunk, _ptr(sin), _ptr(sout), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _dtype(u), _stream()),
          "fftconv_statepass")
    return (out, sout) if return_state else out


def fftconv_statepass_bwd(dy, dt, lam, Bp, Cp, D, chunk: int, dstate_out: Optional[torch.Tensor] = None,
                          need_dstate_in: bool = False, workspace: Optional[torch.Tensor] = None,
                          out: Optional[torch.Tensor] = None):
    """Gradients of fftconv_statepass: du (and dstate_in, B x H x N x 2, if
    need_dstate_in) given dy and optionally dstate_out."""
    lib = _lib.load()
    B, H, L = dy.shape
    dt, lam, Bp, Cp, D = _f32(dt), _cpx(lam), _cpx(Bp), _cpx(Cp), _f32(D)
    N = lam.shape[1]
    need = int(lib.fftconv_statepass_bwd_workspace(B, H, L, N, chunk, _dtype(dy)))
    if workspace is None:
        workspace = _alloc_ws(need, dy.device)
    if out is None:
        out = torch.empty_like(dy)
    gin = _cpx(dstate_out) if dstate_out is not None else None
    gsin = torch.empty((B, H, N, 2), dtype=torch.float32, device=dy.device) if need_dstate_in else None
    check(lib.fftconv_statepass_bwd(_ptr(dy), _ptr(dt), _ptr(lam), _ptr(Bp), _ptr(Cp), _ptr(D), _ptr(out), B, H, L,
                                    N, chunk, _ptr(gin), _ptr(gsin), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _dtype(dy), _stream()),
          "fftconv_statepass_bwd")
    return (out, gsin) if need_dstate_in else out


def h3_mixer_workspace_bytes(B, L, heads, head_dim, N) -> int:
    return int(_lib.load().h3_mixer_workspace(B, L, heads, head_dim, N))


def h3_mixer_fwd(q, k, v, Cshift, dt, lam, Bp, Cp, D, heads: int, workspace: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """H3 mixer core O = Q (.) SSM_diag(SSM_shift(K) (.) V) per head; q, k, v:
    B x L x (heads*head_dim)."""
    lib = _lib.load()
    B, L, dm = q.shape
    hd = dm // heads
    Cshift, dt, lam, Bp, Cp, D = _f32(Cshift), _f32(dt), _cpx(lam), _cpx(Bp), _cpx(Cp), _f32(D)
    N = lam.shape[1]
    S = Cshift.shape[1]
    need = int(lib.h3_mixer_workspace(B, L, heads, hd, N))
    if workspace is None:
        workspace = _alloc_ws(need, q.device)
    if out is None:
        out = torch.empty_like(q)
    check(lib.h3_mixer_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(Cshift), _ptr(dt), _ptr(lam), _ptr(Bp), _ptr(Cp),
                           _ptr(D), _ptr(out), B, L, heads, hd, N, S, _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _dtype(q), _stream()),
          "h3_mixer_fwd")
    return out
