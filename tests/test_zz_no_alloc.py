"""ssm_conv_fwd_noalloc, the entry point for callers that cannot allocate
device memory (its filter scratch is a fixed array inside the library).

Two calls in a row with different inputs, each checked against the fp64
oracle at the workload tolerances and against ssm_conv_fwd, which runs the
same kernels and must return the same bits.  This file is collected last on
purpose: a run that stops at its first failure has run every other test."""
import numpy as np
import pytest
import torch

from fft_long_convolution_flashconv_b200 import api
from fft_long_convolution_flashconv_b200 import workloads as W
from oracle import cref
from oracle import ssm_oracle as O

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "f16": 2e-2, "bf16": 2e-2}
TD = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def _dev(x, dt="f32"):
    return torch.tensor(np.asarray(x), dtype=torch.float64).to(TD[dt]).cuda().contiguous()


def _run(wl):
    p = [_dev(x) for x in (wl.dt, wl.lam, wl.Bp, wl.Cp, wl.D)]
    u = _dev(wl.u, wl.dtype)
    y_na = api.ssm_conv_fwd_noalloc(u, *p)
    torch.cuda.synchronize()
    a = y_na.double().cpu().numpy()
    y_ws = api.ssm_conv_fwd(u, *p)
    torch.cuda.synchronize()
    b = y_ws.double().cpu().numpy()
    f = O.ssm_filter(wl.dt, wl.lam, wl.Bp, wl.Cp, wl.L)
    ref = cref.causal_conv(wl.u, f, wl.D.astype(np.float64))
    return (O.row_rel_err(a.reshape(-1, wl.L), ref.reshape(-1, wl.L)),
            bool(np.array_equal(a, b)))


def test_noalloc_matches_oracle_twice():
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    # call 1: the full H3-layer-shaped workload (H * L = 786,432 of the 1,048,576 scratch floats),
    # 16-bit I/O at L = 1024: the tensor-core convolution
    wl1 = W.make("cfg2_conv_f16_B8_H768_L1024")
    err1, same1 = _run(wl1)
    assert err1 < TOL["f16"], err1
    assert same1
    # call 2, right after, with other inputs and a smaller filter: nothing of call 1 may leak in
    wl2 = W.make_conv(B=3, H=5, L=256, N=16, dtype="f32", seed=99)
    err2, same2 = _run(wl2)
    assert err2 < TOL["f32"], err2
    assert same2
