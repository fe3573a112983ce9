"""Pins the tcgen05 building blocks (shared-memory descriptors, instruction
descriptor, tensor-memory accumulator layout) against a plain matrix product:
D = A B^T computed by one CTA on the tensor cores through the test hook
fc_selftest_umma.  Inputs are exactly representable in fp16/bf16 and the sums
are exact in fp32, so the comparison is bit-exact."""
import ctypes

import numpy as np
import pytest
import torch

from fft_long_convolution_flashconv_b200 import _lib

pytestmark = pytest.mark.gpu


def _hook():
    lib = _lib.load()
    fn = lib.fc_selftest_umma
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 3 + [ctypes.c_void_p]
    return fn


@pytest.mark.parametrize("N,K", [(16, 16), (64, 64), (128, 32), (256, 64), (96, 128), (256, 256)])
@pytest.mark.parametrize("bf16", [0, 1])
def test_umma_matches_matmul(N, K, bf16):
    assert torch.cuda.is_available()
    rng = np.random.default_rng(N * 1000 + K + bf16)
    # small integers: products and sums are exact in fp32
    A = rng.integers(-4, 5, size=(128, K)).astype(np.float32)
    B = rng.integers(-4, 5, size=(N, K)).astype(np.float32)
    dt = torch.bfloat16 if bf16 else torch.float16
    At = torch.tensor(A).to(dt).cuda().contiguous()
    Bt = torch.tensor(B).to(dt).cuda().contiguous()
    D = torch.full((128, N), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = _hook()(At.data_ptr(), Bt.data_ptr(), D.data_ptr(), err.data_ptr(), N, K, bf16,
                 torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 0, "MMA completion wait timed out"
    assert np.array_equal(D.cpu().numpy(), A @ B.T)


def _hook2():
    lib = _lib.load()
    fn = lib.fc_selftest_umma2
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 9 + [ctypes.c_void_p]
    return fn


# (a_mn, b_mn, a_lbo, a_sbo, b_lbo, b_sbo) as functions of (N, K)
LAYOUTS = {
    "kmajor_packed": lambda N, K: (0, 0, 128, (K // 8) * 128, 128, (K // 8) * 128),
    "kmajor_padded_lbo": lambda N, K: (0, 0, 144, (K // 8) * 144, 144, (K // 8) * 144),
    "kmajor_kouter": lambda N, K: (0, 0, 16 * 128, 128, (N // 8) * 128, 128),
    "b_mnmajor": lambda N, K: (0, 1, 128, (K // 8) * 128, (N // 8) * 128, 128),
    "a_mnmajor": lambda N, K: (1, 0, 16 * 128, 128, 128, (K // 8) * 128),
    "both_mnmajor_padded": lambda N, K: (1, 1, 16 * 144, 144, (N // 8) * 144, 144),
}


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("N,K,bf16", [(128, 64, 0), (256, 128, 1), (64, 32, 0)])
def test_umma_general_layouts(layout, N, K, bf16):
    rng = np.random.default_rng(N + K + len(layout))
    A = rng.integers(-4, 5, size=(128, K)).astype(np.float32)
    B = rng.integers(-4, 5, size=(N, K)).astype(np.float32)
    dt = torch.bfloat16 if bf16 else torch.float16
    At = torch.tensor(A).to(dt).cuda().contiguous()
    Bt = torch.tensor(B).to(dt).cuda().contiguous()
    D = torch.full((128, N), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    a_mn, b_mn, a_lbo, a_sbo, b_lbo, b_sbo = LAYOUTS[layout](N, K)
    rc = _hook2()(At.data_ptr(), Bt.data_ptr(), D.data_ptr(), err.data_ptr(), N, K, bf16, a_mn, b_mn, a_lbo,
                  a_sbo, b_lbo, b_sbo, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(D.cpu().numpy(), A @ B.T)
