"""B200-native (sm_100a) diagonal-SSM long convolution of H3 / FlashConv.

The compute lives in libflashconv_b200.so (C ABI, include/flashconv.h);
``api`` holds thin PyTorch wrappers and ``_lib`` the raw ctypes binding.
Import them explicitly (``from fft_long_convolution_flashconv_b200 import
api``); importing the package itself loads nothing.
"""
__all__ = ["api", "workloads"]
