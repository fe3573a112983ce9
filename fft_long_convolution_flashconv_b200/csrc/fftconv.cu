// Dispatch of the CUDA-core fused FFT convolution over the I/O types; the
// per-type instantiations live in fftconv_f32.cu, fftconv_f16.cu and
// fftconv_bf16.cu (kernel in fftconv_impl.cuh).
#include "kernels.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace fc {

template <typename T>
cudaError_t launch_fftconv_dispatch(const T* u, const float* f, int fstride, SsmArgs sp, const float* D, T* y, int B,
                                    int H, long long Lrow, int Lc, int C, int conj_filter, cudaStream_t st);

cudaError_t launch_fftconv(const void* u, const float* f, int fstride, SsmArgs sp, const float* D, void* y, int B,
                           int H, long long Lrow, int Lc, int C, int dtype, cudaStream_t st, int conj_filter) {
  switch (dtype) {
    case 0:
      return launch_fftconv_dispatch<float>((const float*)u, f, fstride, sp, D, (float*)y, B, H, Lrow, Lc, C, conj_filter, st);
    case 1:
      return launch_fftconv_dispatch<__half>((const __half*)u, f, fstride, sp, D, (__half*)y, B, H, Lrow, Lc, C,
                                             conj_filter, st);
    case 2:
      return launch_fftconv_dispatch<__nv_bfloat16>((const __nv_bfloat16*)u, f, fstride, sp, D,
                                                    (__nv_bfloat16*)y, B, H, Lrow, Lc, C, conj_filter, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fc
