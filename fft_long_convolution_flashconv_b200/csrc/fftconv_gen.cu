// Instantiation of the CUDA-core fused FFT convolution (filter generated inside the kernel, L >= 1024); the kernel
// itself is in fftconv_impl.cuh.  Split over several translation units so the
// many fully unrolled radix stages compile in parallel.
#include "fftconv_impl.cuh"

namespace fc {
template <typename T>
cudaError_t launch_fftconv_gen(const T* u, const float* f, int fstride, SsmArgs sp, const float* D, T* y, int B,
                               int H, long long Lrow, int Lc, int C, cudaStream_t st) {
  switch (Lc) {
    case 1024: return launch_fftconv_t<T, 11, true>(u, f, fstride, sp, D, y, B, H, Lrow, C, 0, st);
    case 2048: return launch_fftconv_t<T, 12, true>(u, f, fstride, sp, D, y, B, H, Lrow, C, 0, st);
    case 4096: return launch_fftconv_t<T, 13, true>(u, f, fstride, sp, D, y, B, H, Lrow, C, 0, st);
    case 8192: return launch_fftconv_t<T, 14, true>(u, f, fstride, sp, D, y, B, H, Lrow, C, 0, st);
    default: return cudaErrorInvalidValue;
  }
}
template cudaError_t launch_fftconv_gen<float>(const float*, const float*, int, SsmArgs, const float*, float*, int,
                                               int, long long, int, int, cudaStream_t);
template cudaError_t launch_fftconv_gen<__half>(const __half*, const float*, int, SsmArgs, const float*, __half*, int,
                                                int, long long, int, int, cudaStream_t);
template cudaError_t launch_fftconv_gen<__nv_bfloat16>(const __nv_bfloat16*, const float*, int, SsmArgs,
                                                       const float*, __nv_bfloat16*, int, int, long long, int, int,
                                                       cudaStream_t);
}  // namespace fc

FC_CHECK_READER(fc_check_fftconv_gen)
