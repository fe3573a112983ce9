// Instantiation of the CUDA-core fused FFT convolution (__half I/O, given filter); the kernel
// itself is in fftconv_impl.cuh.  Split over several translation units so the
// many fully unrolled radix stages compile in parallel.
#include "fftconv_impl.cuh"

namespace fc {
template cudaError_t launch_fftconv_dispatch<__half>(const __half*, const float*, int, SsmArgs, const float*, __half*,
                                               int, int, long long, int, int, int, cudaStream_t);
}  // namespace fc

FC_CHECK_READER(fc_check_fftconv_f16)
