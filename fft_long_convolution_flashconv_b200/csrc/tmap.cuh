// Tiled tensor maps (TMA descriptors) for 16-bit operand tiles, built on the
// host through the driver's cuTensorMapEncodeTiled entry point (looked up once
// through the runtime, so the library needs no link against libcuda).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

namespace fc {

typedef CUresult (*TensorMapEncodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                         const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                         CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                         CUtensorMapFloatOOBfill);

inline TensorMapEncodeTiled tensor_map_encoder() {
  static TensorMapEncodeTiled fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<TensorMapEncodeTiled>(p);
  }();
  return fn;
}

// A 5-d map of 16-bit elements with no swizzle and zero fill outside the
// extents: dims[0] is the contiguous one (stride 2 bytes); strides[i] is the
// byte stride of dims[i + 1] (multiples of 16, in any order).
inline cudaError_t encode_map_5d_u16(CUtensorMap* m, const void* base, const cuuint64_t dims[5],
                                     const cuuint64_t strides[4], const cuuint32_t box[5]) {
  TensorMapEncodeTiled enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace fc
