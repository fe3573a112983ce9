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

// A rank-3 map of 16-bit elements (dims[0] contiguous) whose boxes land in
// shared memory with the 128-byte swizzle (box[0] * 2 must be 128 bytes):
// row r of a box occupies bytes [128 r, 128 r + 128) of the destination and
// its 16-byte chunk c sits at chunk c ^ (r % 8).  Zero fill outside the extents.
inline cudaError_t encode_map_3d_u16_sw128(CUtensorMap* m, const void* base, const cuuint64_t dims[3],
                                           const cuuint64_t strides[2], const cuuint32_t box[3]) {
  TensorMapEncodeTiled enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace fc
