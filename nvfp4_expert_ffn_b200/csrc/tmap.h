// Host-side TMA tensor-map encoding (the driver's cuTensorMapEncodeTiled, looked up once
// through the runtime so the library needs no direct link to the driver library).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

namespace moe {

inline PFN_cuTensorMapEncodeTiled_v12000& tmap_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  return fn;
}

inline cudaError_t get_encode() {
  if (tmap_encode_fn()) return cudaSuccess;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess) return e;
  if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
  tmap_encode_fn() = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return cudaSuccess;
}

// Byte tensor of `rank` dims (dims[0] innermost, strides in bytes for dims 1..rank-1),
// copied in boxes of `box` elements with the given shared-memory swizzle.
inline cudaError_t encode_u8(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                             const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swizzle) {
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = tmap_encode_fn()(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void*>(base),
                                dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 16-bit element tensor (bf16 bits), same conventions as encode_u8 (strides in bytes).
inline cudaError_t encode_u16(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                              const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swizzle) {
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = tmap_encode_fn()(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, (cuuint32_t)rank, const_cast<void*>(base),
                                dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace moe
