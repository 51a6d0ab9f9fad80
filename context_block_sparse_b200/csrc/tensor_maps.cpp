// TMA tensor-map encoding for the tcgen05 kernels (host side).  The CUDA
// driver's cuTensorMapEncodeTiled is looked up through the runtime, so the
// library carries no link-time dependency on libcuda.
#include <cuda.h>
#include <cuda_runtime.h>

#include "splitkv_internal.h"

namespace splitkv {
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    cudaGetLastError();
    return EncodeTiledFn(nullptr);
  }();
  return fn;
}

}  // namespace

bool tensor_maps_available() { return encode_fn() != nullptr; }

bool make_bf16_map_3d(void* map, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint32_t box1,
                      uint32_t box2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {dim0, dim1, dim2};
  const cuuint64_t strides[2] = {dim0 * 2, dim0 * dim1 * 2};
  const cuuint32_t box[3] = {64, box1, box2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_bf16_store_map_3d(void* map, void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint32_t box1,
                            uint32_t box2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {dim0, dim1, dim2};
  const cuuint64_t strides[2] = {dim0 * 2, dim0 * dim1 * 2};
  const cuuint32_t box[3] = {32, box1, box2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_f32_map_3d(void* map, void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint32_t box0,
                     uint32_t box1, uint32_t box2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || (box0 * 4 != 64 && box0 * 4 != 128)) return false;
  const cuuint64_t dims[3] = {dim0, dim1, dim2};
  const cuuint64_t strides[2] = {dim0 * 4, dim0 * dim1 * 4};
  const cuuint32_t box[3] = {box0, box1, box2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, box0 * 4 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace splitkv
