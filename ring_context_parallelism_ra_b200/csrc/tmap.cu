#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "tmap.h"

namespace ra {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

int make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d, uint64_t rows,
                      uint64_t heads, uint64_t row_stride_bytes, uint64_t head_stride_bytes,
                      uint32_t box_d, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return -1;
  cuuint64_t dims[3] = {d, rows, heads};
  cuuint64_t strides[2] = {row_stride_bytes, head_stride_bytes};
  cuuint32_t box[3] = {box_d, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -2;
}

}  // namespace ra
