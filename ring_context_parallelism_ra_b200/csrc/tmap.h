// TMA tensor-map construction (host).  The driver's cuTensorMapEncodeTiled is
// fetched once through the runtime's driver-entry-point query, so the library
// does not link libcuda directly.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace ra {

// 3-D bf16 map over [heads][rows][d] with arbitrary row / head strides (bytes,
// multiples of 16), box = [1][box_rows][box_d], 128-byte swizzle, zero fill
// outside the tensor.  Returns 0 on success.
int make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d, uint64_t rows,
                      uint64_t heads, uint64_t row_stride_bytes, uint64_t head_stride_bytes,
                      uint32_t box_d, uint32_t box_rows);

}  // namespace ra
