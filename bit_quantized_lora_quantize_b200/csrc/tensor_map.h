// Host helper: 2-D TMA tensor maps through the driver entry point obtained
// from the runtime (no link-time dependency on libcuda).
#pragma once

#include <cstdint>
#include <cuda.h>

namespace qlora {

// Row-major [rows x inner] tensor with the given row stride (bytes); a box of
// [box_rows x box_inner] elements.  Out-of-range elements of a box read as 0.
// Returns false when the driver rejects the description.
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t inner, int64_t rows,
                 int64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle);

}  // namespace qlora
