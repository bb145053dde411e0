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

// Tensor of `rank` (<= 5) dimensions, innermost first: dims[i] elements,
// byte strides of dimensions 1..rank-1 (multiples of 16, in any order), a box
// of box[i] elements, no swizzle.  Out-of-range elements read as 0.
bool make_map_nd(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box);

}  // namespace qlora
