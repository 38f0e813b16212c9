// tmap.cuh -- host-side TMA tensor-map encoding.  cuTensorMapEncodeTiled is
// fetched once through cudaGetDriverEntryPoint, so the library does not link
// libcuda directly.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace swiglu {

// Encode a 2-D row-major tensor [outer, inner] (inner contiguous) whose rows
// are `row_bytes` apart, to be moved in boxes of [box_outer, box_inner].
// Returns false if the driver entry point is missing or rejects the map.
bool encode_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype,
                    uint64_t inner, uint64_t outer, uint64_t row_bytes,
                    uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

// Encode a 3-D tensor: dims {d0, d1, d2} (d0 contiguous), byte strides of
// dims 1 and 2 (in either order of size), moved in boxes of {b0, b1, b2};
// the box lands in shared memory as [b2][b1][b0].
bool encode_tmap_3d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype,
                    uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
                    uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2,
                    CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE);

// Encode a 4-D tensor (dims[0] contiguous; byte strides of dims 1..3 in any
// order of size), moved in boxes `box`; the box lands as
// [box[3]][box[2]][box[1]][box[0]].
bool encode_tmap_4d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype,
                    const uint64_t dims[4], const uint64_t strides_bytes[3],
                    const uint32_t box[4], CUtensorMapSwizzle swizzle);

}  // namespace swiglu
