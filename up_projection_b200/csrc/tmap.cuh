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

}  // namespace swiglu
