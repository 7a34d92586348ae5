// tmap.h -- host-side encoding of 2-D TMA tensor maps through the driver entry
// point (no link-time dependency on libcuda).
#pragma once

#include <cuda.h>
#include <cstdint>

namespace dsa {

// Encodes a row-major 2-D tensor [outer, inner] of `elem_bytes`-sized elements,
// `row_bytes` apart, copied in boxes of [box_outer, box_inner] with the given
// swizzle.  Out-of-range box elements read as zero.  Returns false on failure.
bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                  uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                  uint32_t box_outer, CUtensorMapSwizzle swizzle);

}  // namespace dsa
