// tmap.cuh -- TMA tensor-map encoding (host side).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace dsa {

// Encodes a tiled tensor map; dims[0] is the innermost (contiguous) extent,
// strides_bytes[i] is the byte stride of dimension i+1 (rank-1 entries).
// Out-of-range elements of a box read as zero.  Returns false on failure.
bool encode_tmap(CUtensorMap *map, CUtensorMapDataType dtype, uint32_t rank, const void *base,
                 const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                 CUtensorMapSwizzle swizzle);

}  // namespace dsa
