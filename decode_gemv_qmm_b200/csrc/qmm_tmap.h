// qmm_tmap.h -- host helper: encode a tiled TMA tensor map.
#pragma once

#include <cuda.h>

#include "qmm_internal.h"

namespace qmm {

// dims[0] is the contiguous dimension; strides_bytes[i] is the byte stride of
// dimension i + 1 (rank - 1 entries); box[i] elements per box in dimension i.
qmm_status encode_tiled(CUtensorMap *map, CUtensorMapDataType type, int rank, const void *base, const uint64_t *dims,
                        const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swizzle);

}  // namespace qmm
