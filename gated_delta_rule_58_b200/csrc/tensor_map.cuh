// Host-side TMA descriptors (CUtensorMap) for the tiled tensor copies.
#pragma once

#include <cuda.h>  // CUtensorMap and its enums; the encoder is looked up from the driver at run time

#include "common.cuh"

namespace gdn {

// Encodes a 3-D tiled tensor map, by default with the 128-byte swizzle, and no
// out-of-bounds fill value (elements outside the tensor read as zero and are not
// written). dims and box are in elements, x innermost; strides are the byte
// strides of dims 1 and 2 (multiples of 16); base must be 16-byte aligned;
// box[0] * element size must be a multiple of 16 bytes and, with the swizzle, at
// most 128 bytes.
gdn_status_t make_tensor_map_3d(CUtensorMap* map, CUtensorMapDataType type, const void* base,
                                const uint64_t dims[3], const uint64_t strides[2], const uint32_t box[3],
                                const char* what, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);

}  // namespace gdn
