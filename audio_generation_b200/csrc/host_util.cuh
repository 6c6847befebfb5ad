#pragma once

#include <cuda.h>
#include <stdint.h>

namespace h3 {

// Encode a bf16 tiled tensor map with 128-byte swizzle and zero fill outside
// the tensor. dims/box innermost first; strides_bytes has rank - 1 entries.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box);

}  // namespace h3
