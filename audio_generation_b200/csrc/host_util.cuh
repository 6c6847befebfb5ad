#pragma once

#include <cuda.h>
#include <stdint.h>

namespace h3 {

// Encode a bf16 tiled tensor map with 128-byte swizzle and zero fill outside
// the tensor. dims/box innermost first; strides_bytes has rank - 1 entries.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box);
// Same for any element type (the e4m3 GEMM operands use UINT8).
bool make_tmap(CUtensorMap* map, const void* base, CUtensorMapDataType type, int rank,
               const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box);

}  // namespace h3
