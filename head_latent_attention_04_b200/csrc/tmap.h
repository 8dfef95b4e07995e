// Host-side TMA tensor-map encoding through the driver entry point (no libcuda link).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "mla_internal.h"

namespace mla {

// Encodes a bf16 tiled tensor map of rank `rank` (dims[0] innermost, strides in
// bytes for dims 1..rank-1) with 128-byte (or 64-byte) swizzle and zero OOB fill.
mla_status_t encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                              const uint64_t* strides_bytes, const uint32_t* box,
                              CUtensorMapSwizzle swizzle);
// The same for bytes (8-bit codes).
mla_status_t encode_tmap_u8(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                            const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle);

}  // namespace mla
