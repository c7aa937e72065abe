// qk_tmap.h -- host-side encoding of TMA tensor maps (CUtensorMap), cached.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace qk {

// Encode (or fetch from the cache) a tiled tensor map.  rank 2 or 3;
// dtype is a CUtensorMapDataType.  Returns false on failure (map untouched).
bool tmap_get(CUtensorMap* out, int dtype, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box, int swizzle);

}  // namespace qk
