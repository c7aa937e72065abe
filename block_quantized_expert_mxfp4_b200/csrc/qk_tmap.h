// qk_tmap.h -- host-side encoding of TMA tensor maps (CUtensorMap), cached.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace qk {

// Encode (or fetch from the cache) a tiled tensor map.  rank 2 to 4;
// dtype is a CUtensorMapDataType, l2promo a CUtensorMapL2promotion (the L2
// fill granularity of the copy's DRAM requests).  Returns false on failure
// (map untouched).
bool tmap_get(CUtensorMap* out, int dtype, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box, int swizzle,
              int l2promo = CU_TENSOR_MAP_L2_PROMOTION_NONE);

}  // namespace qk
