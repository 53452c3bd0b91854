// tma.h -- host-side creation of TMA tensor maps (cuTensorMapEncodeTiled,
// reached through the runtime's driver entry point so that the library does
// not link libcuda).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace ssm {

// Encodes a tiled tensor map of `rank` dims (innermost first).  `strides`
// holds rank-1 byte strides.  Returns false if the driver entry point is
// unavailable or the encoding is rejected.
bool encode_tiled(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *ptr,
                  const uint64_t *dims, const uint64_t *strides, const uint32_t *box,
                  CUtensorMapSwizzle swizzle);

}  // namespace ssm
