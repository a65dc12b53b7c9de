// Host-side encoding of TMA tensor maps (cuTensorMapEncodeTiled, reached
// through the runtime's driver entry point so the library needs no -lcuda).
#pragma once

#include <cuda.h>

namespace kvq {

// Tiled map with 128-byte swizzle, zero fill out of bounds.  dims[0] is the
// innermost extent (elements), strides[i] the byte pitch of dimension i + 1,
// box the copied tile.  Returns false when the driver rejects the map.
bool make_tensor_map(CUtensorMap* m, CUtensorMapDataType type, void* base, int rank, const cuuint64_t* dims,
                     const cuuint64_t* strides, const cuuint32_t* box);

}  // namespace kvq
