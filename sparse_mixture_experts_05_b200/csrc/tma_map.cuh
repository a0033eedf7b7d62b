// tma_map.cuh -- host-side encoding of TMA tensor maps for kernels outside the
// expert GEMMs (tma_map.cu).
#pragma once

#include <cuda.h>
#include <cstdint>

namespace moe {

// 3-D bf16 tensor map: dims innermost first, strides (bytes) of dims 1 and 2,
// box extents, 128-byte swizzle, coordinates past a dimension read as zeros.
// False when the driver entry point is missing or rejects the arguments.
bool make_bf16_map_3d(CUtensorMap* map, const void* base, const uint64_t (&dims)[3],
                      const uint64_t (&strides)[2], const uint32_t (&box)[3]);

}  // namespace moe
