// dispatch.cuh -- host entries of the dispatch kernels (dispatch.cu).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/moe.h"

namespace moe {

// offsets [E+1], perm_tok [T*k], inv [T,k] from idx [T,k].
int launch_dispatch_index(const moe_shape& s, const int32_t* idx, int32_t* offsets,
                          int32_t* perm_tok, int32_t* inv, cudaStream_t stream);

// x_sorted[inv[t,s]] = x[t].  `cnt` (nullable, [T, d / 128] int32) is zeroed
// on the way: the counters of a combine fused into the down projection.
int launch_dispatch_scatter(const moe_shape& s, const void* x, const int32_t* inv, void* x_sorted,
                            cudaStream_t stream, int* cnt = nullptr);

}  // namespace moe
