// block.cuh -- host entry of the RMSNorm kernel (block.cu).
#pragma once

#include <cuda_runtime.h>

#include "../../include/moe.h"

namespace moe {

// u = bf16(U / sqrt(mean(U^2) + eps) * gamma), row by row.
int launch_rmsnorm(const moe_shape& s, const void* U, const void* gamma, float eps, void* u,
                   cudaStream_t stream);

}  // namespace moe
