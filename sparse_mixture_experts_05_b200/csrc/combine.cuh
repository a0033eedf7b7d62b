// combine.cuh -- host entry of the combine kernel (combine.cu).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/moe.h"

namespace moe {

// y[t] = bf16( sum over slots s, in order, of gate[t,s] * o[inv[t,s]] ), plus
// residual[t] (bf16, nullable) added in float32 before the rounding.
int launch_combine(const moe_shape& s, const float* o, const int32_t* inv, const float* gate,
                   void* y, cudaStream_t stream, const void* residual = nullptr);

}  // namespace moe
