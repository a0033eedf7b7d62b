// aux_loss.cuh -- host entry of the load-balancing term kernel (aux_loss.cu).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/moe.h"

namespace moe {

int launch_aux_loss(const moe_shape& s, const float* logits, const int32_t* idx,
                    const uint8_t* mask, float* aux_out, float* f_out, float* P_out,
                    cudaStream_t stream);

}  // namespace moe
