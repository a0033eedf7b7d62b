// router.cuh -- host entry of the router kernel (router.cu).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/moe.h"

namespace moe {

// Logits (+ bias), top-k (ties -> lower expert id) and softmax over the k.
int launch_router(const moe_shape& s, const void* x, const void* Wg, const float* bias,
                  int32_t* idx, float* gate, float* logits, cudaStream_t stream);

}  // namespace moe
