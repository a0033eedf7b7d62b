// router.cuh -- host entry of the router kernel (router.cu).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/moe.h"

namespace moe {

// Logits (+ bias), top-k (ties -> lower expert id) and softmax over the k.
// ksplit: how many parts d is split into for the partial sums of a logit (4, 8
// or 16); 0 picks router_ksplit(s).
int launch_router(const moe_shape& s, const void* x, const void* Wg, const float* bias,
                  int32_t* idx, float* gate, float* logits, cudaStream_t stream, int ksplit = 0);

// The split launch_router picks for shape s (depends on T, d and the SM count).
int router_ksplit(const moe_shape& s);

}  // namespace moe
