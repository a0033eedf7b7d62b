// router.cuh -- host entry of the router kernel (router.cu).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/moe.h"

namespace moe {

// Logits (+ bias), top-k (ties -> lower expert id) and softmax over the k.
// cluster: CTAs that share one token tile's contraction (1, 2, 4 or 8; d is
// split into 8 * cluster ranges whose partial sums are added in order); 0 picks
// router_cluster(s).
// RMSNorm_2 of the block edge, fused into the router: x is then the residual
// stream U, the router works on u = bf16((U * inv) * gamma), inv = 1 / sqrt(
// mean_j U_j^2 + eps), and writes u [T, d] bf16 for the scatter.
struct RouterNorm {
    const void* gamma;  // [d] bf16
    float eps;
    void* u;            // [T, d] bf16 (out)
};

// status: the workspace status word (nullable); with clear_status the router
// zeroes it first (it is the first kernel of a forward), and an expired
// bounded wait of the streaming kernel is recorded there.
int launch_router(const moe_shape& s, const void* x, const void* Wg, const float* bias,
                  int32_t* idx, float* gate, float* logits, cudaStream_t stream, int cluster = 0,
                  const RouterNorm* norm = nullptr, int* status = nullptr,
                  bool clear_status = false);

// The cluster size launch_router picks for shape s (depends on T, d and the SM count).
int router_cluster(const moe_shape& s);

}  // namespace moe
