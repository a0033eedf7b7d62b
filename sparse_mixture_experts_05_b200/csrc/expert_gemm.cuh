// expert_gemm.cuh -- host entry of the grouped expert GEMMs (expert_gemm.cu).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/moe.h"

namespace moe {

// Runs GEMM1 (x_sorted W1 | x_sorted W3 -> h = SiLU(a) (.) b, bf16) and GEMM2
// (h W2 -> o, fp32) over the expert groups described by `offsets`.
// `err` is the device status word; `stall_after` >= 0 makes the producer stop
// after that many pipeline stages (test of the bounded-wait error path).
// `mid_event` (a cudaEvent_t, nullable) is recorded between GEMM1 and GEMM2.
// b1, b3 [E, d_ff] and b2 [E, d] (float32, each nullable) are the biases of the
// expert Linear layers: a = x W1 + b1, b = x W3 + b3, o = h W2 + b2.
int expert_gemms(const moe_shape& s, const void* x_sorted, const int32_t* offsets, const void* W1,
                 const void* W3, const void* W2, void* h, float* o, int* err,
                 uint64_t timeout_ns, int stall_after, cudaStream_t stream,
                 void* mid_event, const float* b1 = nullptr, const float* b3 = nullptr,
                 const float* b2 = nullptr);

}  // namespace moe
