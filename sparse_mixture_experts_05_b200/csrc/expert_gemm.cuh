// expert_gemm.cuh -- host entry of the grouped expert GEMMs (expert_gemm.cu).
#pragma once

#include <cuda.h>
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

// 3-D bf16 tensor map (dims innermost first, strides in bytes of dims 1 and 2),
// 128-byte swizzle, coordinates past a dimension read as zeros.
bool make_bf16_map_3d(CUtensorMap* map, const void* base, const uint64_t (&dims)[3],
                      const uint64_t (&strides)[2], const uint32_t (&box)[3]);

}  // namespace moe
