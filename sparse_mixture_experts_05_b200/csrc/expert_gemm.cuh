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
//
// With `fuse` (nullable) and combine_fusable(s), GEMM2 also forms y = sum over
// slots of gate * o (plus the residual) in its epilogue, the combine kernel's
// result bit for bit, and no combine is needed.  fuse->cnt ([T, d / 128] int32)
// must be zero at launch; every slot of every token must have a row (a routed
// batch).  combine_fused(s) says whether fusing pays on this device (it needs
// several rounds of GEMM2's CTA-pair tiles).
struct FusedCombine {
    const int32_t* perm_tok = nullptr;  // [R] token of each sorted row
    const int32_t* inv = nullptr;       // [T, k] sorted row of each (token, slot)
    const float* gate = nullptr;        // [T, k]
    const void* residual = nullptr;     // [T, d] bf16, or nullptr
    void* y = nullptr;                  // [T, d] bf16
    int* cnt = nullptr;                 // [T, d / 128], zero at launch
};

// Whether expert_gemms can fuse the combine into GEMM2 for this shape, and
// whether the forward does (queries the device's SM count).
bool combine_fusable(const moe_shape& s);
bool combine_fused(const moe_shape& s);

int expert_gemms(const moe_shape& s, const void* x_sorted, const int32_t* offsets, const void* W1,
                 const void* W3, const void* W2, void* h, float* o, int* err,
                 uint64_t timeout_ns, int stall_after, cudaStream_t stream,
                 void* mid_event, const float* b1 = nullptr, const float* b3 = nullptr,
                 const float* b2 = nullptr, const FusedCombine* fuse = nullptr);

}  // namespace moe
