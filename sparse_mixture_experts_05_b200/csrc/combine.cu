// combine.cu -- gate-weighted un-permute of the expert outputs.
//
// Mixtral textbook page, section "Алгоритм": Y.index_add_(0, tok,
// W[tok, slot] * Expert_e(X[tok])) -- every token receives exactly k terms.
// Each token's terms are gathered from their sorted rows and added in slot
// order: products and sums are separately rounded float32 operations (no fused
// multiply-add), so the result does not depend on scheduling and needs no
// atomics; y is rounded once to bf16 (nearest even).  One warp per token row,
// 8 columns (two 16-byte loads per term, one 16-byte store) per lane step.
#include <cuda_runtime.h>

#include <algorithm>

#include "combine.cuh"
#include "common.cuh"

namespace moe {
namespace combine {

__global__ void __launch_bounds__(256)
    combine_kernel(const float4* __restrict__ o, const int32_t* __restrict__ inv,
                   const float* __restrict__ gate, int T, int d8, int k, uint4* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        int row[8];
        float g[8];
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            row[s] = s < k ? inv[(int64_t)t * k + s] : -1;
            g[s] = s < k ? gate[(int64_t)t * k + s] : 0.f;
        }
        for (int c = lane; c < d8; c += 32) {
            float acc[8];
            bool first = true;
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                if (s >= k) break;
                if (row[s] < 0) continue;
                const float4* src = o + ((int64_t)row[s] * d8 + c) * 2;
                const float4 v0 = __ldg(src);
                const float4 v1 = __ldg(src + 1);
                const float p[8] = {__fmul_rn(g[s], v0.x), __fmul_rn(g[s], v0.y),
                                    __fmul_rn(g[s], v0.z), __fmul_rn(g[s], v0.w),
                                    __fmul_rn(g[s], v1.x), __fmul_rn(g[s], v1.y),
                                    __fmul_rn(g[s], v1.z), __fmul_rn(g[s], v1.w)};
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = first ? p[j] : __fadd_rn(acc[j], p[j]);
                first = false;
            }
            if (first) {
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = 0.f;
            }
            y[(int64_t)t * d8 + c] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                                pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
        }
    }
}

}  // namespace combine

int launch_combine(const moe_shape& s, const float* o, const int32_t* inv, const float* gate,
                   void* y, cudaStream_t stream) {
    using namespace combine;
    if (s.T == 0) return MOE_OK;
    const int grid = std::max(1, std::min((s.T + 7) / 8, device_sm_count() * 8));
    combine_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(o), inv, gate, s.T,
                                             s.d / 8, s.k, static_cast<uint4*>(y));
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
