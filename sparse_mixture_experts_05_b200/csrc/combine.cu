// combine.cu -- gate-weighted un-permute of the expert outputs.
//
// Mixtral textbook page, section "Алгоритм": each token's output accumulates
// the gate-weighted outputs of the experts it was routed to -- exactly k terms.
// Each token's terms are gathered from their sorted rows and added in slot
// order: products and sums are separately rounded float32 operations (no fused
// multiply-add), so the result does not depend on scheduling and needs no
// atomics; y is rounded once to bf16 (nearest even).  Each thread produces 8
// columns of one token (two 16-byte loads per term, one 16-byte store).
#include <cuda_runtime.h>

#include <algorithm>

#include "combine.cuh"
#include "combine_math.cuh"
#include "common.cuh"

namespace moe {
namespace combine {

// One thread per (token, 8-column chunk): at small T this spreads the few rows
// over the whole GPU instead of one warp per row.  All of a thread's inverse-map
// and gate loads are issued first, then all of its expert-row loads, so the
// row loads do not wait on each other.  KMAX >= k bounds the slot arrays (2 for
// the common top-2, 8 otherwise).
template <int KMAX>
__global__ void __launch_bounds__(256)
    combine_kernel(const float4* __restrict__ o, const int32_t* __restrict__ inv,
                   const float* __restrict__ gate, int T, int d8, int k,
                   const uint4* __restrict__ residual, uint4* __restrict__ y) {
    grid_dependency_wait();
    const int64_t total = (int64_t)T * d8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int t = (int)(i / d8);
        const int c = (int)(i - (int64_t)t * d8);
        int rows[KMAX];
        float gs[KMAX];
#pragma unroll
        for (int s = 0; s < KMAX; ++s) {
            rows[s] = s < k ? __ldg(inv + (int64_t)t * k + s) : -1;
            gs[s] = s < k ? __ldg(gate + (int64_t)t * k + s) : 0.f;
        }
        float4 v[KMAX][2];
#pragma unroll
        for (int s = 0; s < KMAX; ++s) {
            // a skipped slot (row < 0) reads row 0, which always exists, and is ignored
            const float4* src = o + ((int64_t)(rows[s] < 0 ? 0 : rows[s]) * d8 + c) * 2;
            if (s < k) {
                v[s][0] = __ldg(src);
                v[s][1] = __ldg(src + 1);
            }
        }
        float vv[KMAX][8];
#pragma unroll
        for (int s = 0; s < KMAX; ++s) {
            if (s >= k) break;
            const float f[8] = {v[s][0].x, v[s][0].y, v[s][0].z, v[s][0].w,
                                v[s][1].x, v[s][1].y, v[s][1].z, v[s][1].w};
#pragma unroll
            for (int j = 0; j < 8; ++j) vv[s][j] = f[j];
        }
        float res[8], out[8];
        if (residual) {
            const uint4 r = __ldg(residual + i);
            const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                res[2 * j] = bf16_lo(w[j]);
                res[2 * j + 1] = bf16_hi(w[j]);
            }
        }
        combine_columns<KMAX, 8>(vv, gs, rows, k, residual != nullptr, res, out);
        y[i] = make_uint4(pack_bf16x2(out[0], out[1]), pack_bf16x2(out[2], out[3]),
                          pack_bf16x2(out[4], out[5]), pack_bf16x2(out[6], out[7]));
    }
}

}  // namespace combine

int launch_combine(const moe_shape& s, const float* o, const int32_t* inv, const float* gate,
                   void* y, cudaStream_t stream, const void* residual) {
    using namespace combine;
    if (s.T == 0) return MOE_OK;
    const int64_t work = (int64_t)s.T * (s.d / 8);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256,
                                                                 (int64_t)device_sm_count() * 8));
    auto kern = s.k <= 2 ? combine_kernel<2> : combine_kernel<8>;
    return launch_pdl(kern, dim3(grid), dim3(256), 0, stream, reinterpret_cast<const float4*>(o),
                      inv, gate, s.T, s.d / 8, s.k, static_cast<const uint4*>(residual),
                      static_cast<uint4*>(y)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

}  // namespace moe
