// block.cu -- the edges of the decoder block around the MoE layer.
//
// Mixtral textbook page, section "Прямой проход в формулах":
//     H = U + MoE(RMSNorm_2(U)),   RMSNorm(z) = z / sqrt(mean_j z_j^2 + eps) (.) gamma.
// rmsnorm_kernel writes the normalised rows u (bf16, the layer's input); the
// residual add is folded into the combine kernel (combine.cu).
//
// One warp per row: each lane sums the squares of its 8-element chunks in
// float32, a butterfly gives the row total, and the second pass scales the
// chunks by 1/sqrt(mean + eps) and gamma and rounds to bf16.  HBM-bound: U is
// read once and u written once.  For rows of up to 32 * kCached chunks (d <=
// 4096) a lane keeps its chunks in registers between the passes and issues all
// of its loads before it uses any; wider rows are read a second time (from L2).
#include <cuda_runtime.h>

#include <algorithm>

#include "block.cuh"
#include "common.cuh"

namespace moe {
namespace block {

constexpr int kCached = 16;  // 16-byte chunks a lane holds in registers

__device__ __forceinline__ float sum_squares(const uint4& v, float ss) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float lo = bf16_lo(w[j]), hi = bf16_hi(w[j]);
        ss = __fadd_rn(ss, __fmul_rn(lo, lo));
        ss = __fadd_rn(ss, __fmul_rn(hi, hi));
    }
    return ss;
}

__device__ __forceinline__ uint4 scale_row_chunk(const uint4& v, const uint4& g, float inv) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        r[j] = pack_bf16x2(__fmul_rn(__fmul_rn(bf16_lo(w[j]), inv), bf16_lo(gw[j])),
                           __fmul_rn(__fmul_rn(bf16_hi(w[j]), inv), bf16_hi(gw[j])));
    return make_uint4(r[0], r[1], r[2], r[3]);
}

__global__ void __launch_bounds__(256)
    rmsnorm_kernel(const uint4* __restrict__ U, const uint4* __restrict__ gamma, int T, int d8,
                   float eps, uint4* __restrict__ u) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const bool cached = d8 <= 32 * kCached;
    grid_dependency_wait();
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        const uint4* row = U + (int64_t)t * d8;
        uint4* out = u + (int64_t)t * d8;
        float ss = 0.f;
        if (cached) {
            uint4 v[kCached];
#pragma unroll
            for (int i = 0; i < kCached; ++i)
                if (lane + 32 * i < d8) v[i] = __ldg(row + lane + 32 * i);
#pragma unroll
            for (int i = 0; i < kCached; ++i)
                if (lane + 32 * i < d8) ss = sum_squares(v[i], ss);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
            const float inv =
                __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)(d8 * 8)), eps)));
#pragma unroll
            for (int i = 0; i < kCached; ++i) {
                const int c = lane + 32 * i;
                if (c < d8) out[c] = scale_row_chunk(v[i], __ldg(gamma + c), inv);
            }
        } else {
            for (int c = lane; c < d8; c += 32) ss = sum_squares(__ldg(row + c), ss);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
            const float inv =
                __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)(d8 * 8)), eps)));
            for (int c = lane; c < d8; c += 32)
                out[c] = scale_row_chunk(__ldg(row + c), __ldg(gamma + c), inv);
        }
    }
}

}  // namespace block

int launch_rmsnorm(const moe_shape& s, const void* U, const void* gamma, float eps, void* u,
                   cudaStream_t stream) {
    if (s.T == 0) return MOE_OK;
    const int grid = std::max(1, std::min((s.T + 7) / 8, device_sm_count() * 8));
    return launch_pdl(block::rmsnorm_kernel, dim3(grid), dim3(256), 0, stream,
                      static_cast<const uint4*>(U), static_cast<const uint4*>(gamma), s.T,
                      s.d / 8, eps, static_cast<uint4*>(u)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

}  // namespace moe
