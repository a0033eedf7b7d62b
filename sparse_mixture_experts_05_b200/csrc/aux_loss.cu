// aux_loss.cu -- load-balancing auxiliary term of the router.
//
// Mixtral textbook page, section "Load-balancing loss": the training loss adds
// alpha * E * sum_{s<k} sum_{i<E} f_{s,i} P_i, where f_{s,i} is the fraction of
// (non-padding) tokens whose top-k slot s holds expert i and P_i is the mean over
// those tokens of the softmax over all E router logits; under uniform load the
// term equals alpha * k.  This kernel returns the term without alpha.
//
// One CTA of 1024 threads: thread i takes tokens i, i+1024, ...; slot counts are
// exact integers (shared-memory atomics, order-free); the float32 sums of the
// softmax run per thread and then through a fixed butterfly and a fixed
// warp-order sum, so the result does not depend on scheduling.  The final
// combination runs in double on one thread.
#include <cuda_runtime.h>

#include "aux_loss.cuh"
#include "common.cuh"

namespace moe {
namespace aux {

constexpr int kThreads = 1024;
constexpr int kMaxE = 32;
constexpr int kMaxK = 8;

__global__ void __launch_bounds__(kThreads, 1)
    aux_loss_kernel(const float* __restrict__ logits, const int32_t* __restrict__ idx,
                    const uint8_t* __restrict__ mask, int T, int E, int k, float* aux_out,
                    float* f_out, float* P_out) {
    __shared__ int s_cnt[kMaxK * kMaxE];
    __shared__ float s_P[kThreads / 32][kMaxE];
    __shared__ int s_n[kThreads / 32];
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    for (int i = tid; i < kMaxK * kMaxE; i += kThreads) s_cnt[i] = 0;
    __syncthreads();

    float P[kMaxE];
#pragma unroll
    for (int e = 0; e < kMaxE; ++e) P[e] = 0.f;
    int n = 0;
    for (int t = tid; t < T; t += kThreads) {
        if (mask && !mask[t]) continue;
        ++n;
        const float* g = logits + (int64_t)t * E;
        float m = g[0];
        for (int e = 1; e < E; ++e) m = fmaxf(m, g[e]);
        float ex[kMaxE];
        float den = 0.f;
#pragma unroll
        for (int e = 0; e < kMaxE; ++e) {
            ex[e] = e < E ? expf(g[e] - m) : 0.f;
            den = __fadd_rn(den, ex[e]);
        }
#pragma unroll
        for (int e = 0; e < kMaxE; ++e) P[e] = __fadd_rn(P[e], __fdiv_rn(ex[e], den));
        for (int s = 0; s < k; ++s) {
            const int e = idx[(int64_t)t * k + s];
            if (e >= 0 && e < E) atomicAdd(&s_cnt[s * kMaxE + e], 1);
        }
    }
    // fixed butterfly inside the warp, then warps in index order
#pragma unroll
    for (int e = 0; e < kMaxE; ++e)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) P[e] = __fadd_rn(P[e], __shfl_xor_sync(0xffffffffu, P[e], off));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
    if (lane == 0) {
#pragma unroll
        for (int e = 0; e < kMaxE; ++e) s_P[warp][e] = P[e];
        s_n[warp] = n;
    }
    __syncthreads();
    if (tid == 0) {
        int total = 0;
        for (int w = 0; w < kThreads / 32; ++w) total += s_n[w];
        double aux = 0.0;
        for (int e = 0; e < E; ++e) {
            float pe = 0.f;
            for (int w = 0; w < kThreads / 32; ++w) pe = __fadd_rn(pe, s_P[w][e]);
            const double Pe = total > 0 ? (double)pe / total : 0.0;
            if (P_out) P_out[e] = (float)Pe;
            for (int s = 0; s < k; ++s) {
                const double fse = total > 0 ? (double)s_cnt[s * kMaxE + e] / total : 0.0;
                if (f_out) f_out[s * E + e] = (float)fse;
                aux += fse * Pe;
            }
        }
        aux_out[0] = (float)(aux * E);
    }
}

}  // namespace aux

int launch_aux_loss(const moe_shape& s, const float* logits, const int32_t* idx,
                    const uint8_t* mask, float* aux_out, float* f_out, float* P_out,
                    cudaStream_t stream) {
    aux::aux_loss_kernel<<<1, aux::kThreads, 0, stream>>>(logits, idx, mask, s.T, s.E, s.k,
                                                          aux_out, f_out, P_out);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
