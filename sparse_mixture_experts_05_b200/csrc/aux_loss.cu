// aux_loss.cu -- load-balancing auxiliary term of the router.
//
// Mixtral textbook page, section "Load-balancing loss": the training loss adds
// alpha * E * sum_{s<k} sum_{i<E} f_{s,i} P_i, where f_{s,i} is the fraction of
// (non-padding) tokens whose top-k slot s holds expert i and P_i is the mean over
// those tokens of the softmax over all E router logits; under uniform load the
// term equals alpha * k.  This kernel returns the term without alpha.
//
// One CTA of 1024 threads: thread i takes tokens i, i+1024, ...; slot counts are
// exact integers (per-warp counters, lanes with the same expert grouped by
// __match_any_sync, summed over warps at the end); the float32 sums of the
// softmax run per thread and then through a fixed butterfly and a fixed
// warp-order sum, so the result does not depend on scheduling.  The final
// combination runs in double on one thread.
#include <cuda_runtime.h>

#include <cmath>

#include "aux_loss.cuh"
#include "common.cuh"

namespace moe {
namespace aux {

constexpr int kThreads = 1024;
constexpr int kMaxE = 32;
constexpr int kMaxK = 8;

// EMAX >= E bounds the per-thread arrays (8, 16 or 32 experts).
template <int EMAX>
__global__ void __launch_bounds__(kThreads, 1)
    aux_loss_kernel(const float* __restrict__ logits, const int32_t* __restrict__ idx,
                    const uint8_t* __restrict__ mask, int T, int E, int k, float* aux_out,
                    float* f_out, float* P_out) {
    constexpr int kWarps = kThreads / 32;
    __shared__ int s_cnt[kWarps][kMaxK * EMAX];  // per-warp slot counts
    __shared__ float s_P[kWarps][EMAX];
    __shared__ int s_n[kWarps];
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    for (int i = lane; i < kMaxK * EMAX; i += 32) s_cnt[warp][i] = 0;
    __syncwarp();

    float P[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) P[e] = 0.f;
    int n = 0;
    const unsigned lt_mask = (1u << lane) - 1u;
    // thread tid takes tokens tid, tid + kThreads, ... (the loop runs warp-uniformly)
    for (int base = warp * 32; base < T; base += kThreads) {
        const int t = base + lane;
        const bool counted = t < T && (!mask || mask[t]);
        if (counted) {
            ++n;
            const float* g = logits + (int64_t)t * E;
            float gv[EMAX];
            float m = -INFINITY;
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                gv[e] = e < E ? g[e] : -INFINITY;
                m = fmaxf(m, gv[e]);
            }
            float ex[EMAX];
            float den = 0.f;
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                ex[e] = e < E ? expf(gv[e] - m) : 0.f;
                den = __fadd_rn(den, ex[e]);
            }
#pragma unroll
            for (int e = 0; e < EMAX; ++e) P[e] = __fadd_rn(P[e], __fdiv_rn(ex[e], den));
        }
        // slot counts: lanes choosing the same expert in slot s are counted by one
        for (int s = 0; s < k; ++s) {
            const int e = counted ? idx[(int64_t)t * k + s] : -1;
            const int key = (e >= 0 && e < E) ? e : -1;
            const unsigned same = __match_any_sync(0xffffffffu, key);
            if (key >= 0 && (same & lt_mask) == 0) s_cnt[warp][s * EMAX + key] += __popc(same);
            __syncwarp();
        }
    }
    // fixed butterfly inside the warp, then warps in index order
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) P[e] = __fadd_rn(P[e], __shfl_xor_sync(0xffffffffu, P[e], off));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
    if (lane == 0) {
#pragma unroll
        for (int e = 0; e < EMAX; ++e) s_P[warp][e] = P[e];
        s_n[warp] = n;
    }
    __syncthreads();
    if (tid == 0) {
        int total = 0;
        for (int w = 0; w < kWarps; ++w) total += s_n[w];
        double aux = 0.0;
        for (int e = 0; e < E; ++e) {
            float pe = 0.f;
            for (int w = 0; w < kWarps; ++w) pe = __fadd_rn(pe, s_P[w][e]);
            const double Pe = total > 0 ? (double)pe / total : 0.0;
            if (P_out) P_out[e] = (float)Pe;
            for (int s = 0; s < k; ++s) {
                int c = 0;
                for (int w = 0; w < kWarps; ++w) c += s_cnt[w][s * EMAX + e];
                const double fse = total > 0 ? (double)c / total : 0.0;
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
    if (s.E > aux::kMaxE || s.k > aux::kMaxK) return MOE_ERR_UNSUPPORTED;
    auto kern = s.E <= 8 ? aux::aux_loss_kernel<8>
                : (s.E <= 16 ? aux::aux_loss_kernel<16> : aux::aux_loss_kernel<32>);
    kern<<<1, aux::kThreads, 0, stream>>>(logits, idx, mask, s.T, s.E, s.k, aux_out, f_out, P_out);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
