// dispatch.cu -- per-expert token lists and the expert-sorted copy of x.
//
// Mixtral textbook page, section "Алгоритм": for each expert e,
// (tok, slot) = where(topk_idx == e) lists the tokens that chose e in ascending
// token order, and the expert runs once over X[tok].  Here the lists of all
// experts are laid end to end (offsets[e] .. offsets[e+1]-1), which is the order
// an exclusive scan of the per-expert counts produces.
//
// Two launches:
//  1. index kernel (one CTA of 1024 threads): thread i owns a contiguous run of
//     tokens; per-thread per-expert counts, an exclusive scan over threads for
//     each expert, then each thread walks its run again and hands out positions
//     in token order.  Integer-only and deterministic (no atomics on positions).
//  2. scatter kernel: reads each x row once and writes it to its k sorted rows
//     (16-byte vector copies, one thread per 16-byte chunk).
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "dispatch.cuh"

namespace moe {
namespace dispatch {

constexpr int kIndexThreads = 1024;

__device__ __forceinline__ int warp_inclusive_scan(int v, int lane) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
    }
    return v;
}

__global__ void __launch_bounds__(kIndexThreads, 1)
    index_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                 int32_t* __restrict__ offsets, int32_t* __restrict__ perm_tok,
                 int32_t* __restrict__ inv, int* status_to_clear) {
    extern __shared__ int s_cnt[];  // [E][1024]: entries of expert e in thread i's run
    __shared__ int s_total[32];
    __shared__ int s_base[33];
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    grid_dependency_wait();
    if (status_to_clear && tid == 0) *status_to_clear = 0;

    const int per = (T + kIndexThreads - 1) / kIndexThreads;
    const int t_begin = min(T, tid * per);
    const int t_end = min(T, t_begin + per);

    for (int e = 0; e < E; ++e) s_cnt[e * kIndexThreads + tid] = 0;
    for (int t = t_begin; t < t_end; ++t)
        for (int s = 0; s < k; ++s) {
            const int e = idx[(int64_t)t * k + s];
            if (e >= 0 && e < E) s_cnt[e * kIndexThreads + tid] += 1;
        }
    __syncthreads();

    // Exclusive scan over threads (= over token runs in order), one warp per expert.
    if (warp < E) {
        int carry = 0;
        for (int c = 0; c < kIndexThreads; c += 32) {
            const int v = s_cnt[warp * kIndexThreads + c + lane];
            const int incl = warp_inclusive_scan(v, lane);
            s_cnt[warp * kIndexThreads + c + lane] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) s_total[warp] = carry;
    }
    __syncthreads();
    if (tid == 0) {
        s_base[0] = 0;
        for (int e = 0; e < E; ++e) s_base[e + 1] = s_base[e] + s_total[e];
        for (int e = 0; e <= E; ++e) offsets[e] = s_base[e];
    }
    __syncthreads();

    for (int e = 0; e < E; ++e) s_cnt[e * kIndexThreads + tid] += s_base[e];
    for (int t = t_begin; t < t_end; ++t)
        for (int s = 0; s < k; ++s) {
            const int64_t j = (int64_t)t * k + s;
            const int e = idx[j];
            if (e >= 0 && e < E) {
                const int pos = s_cnt[e * kIndexThreads + tid]++;
                perm_tok[pos] = t;
                inv[j] = pos;
            } else {
                inv[j] = -1;
            }
        }
}

// x_sorted[inv[t, s]] = x[t] for every slot s of token t; one thread per
// (token, 16-byte chunk), so x is read once and the k copies are written with
// coalesced 16-byte stores however few tokens there are.
__global__ void __launch_bounds__(256)
    scatter_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ inv, int T, int chunks,
                   int k, uint4* __restrict__ x_sorted) {
    grid_dependency_wait();
    const int64_t total = (int64_t)T * chunks;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int t = (int)(i / chunks);
        const int c = (int)(i - (int64_t)t * chunks);
        const uint4 v = __ldg(x + i);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            if (s >= k) break;
            const int dst = __ldg(inv + (int64_t)t * k + s);
            if (dst >= 0) x_sorted[(int64_t)dst * chunks + c] = v;
        }
    }
}

}  // namespace dispatch

int launch_dispatch_index(const moe_shape& s, const int32_t* idx, int32_t* offsets,
                          int32_t* perm_tok, int32_t* inv, int* status_to_clear,
                          cudaStream_t stream) {
    using namespace dispatch;
    const size_t smem = (size_t)s.E * kIndexThreads * sizeof(int);
    if (!ensure_dynamic_smem(reinterpret_cast<const void*>(index_kernel), (int)smem))
        return MOE_ERR_CUDA;
    return launch_pdl(index_kernel, dim3(1), dim3(kIndexThreads), smem, stream, idx, s.T, s.E, s.k,
                      offsets, perm_tok, inv, status_to_clear) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

int launch_dispatch_scatter(const moe_shape& s, const void* x, const int32_t* inv, void* x_sorted,
                            cudaStream_t stream) {
    using namespace dispatch;
    if (s.T == 0) return MOE_OK;
    const int64_t work = (int64_t)s.T * (s.d / 8);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256,
                                                                 (int64_t)device_sm_count() * 8));
    return launch_pdl(scatter_kernel, dim3(grid), dim3(256), 0, stream,
                      static_cast<const uint4*>(x), inv, s.T, s.d / 8, s.k,
                      static_cast<uint4*>(x_sorted)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

}  // namespace moe
