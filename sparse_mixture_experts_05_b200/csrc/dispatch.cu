// dispatch.cu -- per-expert token lists and the expert-sorted copy of x.
//
// Mixtral textbook page, section "Алгоритм": for each expert e, the
// (token, slot) pairs whose top-k list names e, taken in ascending token order,
// and the expert runs once over those tokens' rows.  Here the lists of all
// experts are laid end to end (offsets[e] .. offsets[e+1]-1), which is the order
// an exclusive scan of the per-expert counts produces.
//
// Two launches:
//  1. index kernel (one CTA of 1024 threads): each warp owns a contiguous run
//     of slots; warp-wide grouping by expert id (__match_any_sync) gives counts
//     and in-order ranks, one warp scans the per-warp counts into offsets and
//     starting positions, and a second pass hands out positions in token order.
//     Integer-only and deterministic (no atomics on positions).
//  2. scatter kernel: reads each x row once and writes it to its k sorted rows
//     (16-byte vector copies, one thread per 16-byte chunk).
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "dispatch.cuh"

namespace moe {
namespace dispatch {

constexpr int kIndexThreads = 1024;  // 32 warps
constexpr int kIndexWarps = kIndexThreads / 32;
constexpr int kMaxExperts = 32;
constexpr int kBatch = 8;  // groups of 32 slots whose ids are loaded together

// One CTA.  The T*k slots (slot j = t*k + s, ascending in t) are cut into 32
// contiguous runs, one per warp, taken 32 slots at a time.  In each group of
// 32 slots, __match_any_sync on the expert id gives every lane the lanes that
// chose the same expert: their number and this lane's rank among them (lane
// order = slot order).  Pass 1 sums the per-warp, per-expert counts; one warp
// turns them into offsets and per-warp starting positions (expert-major, then
// warp order); pass 2 repeats the grouping and hands out positions.  Stable
// (slot order within each expert), deterministic, no atomics.
__global__ void __launch_bounds__(kIndexThreads, 1)
    index_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                 int32_t* __restrict__ offsets, int32_t* __restrict__ perm_tok,
                 int32_t* __restrict__ inv, int* status_to_clear) {
    __shared__ int s_pos[kIndexWarps][kMaxExperts + 1];  // counts, then next positions
    __shared__ int s_total[kMaxExperts];                  // rows per expert
    __shared__ int s_base[kMaxExperts];                   // first sorted row of each expert
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    grid_dependency_wait();
    if (status_to_clear && tid == 0) *status_to_clear = 0;

    const int n = T * k;
    const int per_warp = ((n + kIndexWarps - 1) / kIndexWarps + 31) / 32 * 32;
    const int j0 = min(n, warp * per_warp);
    const int j1 = min(n, j0 + per_warp);
    const unsigned lt_mask = (1u << lane) - 1u;

    if (lane <= kMaxExperts) s_pos[warp][lane] = 0;
    __syncwarp();
    // pass 1: per-warp counts (the ids of kBatch groups are loaded before any is
    // used, so their load latencies overlap).  When the warp's run fits in one
    // batch (T*k <= 8192) pass 2 reuses the ids kept in registers.
    const bool one_batch = j1 - j0 <= 32 * kBatch;
    int kept[kBatch];
    for (int base = j0; base < j1; base += 32 * kBatch) {
        int ids[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int j = base + u * 32 + lane;
            ids[u] = j < j1 ? idx[j] : -1;
            kept[u] = ids[u];
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int e = ids[u];
            const bool valid = e >= 0 && e < E;
            const unsigned same = __match_any_sync(0xffffffffu, valid ? e : -1);
            if (valid && (same & lt_mask) == 0) s_pos[warp][e] += __popc(same);
            __syncwarp();
        }
    }
    __syncthreads();

    // offsets and per-warp starting positions: warp e scans expert e's counts
    // over the 32 warps (lane = warp), then warp 0 scans the experts' totals
    {
        int excl_w = 0;
        if (warp < E) {
            const int c = s_pos[lane][warp];
            int incl = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            excl_w = incl - c;  // rows of expert `warp` in warps before `lane`
            if (lane == 31) s_total[warp] = incl;
        }
        __syncthreads();
        if (warp == 0) {
            const int total = lane < E ? s_total[lane] : 0;
            int incl = total;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            if (lane < E) {
                s_base[lane] = incl - total;
                offsets[lane] = incl - total;
            }
            if (lane == 31) offsets[E] = incl;
        }
        __syncthreads();
        if (warp < E) s_pos[lane][warp] = s_base[warp] + excl_w;
    }
    __syncthreads();

    // pass 2: positions in slot order
    for (int base = j0; base < j1; base += 32 * kBatch) {
        int ids[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int j = base + u * 32 + lane;
            ids[u] = one_batch ? kept[u] : (j < j1 ? idx[j] : -1);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int j = base + u * 32 + lane;
            const bool in = j < j1;
            const int e = ids[u];
            const bool valid = e >= 0 && e < E;
            const unsigned same = __match_any_sync(0xffffffffu, valid ? e : -1);
            if (valid) {
                const int pos = s_pos[warp][e] + __popc(same & lt_mask);
                perm_tok[pos] = j / k;
                inv[j] = pos;
            } else if (in) {
                inv[j] = -1;
            }
            __syncwarp();
            if (valid && (same & lt_mask) == 0) s_pos[warp][e] += __popc(same);
            __syncwarp();
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
    if (s.E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
    return launch_pdl(index_kernel, dim3(1), dim3(kIndexThreads), 0, stream, idx, s.T, s.E, s.k,
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
