// dispatch.cu -- per-expert token lists and the expert-sorted copy of x.
//
// Mixtral textbook page, section "Алгоритм": for each expert e, the
// (token, slot) pairs whose top-k list names e, taken in ascending token order,
// and the expert runs once over those tokens' rows.  Here the lists of all
// experts are laid end to end (offsets[e] .. offsets[e+1]-1), which is the order
// an exclusive scan of the per-expert counts produces.
//
// Two launches:
//  1. index kernel (a cluster of 1 to 8 CTAs of 1024 threads, sized so each
//     warp owns a run of about 64 slots): each warp owns a contiguous run of
//     slots; warp-wide grouping by expert id (__match_any_sync) gives counts and
//     in-order ranks, the CTAs scan the per-warp counts (sharing their
//     per-expert totals through distributed shared memory) into offsets and
//     starting positions, and a second pass hands out positions in token order.
//     Integer-only and deterministic (no atomics on positions).
//  2. scatter kernel: reads each x row once and writes it to its k sorted rows
//     (16-byte vector copies, one thread per 16-byte chunk).
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "dispatch.cuh"
#include "sm100.cuh"

namespace moe {
namespace dispatch {

constexpr int kIndexThreads = 1024;  // 32 warps
constexpr int kIndexWarps = kIndexThreads / 32;
constexpr int kMaxExperts = 32;
constexpr int kBatch = 8;  // groups of 32 slots whose ids are loaded together
constexpr int kMaxIndexCluster = 8;
constexpr int kSlotsPerWarp = 64;  // target run length per warp when choosing the cluster size

__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ int ld_shared_cluster_s32(uint32_t addr) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// A cluster of C CTAs (C = 1 .. 8, chosen from T*k).  The T*k slots (slot
// j = t*k + s, ascending in t) are cut into 32 C contiguous runs, one per warp
// in cluster order (CTA rank, then warp), taken 32 slots at a time.  In each
// group of 32 slots, __match_any_sync on the expert id gives every lane the
// lanes that chose the same expert: their number and this lane's rank among
// them (lane order = slot order).  Pass 1 sums the per-warp, per-expert counts;
// warp e of every CTA scans expert e's counts over its 32 warps, the CTAs read
// each other's per-expert totals through distributed shared memory (so each
// knows the rows of every expert in earlier CTAs and in all), and the
// per-warp starting positions follow (expert-major, then slot order); pass 2
// repeats the grouping and hands out positions.  Stable (slot order within each
// expert), deterministic, no atomics.
__global__ void __launch_bounds__(kIndexThreads, 1)
    index_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                 int32_t* __restrict__ offsets, int32_t* __restrict__ perm_tok,
                 int32_t* __restrict__ inv) {
    __shared__ int s_pos[kIndexWarps][kMaxExperts + 1];  // counts, then next positions
    __shared__ int s_total[kMaxExperts];                  // this CTA's rows per expert
    __shared__ int s_base[kMaxExperts];                   // first row of each expert in this CTA
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int rank = (int)sm100::cluster_ctarank();
    const int C = (int)cluster_size();
    grid_dependency_wait();

    const int n = T * k;
    const int nwarps = kIndexWarps * C;
    const int gwarp = rank * kIndexWarps + warp;
    const int per_warp = ((n + nwarps - 1) / nwarps + 31) / 32 * 32;
    const int j0 = min(n, gwarp * per_warp);
    const int j1 = min(n, j0 + per_warp);
    const unsigned lt_mask = (1u << lane) - 1u;

    if (lane <= kMaxExperts) s_pos[warp][lane] = 0;
    __syncwarp();    // pass 1: per-warp counts (the ids of kBatch groups are loaded before any is
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
            if (base + u * 32 >= j1) break;  // warp-uniform: past the warp's run
            const int e = ids[u];
            const bool valid = e >= 0 && e < E;
            const unsigned same = __match_any_sync(0xffffffffu, valid ? e : -1);
            if (valid && (same & lt_mask) == 0) s_pos[warp][e] += __popc(same);
            __syncwarp();
        }
    }
    __syncthreads();

    // offsets and per-warp starting positions: warp e scans expert e's counts
    // over this CTA's 32 warps (lane = warp); then every CTA reads all CTAs'
    // totals: rows of expert e in earlier CTAs, and in all
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
            excl_w = incl - c;  // rows of expert `warp` in this CTA's warps before `lane`
            if (lane == 31) s_total[warp] = incl;
        }
        sm100::cluster_sync_all();
        if (warp == 0) {
            int before = 0, total = 0;  // rows of expert `lane` in earlier CTAs / in all
            if (lane < E) {
                const uint32_t src0 = sm100::smem_u32(&s_total[lane]);
                for (int c = 0; c < C; ++c) {
                    const int t = ld_shared_cluster_s32(sm100::map_to_cta(src0, (uint32_t)c));
                    if (c < rank) before += t;
                    total += t;
                }
            }
            int incl = total;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            const int expert_start = incl - total;
            if (lane < E) {
                s_base[lane] = expert_start + before;
                if (rank == 0) offsets[lane] = expert_start;
            }
            if (lane == 31 && rank == 0) offsets[E] = incl;
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
            if (base + u * 32 >= j1) break;  // warp-uniform: past the warp's run
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
    // no CTA leaves while another may still read its per-expert totals
    sm100::cluster_sync_all();
}

// x_sorted[inv[t, s]] = x[t] for every slot s of token t; one thread per
// (token, 16-byte chunk), so x is read once and the k copies are written with
// coalesced 16-byte stores however few tokens there are.  With `cnt`, the
// thread of every 16th chunk (the first of 128 columns) also zeroes that
// column chunk's counter.
__global__ void __launch_bounds__(256)
    scatter_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ inv, int T, int chunks,
                   int k, uint4* __restrict__ x_sorted, int* __restrict__ cnt) {
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
        if (cnt && (c & 15) == 0) cnt[(int64_t)t * (chunks >> 4) + (c >> 4)] = 0;
    }
}

}  // namespace dispatch

int launch_dispatch_index(const moe_shape& s, const int32_t* idx, int32_t* offsets,
                          int32_t* perm_tok, int32_t* inv, cudaStream_t stream) {
    using namespace dispatch;
    if (s.E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
    // cluster size: enough CTAs for runs of about kSlotsPerWarp slots per warp
    const int64_t n = (int64_t)s.T * s.k;
    int C = 1;
    while (C < kMaxIndexCluster && n > (int64_t)C * kIndexWarps * kSlotsPerWarp) C *= 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C);
    cfg.blockDim = dim3(kIndexThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, index_kernel, idx, s.T, s.E, s.k, offsets, perm_tok,
                              inv) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

int launch_dispatch_scatter(const moe_shape& s, const void* x, const int32_t* inv, void* x_sorted,
                            cudaStream_t stream, int* cnt) {
    using namespace dispatch;
    if (s.T == 0) return MOE_OK;
    const int64_t work = (int64_t)s.T * (s.d / 8);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256,
                                                                 (int64_t)device_sm_count() * 8));
    return launch_pdl(scatter_kernel, dim3(grid), dim3(256), 0, stream,
                      static_cast<const uint4*>(x), inv, s.T, s.d / 8, s.k,
                      static_cast<uint4*>(x_sorted), cnt) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

}  // namespace moe
