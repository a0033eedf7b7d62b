// router.cu -- router logits, top-k selection and softmax over the selected k.
//
// Mixtral textbook page, section "Прямой проход в формулах": g = u W_r,
// S = TopK(g, k), w_i = exp(g_i) / sum_{j in S} exp(g_j); section "MoE изнутри":
// the softmax runs over the k selected logits only, in float32.
//
// The contraction x[T,d] . Wg[d,E] is skinny (E = 8) and HBM-bound on reading
// x once; it runs on mma.sync m16n8k16 (bf16 in, fp32 accumulate) so the issue
// slots stay free for loads.  A warp owns 16 tokens and 1/KSPLIT of d; the
// KSPLIT partial sums are added in a fixed order, so results are deterministic.
// KSPLIT grows when there are few tokens (decode) so that more warps share the
// one tile of 16 tokens and the kernel is not bound by one warp's load latency.
//
// k-permutation: a dot product may pair its terms in any order, so a lane loads
// 8 consecutive x elements (one 16-byte load) and feeds them to two MMAs as
// fragment positions {2t,2t+1,2t+8,2t+9}; the router weights are staged in
// shared memory in the matching order (one 16-byte load per lane per 32 k).
//
// Top-k: the four lanes of a quad hold the E logits of one token; k rounds of a
// quad-shuffle argmax pick the largest logit not yet taken, lower expert index
// first on ties (slot 0 = largest).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cfloat>
#include <climits>

#include "common.cuh"
#include "router.cuh"

namespace moe {
namespace router {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxK = 8;

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ bool better(float v, int id, float bv, int bid) {
    return v > bv || (v == bv && id < bid) || bid == INT_MAX;
}

template <int NT, int KSPLIT>
__global__ void __launch_bounds__(kThreads, 1)
    router_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ wg,
                  const float* __restrict__ bias, int T, int d, int E, int k,
                  int32_t* __restrict__ idx, float* __restrict__ gate,
                  float* __restrict__ logits) {
    constexpr int kSlots = kWarps / KSPLIT;  // token tiles of 16 per block iteration
    extern __shared__ uint4 s_wg[];  // [d/32][NT][32 lanes] x 8 bf16
    __shared__ float s_red[kSlots][KSPLIT][NT][32][4];
    grid_dependency_wait();

    // Stage W_r in fragment order: entry (kb, nt, lane) holds
    // Wg[kb*32 + (lane&3)*8 + j][nt*8 + (lane>>2)] for j = 0..7 (zero for n >= E),
    // i.e. element (r, n) goes to half-word r % 8 of entry
    // (r / 32, n / 8, (n % 8) * 4 + (r % 32) / 8).  Each thread reads whole rows
    // of W_r (16-byte loads when a row is a multiple of 16 bytes) and scatters
    // their elements; a warp's 32 consecutive rows land in one 64-byte span per
    // column, so the 2-byte shared stores do not conflict.
    uint16_t* s_half = reinterpret_cast<uint16_t*>(s_wg);
    auto put = [&](int r, int n, uint16_t v) {
        const int entry = ((r >> 5) * NT + (n >> 3)) * 32 + (n & 7) * 4 + ((r & 31) >> 3);
        s_half[entry * 8 + (r & 7)] = v;
    };
    if ((E & 7) == 0) {
        const int vec = E >> 3;  // 16-byte pieces per row
#pragma unroll 4
        for (int r = threadIdx.x; r < d; r += blockDim.x) {
            const uint4* row = reinterpret_cast<const uint4*>(wg + (int64_t)r * E);
            for (int q = 0; q < vec; ++q) {
                const uint4 v = __ldg(row + q);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    put(r, q * 8 + 2 * h, (uint16_t)(w[h] & 0xFFFFu));
                    put(r, q * 8 + 2 * h + 1, (uint16_t)(w[h] >> 16));
                }
            }
        }
    } else {
        for (int r = threadIdx.x; r < d; r += blockDim.x)
            for (int n = 0; n < NT * 8; ++n)
                put(r, n, n < E ? __ldg(wg + (int64_t)r * E + n) : (uint16_t)0);
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int slot = warp / KSPLIT;
    const int kq = warp % KSPLIT;
    const int g = lane >> 2;
    const int t4 = lane & 3;
    const int kper = d / KSPLIT;
    const int ntiles = (T + 15) / 16;

    for (int base = blockIdx.x * kSlots; base < ntiles; base += gridDim.x * kSlots) {
        const int tile = base + slot;
        float c[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0.f;
        if (tile < ntiles) {
            const int r0 = tile * 16 + g;
            const int r1 = r0 + 8;
            const bool v0 = r0 < T, v1 = r1 < T;
            const uint4* x0 = reinterpret_cast<const uint4*>(x + (int64_t)(v0 ? r0 : 0) * d);
            const uint4* x1 = reinterpret_cast<const uint4*>(x + (int64_t)(v1 ? r1 : 0) * d);
            const int kbeg = kq * kper, kend = kbeg + kper;
#pragma unroll 4
            for (int kb = kbeg; kb < kend; kb += 32) {
                const int ci = (kb >> 3) + t4;
                const uint4 a0 = v0 ? __ldg(x0 + ci) : make_uint4(0, 0, 0, 0);
                const uint4 a1 = v1 ? __ldg(x1 + ci) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint4 b = s_wg[((kb >> 5) * NT + nt) * 32 + lane];
                    mma_bf16_16816(c[nt], a0.x, a1.x, a0.y, a1.y, b.x, b.y);
                    mma_bf16_16816(c[nt], a0.z, a1.z, a0.w, a1.w, b.z, b.w);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) s_red[slot][kq][nt][lane][i] = c[nt][i];
        }
        __syncthreads();
        if (kq == 0 && tile < ntiles) {
            // v[nt][i]: token (i < 2 ? g : g+8), expert nt*8 + 2*t4 + (i & 1)
            float v[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float sum = s_red[slot][0][nt][lane][i];
#pragma unroll
                    for (int q = 1; q < KSPLIT; ++q) sum = __fadd_rn(sum, s_red[slot][q][nt][lane][i]);
                    const int n = nt * 8 + 2 * t4 + (i & 1);
                    if (bias && n < E) sum = __fadd_rn(sum, bias[n]);
                    v[nt][i] = sum;
                }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int row = tile * 16 + g + 8 * half;
                const bool rv = row < T;
                if (logits && rv) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int n = nt * 8 + 2 * t4 + j;
                            if (n < E) logits[(int64_t)row * E + n] = v[nt][2 * half + j];
                        }
                }
                uint32_t taken = 0;  // bit (nt*2 + j) of this lane's candidates
                float sel_v[kMaxK];
                int sel_id[kMaxK];
#pragma unroll
                for (int s = 0; s < kMaxK; ++s) {
                    if (s >= k) break;
                    float bv = -FLT_MAX;
                    int bid = INT_MAX;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int n = nt * 8 + 2 * t4 + j;
                            const int bit = nt * 2 + j;
                            const float cv = v[nt][2 * half + j];
                            if (n < E && !(taken & (1u << bit)) && better(cv, n, bv, bid)) {
                                bv = cv;
                                bid = n;
                            }
                        }
#pragma unroll
                    for (int off = 1; off <= 2; off <<= 1) {
                        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                        const int oid = __shfl_xor_sync(0xffffffffu, bid, off);
                        if (oid != INT_MAX && better(ov, oid, bv, bid)) {
                            bv = ov;
                            bid = oid;
                        }
                    }
                    // the lane that holds the winner marks it taken
                    if (bid != INT_MAX && ((bid & 7) >> 1) == t4)
                        taken |= 1u << ((bid >> 3) * 2 + (bid & 1));
                    sel_v[s] = bv;
                    sel_id[s] = bid;
                }
                if (rv && t4 == 0) {
                    const float m = sel_v[0];
                    float den = 0.f;
                    float ex[kMaxK];
#pragma unroll
                    for (int s = 0; s < kMaxK; ++s) {
                        if (s >= k) break;
                        ex[s] = expf(sel_v[s] - m);
                        den = __fadd_rn(den, ex[s]);
                    }
#pragma unroll
                    for (int s = 0; s < kMaxK; ++s) {
                        if (s >= k) break;
                        idx[(int64_t)row * k + s] = sel_id[s];
                        gate[(int64_t)row * k + s] = __fdiv_rn(ex[s], den);
                    }
                }
            }
        }
        __syncthreads();
    }
}

}  // namespace router

int router_ksplit(const moe_shape& s) {
    using namespace router;
    const int ntiles = (s.T + 15) / 16;
    const int sms = device_sm_count();
    // Largest split of d (into 16, 8 or 4 parts, each a whole number of 32-wide
    // k blocks) that still needs no more CTAs than there are SMs: few tokens
    // (decode) then get 16 warps per tile instead of 4.
    for (int cand : {16, 8}) {
        const int ctas = (ntiles * cand + kWarps - 1) / kWarps;
        if ((s.d / 32) % cand == 0 && ctas <= sms) return cand;
    }
    return 4;
}

int launch_router(const moe_shape& s, const void* x, const void* Wg, const float* bias,
                  int32_t* idx, float* gate, float* logits, cudaStream_t stream, int ksplit) {
    using namespace router;
    if (s.T == 0) return MOE_OK;
    const int NT = (s.E + 7) / 8;
    const size_t smem = (size_t)s.d * NT * 16;
    const int ntiles = (s.T + 15) / 16;
    const int sms = device_sm_count();
    // The split decides the order in which the partial sums of a logit are
    // added; a caller that runs one batch in token chunks passes the split of
    // the whole batch so every chunk rounds the same way.
    if (ksplit <= 0) ksplit = router_ksplit(s);
    if (ksplit != 4 && ksplit != 8 && ksplit != 16) return MOE_ERR_INVALID_ARG;
    if ((s.d / 32) % ksplit != 0) return MOE_ERR_INVALID_ARG;
    const int slots = kWarps / ksplit;
    const int grid = std::max(1, std::min(sms, (ntiles + slots - 1) / slots));
    const uint16_t* xp = static_cast<const uint16_t*>(x);
    const uint16_t* wp = static_cast<const uint16_t*>(Wg);
    auto run = [&](auto kern) {
        if (!ensure_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem))
            return MOE_ERR_CUDA;
        return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, stream, xp, wp, bias, s.T, s.d,
                          s.E, s.k, idx, gate, logits) == cudaSuccess
                   ? MOE_OK
                   : MOE_ERR_CUDA;
    };
#define MOE_ROUTER_CASE(N)                                                  \
    case N:                                                                 \
        return ksplit == 16 ? run(router_kernel<N, 16>)                     \
               : ksplit == 8 ? run(router_kernel<N, 8>) : run(router_kernel<N, 4>);
    switch (NT) {
        MOE_ROUTER_CASE(1)
        MOE_ROUTER_CASE(2)
        MOE_ROUTER_CASE(3)
        MOE_ROUTER_CASE(4)
        default:
            return MOE_ERR_UNSUPPORTED;
    }
#undef MOE_ROUTER_CASE
}

}  // namespace moe
