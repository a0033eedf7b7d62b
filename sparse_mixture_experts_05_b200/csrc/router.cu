// router.cu -- router logits, top-k selection and softmax over the selected k.
//
// Mixtral textbook page, section "Прямой проход в формулах": g = u W_r,
// S = TopK(g, k), w_i = exp(g_i) / sum_{j in S} exp(g_j); section "MoE изнутри":
// the softmax runs over the k selected logits only, in float32.
//
// The contraction x[T,d] . Wg[d,E] is skinny (E = 8) and HBM-bound on reading
// x once; it runs on mma.sync m16n8k16 (bf16 in, fp32 accumulate) so the issue
// slots stay free for loads.
//
// Work split.  A warp owns one tile of 16 tokens and a contiguous range of the
// 32-wide k blocks of d.  The d axis is cut into KS = 8 C ranges: the 8 warps of
// a CTA take 8 of them, and a cluster of C CTAs (C = 1, 2, 4 or 8) covers all
// of d for the same token tile.  C grows when there are few token tiles
// (decode: one tile over 8 CTAs) so that the loads spread over more SMs; each
// CTA stages only the W_r rows of its own k range.  The KS partial sums of a
// logit are added in range order by one warp of the cluster's first CTA, which
// reads the other CTAs' partials through distributed shared memory; the order
// depends only on C and d, so results are deterministic and a caller that runs
// one batch in token chunks can pass the whole batch's C.
//
// W_r staging.  Each warp copies the W_r rows of its own k range (8 experts =
// 16 bytes per row and 8-expert plane) as they are, with 16-byte asynchronous
// copies, into shared memory, row r of a 32-row k block at 16-byte slot
// r ^ (((r >> 3) & 3) << 1): the copy needs no registers, overlaps the warp's
// first x loads, and the warp waits only for its own copies.  B fragments come out of
// it with ldmatrix .trans, whose per-lane row addresses pick the rows in the
// order of the k permutation below; the slot swizzle makes the eight rows of
// every 8x8 matrix fall in distinct bank groups.
//
// k permutation: a dot product may pair its terms in any order, so a lane loads
// 8 consecutive x elements (one 16-byte load) and feeds them to two MMAs as
// fragment positions {2t,2t+1,2t+8,2t+9}; the B fragments are read in the same
// order (matrix m of a k block holds rows 8i + 2m + {0,1}, i = 0..3).
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
#include "sm100.cuh"
#include "tma_map.cuh"

namespace moe {
namespace router {

constexpr int kRoleRouter = 5;  // status role of the streaming kernel's waits

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxK = 8;
constexpr int kMaxCluster = 8;
constexpr int kGroup = 8;  // k blocks whose x loads are issued together

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t (&b)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3])
                 : "r"(addr));
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ float4 ld_shared_cluster_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

// RMSNorm helpers (block edge, see router_kernel's kNorm): the sum of squares of
// 8 bf16 values added in order to ss, and bf16((x * inv) * gamma) of 8 values.
__device__ __forceinline__ float sum_squares8(const uint4& v, float ss) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float lo = bf16_lo(w[j]), hi = bf16_hi(w[j]);
        ss = __fadd_rn(ss, __fmul_rn(lo, lo));
        ss = __fadd_rn(ss, __fmul_rn(hi, hi));
    }
    return ss;
}

__device__ __forceinline__ uint4 rms_scale8(const uint4& v, const uint4& gm, float inv) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const uint32_t gw[4] = {gm.x, gm.y, gm.z, gm.w};
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        r[j] = pack_bf16x2(__fmul_rn(__fmul_rn(bf16_lo(w[j]), inv), bf16_lo(gw[j])),
                           __fmul_rn(__fmul_rn(bf16_hi(w[j]), inv), bf16_hi(gw[j])));
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// 16-byte slot of row r (local to the CTA's staged range) of a W_r plane.
__device__ __forceinline__ int w_slot(int r) { return r ^ (((r >> 3) & 3) << 1); }

// Copies the W_r rows g0 + r0 .. g0 + r0 + nr - 1 of every 8-expert plane into
// shared memory (plane nt starts plane_rows 16-byte rows after plane nt - 1;
// local row r goes to slot w_slot(r)).  E a multiple of 8: 16-byte asynchronous
// copies, waited for with cp_async_wait_all; otherwise plain stores (experts
// past E read as zero).
template <int NT>
__device__ __forceinline__ void stage_wr(uint8_t* s_w, int plane_rows, int g0, int r0, int nr,
                                         const uint16_t* __restrict__ wg, int E, int lane) {
    if ((E & 7) == 0) {
        const uint32_t a = sm100::smem_u32(s_w);
        for (int i = lane; i < NT * nr; i += 32) {
            const int nt = i / nr;
            const int r = r0 + i - nt * nr;
            cp_async_16(a + (uint32_t)((nt * plane_rows + w_slot(r)) * 16),
                        wg + (int64_t)(g0 + r) * E + nt * 8);
        }
    } else {
        for (int i = lane; i < NT * nr * 8; i += 32) {
            const int j = i & 7;
            const int rest = i >> 3;
            const int nt = rest / nr;
            const int r = r0 + rest - nt * nr;
            const int n = nt * 8 + j;
            const uint16_t v = n < E ? wg[(int64_t)(g0 + r) * E + n] : (uint16_t)0;
            reinterpret_cast<uint16_t*>(s_w)[(nt * plane_rows + w_slot(r)) * 8 + j] = v;
        }
    }
}

__device__ __forceinline__ bool better(float v, int id, float bv, int bid) {
    return v > bv || (v == bv && id < bid) || bid == INT_MAX;
}

// Top-k of the logits v (fragment layout of the MMA accumulator: v[nt][i] is
// token row0 + (i < 2 ? g : g + 8), expert nt*8 + 2*t4 + (i & 1)), softmax over
// the k, and the stores of idx, gate and (optionally) the logits for the rows
// below row_end.  Kept out of line: it runs in one warp per tile, after the x
// loads' registers are dead.
template <int NT>
__device__ __noinline__ void select_and_store(float (&v)[NT][4], int row0, int row_end, int E,
                                              int k, int g, int t4, int32_t* __restrict__ idx,
                                              float* __restrict__ gate,
                                              float* __restrict__ logits) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int row = row0 + g + 8 * half;
        const bool rv = row < row_end;
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
            if (bid != INT_MAX && ((bid & 7) >> 1) == t4) taken |= 1u << ((bid >> 3) * 2 + (bid & 1));
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

// Dynamic shared memory: NT planes of W_r rows [rows_cap][16 bytes], then the
// partial sums [2 buffers][kWarps][32 lanes][NT] float4.
//
// kNorm (the block edge RMSNorm_2 of the Mixtral page's block equation, fused
// here because the router reads every row of its input anyway): x is the
// residual stream U, and the layer's input is u = bf16((U * inv) * gamma) with
// inv = 1 / sqrt(mean_j U_j^2 + eps) per row.  Per token tile, pass A reads the
// warp's k range and adds the squares per row (in order within a lane, then
// over the quad, then over the 8 C ranges in range order after a cluster
// barrier, every warp for its own rows); pass B reads the range again (from
// L2), forms u, writes it to u_out (the scatter's input) and feeds the same u to
// the MMAs.
template <int NT, bool kNorm>
__global__ void __launch_bounds__(kThreads, 2)
    router_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ wg,
                  const float* __restrict__ bias, int T, int d, int E, int k, int C,
                  int32_t* __restrict__ idx, float* __restrict__ gate,
                  float* __restrict__ logits, const uint16_t* __restrict__ gamma, float eps,
                  uint16_t* __restrict__ u_out, int* __restrict__ status_to_clear) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ float s_ss[kWarps][16];  // kNorm: per-warp sums of squares of the tile's rows
    // k blocks whose x loads are issued together (halved when normalising, which
    // holds more per lane: the scaled u and the gamma chunks)
    constexpr int kG = kNorm ? kGroup / 2 : kGroup;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int g = lane >> 2;
    const int t4 = lane & 3;
    const int rank = (int)sm100::cluster_ctarank();
    const int nkb = d >> 5;
    const int KS = C * kWarps;
    const int rows_cap = ((nkb + C - 1) / C) * 32;
    const int cta_kb0 = (rank * nkb) / C;
    const uint32_t s_w = sm100::smem_u32(smem);
    const uint32_t s_part = s_w + (uint32_t)(NT * rows_cap * 16);
    grid_dependency_wait();
    if (status_to_clear && blockIdx.x == 0 && tid == 0) *status_to_clear = 0;

    const int q = rank * kWarps + warp;          // this warp's k range
    const int kb_lo = (q * nkb) / KS;
    const int kb_hi = ((q + 1) * nkb) / KS;
    // Each warp stages the W_r rows of its own k range, plane by plane (8
    // experts per plane), so it waits only for its own copies (no block barrier).
    stage_wr<NT>(smem, rows_cap, cta_kb0 * 32, (kb_lo - cta_kb0) * 32, (kb_hi - kb_lo) * 32, wg,
                 E, lane);

    // ldmatrix: lane supplies row i = lane & 7 of matrix m = lane >> 3, i.e. row
    // 8 (i >> 1) + 2 m + (i & 1) of the k block
    const int lrow = 8 * ((lane & 7) >> 1) + 2 * (lane >> 3) + (lane & 1);
    const uint32_t lane_off = (uint32_t)(w_slot(lrow) * 16);
    const int ntiles = (T + 15) >> 4;
    const int cluster = blockIdx.x / C;
    const int nclusters = gridDim.x / C;

    int it = 0;
    for (int tile = cluster; tile < ntiles; tile += nclusters, ++it) {
        float c[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0.f;
        const int r0 = tile * 16 + g;
        const int r1 = r0 + 8;
        const bool v0 = r0 < T, v1 = r1 < T;
        const uint4* x0 = reinterpret_cast<const uint4*>(x + (int64_t)(v0 ? r0 : 0) * d) + t4;
        const uint4* x1 = reinterpret_cast<const uint4*>(x + (int64_t)(v1 ? r1 : 0) * d) + t4;
        float inv0 = 1.0f, inv1 = 1.0f;
        if constexpr (kNorm) {
            // pass A: sums of squares of rows r0 and r1 over this warp's range
            float ss0 = 0.0f, ss1 = 0.0f;
            for (int kb = kb_lo; kb < kb_hi; kb += kG) {
                const int n = min(kG, kb_hi - kb);
                uint4 a0[kG], a1[kG];
#pragma unroll
                for (int j = 0; j < kG; ++j) {
                    if (j < n) {
                        a0[j] = v0 ? __ldg(x0 + (kb + j) * 4) : make_uint4(0, 0, 0, 0);
                        a1[j] = v1 ? __ldg(x1 + (kb + j) * 4) : make_uint4(0, 0, 0, 0);
                    }
                }
#pragma unroll
                for (int j = 0; j < kG; ++j) {
                    if (j < n) {
                        ss0 = sum_squares8(a0[j], ss0);
                        ss1 = sum_squares8(a1[j], ss1);
                    }
                }
            }
            // the four lanes of a quad hold the same rows: fl(a+b) = fl(b+a), so
            // every lane of the quad gets the same bits
            ss0 = __fadd_rn(ss0, __shfl_xor_sync(0xffffffffu, ss0, 1));
            ss0 = __fadd_rn(ss0, __shfl_xor_sync(0xffffffffu, ss0, 2));
            ss1 = __fadd_rn(ss1, __shfl_xor_sync(0xffffffffu, ss1, 1));
            ss1 = __fadd_rn(ss1, __shfl_xor_sync(0xffffffffu, ss1, 2));
            if (t4 == 0) {
                s_ss[warp][g] = ss0;
                s_ss[warp][g + 8] = ss1;
            }
            sm100::cluster_sync_all();
            // the row totals over all 8 C ranges, in range order (loads of a CTA
            // issued together)
            float tot0 = 0.0f, tot1 = 0.0f;
            const uint32_t ss_base = sm100::smem_u32(&s_ss[0][0]);
            for (int cc = 0; cc < C; ++cc) {
                const uint32_t src = sm100::map_to_cta(ss_base, (uint32_t)cc);
#pragma unroll
                for (int w0 = 0; w0 < kWarps; w0 += 4) {
                    float p0[4], p1[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        p0[w] = ld_shared_cluster_f32(src + (uint32_t)(((w0 + w) * 16 + g) * 4));
                        p1[w] = ld_shared_cluster_f32(src + (uint32_t)(((w0 + w) * 16 + g + 8) * 4));
                    }
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        tot0 = (cc == 0 && w0 + w == 0) ? p0[w] : __fadd_rn(tot0, p0[w]);
                        tot1 = (cc == 0 && w0 + w == 0) ? p1[w] : __fadd_rn(tot1, p1[w]);
                    }
                }
            }
            inv0 = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot0, (float)d), eps)));
            inv1 = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot1, (float)d), eps)));
        }
        for (int kb = kb_lo, first = 1; first || kb < kb_hi; kb += kG, first = 0) {
            const int n = min(kG, kb_hi - kb);
            uint4 a0[kG], a1[kG];
#pragma unroll
            for (int j = 0; j < kG; ++j) {
                if (j < n) {
                    a0[j] = v0 ? __ldg(x0 + (kb + j) * 4) : make_uint4(0, 0, 0, 0);
                    a1[j] = v1 ? __ldg(x1 + (kb + j) * 4) : make_uint4(0, 0, 0, 0);
                }
            }
            if constexpr (kNorm) {
                // pass B: u = bf16((x * inv) * gamma), stored for the scatter
                const uint4* g4 = reinterpret_cast<const uint4*>(gamma) + t4;
                uint4* u0 = reinterpret_cast<uint4*>(u_out + (int64_t)(v0 ? r0 : 0) * d) + t4;
                uint4* u1 = reinterpret_cast<uint4*>(u_out + (int64_t)(v1 ? r1 : 0) * d) + t4;
#pragma unroll
                for (int j = 0; j < kG; ++j) {
                    if (j < n) {
                        const uint4 gm = __ldg(g4 + (kb + j) * 4);
                        a0[j] = rms_scale8(a0[j], gm, inv0);
                        a1[j] = rms_scale8(a1[j], gm, inv1);
                        if (v0) u0[(kb + j) * 4] = a0[j];
                        if (v1) u1[(kb + j) * 4] = a1[j];
                    }
                }
            }
            if (first && it == 0) {  // this warp's W_r rows must have landed
                cp_async_wait_all();
                __syncwarp();
            }
#pragma unroll
            for (int j = 0; j < kG; ++j) {
                if (j < n) {
                    const uint32_t blk = s_w + (uint32_t)((kb + j - cta_kb0) * 32 * 16) + lane_off;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        uint32_t b[4];
                        ldmatrix_x4_trans(blk + (uint32_t)(nt * rows_cap * 16), b);
                        mma_bf16_16816(c[nt], a0[j].x, a1[j].x, a0[j].y, a1[j].y, b[0], b[1]);
                        mma_bf16_16816(c[nt], a0[j].z, a1[j].z, a0[j].w, a1[j].w, b[2], b[3]);
                    }
                }
            }
        }
        // partial sums of this warp, then one cluster barrier per tile (the buffer
        // alternates: the reducing warp has read a buffer before it arrives at
        // the barrier after next, which every writer of that buffer waits for)
        float4* mine = reinterpret_cast<float4*>(smem + NT * rows_cap * 16) +
                       (((it & 1) * kWarps + warp) * 32 + lane) * NT;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mine[nt] = make_float4(c[nt][0], c[nt][1], c[nt][2], c[nt][3]);
        sm100::cluster_sync_all();
        if (rank == 0 && warp == 0) {
            // partial sums of ranges q = 0 .. KS-1, added left to right; the loads
            // of a batch of ranges are issued before any is added (a remote
            // shared-memory load takes hundreds of cycles)
            constexpr int kBatch = NT == 1 ? kWarps : (NT == 2 ? kWarps / 2 : kWarps / 4);
            float v[NT][4];
            const uint32_t buf = s_part + (uint32_t)(((it & 1) * kWarps * 32 + lane) * NT * 16);
            for (int cc = 0; cc < C; ++cc) {
                const uint32_t src = sm100::map_to_cta(buf, (uint32_t)cc);
#pragma unroll
                for (int w0 = 0; w0 < kWarps; w0 += kBatch) {
                    float4 p[kBatch][NT];
#pragma unroll
                    for (int w = 0; w < kBatch; ++w)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            p[w][nt] = ld_shared_cluster_f4(
                                src + (uint32_t)(((w0 + w) * 32 * NT + nt) * 16));
#pragma unroll
                    for (int w = 0; w < kBatch; ++w)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            if (cc == 0 && w0 + w == 0) {
                                v[nt][0] = p[w][nt].x; v[nt][1] = p[w][nt].y;
                                v[nt][2] = p[w][nt].z; v[nt][3] = p[w][nt].w;
                            } else {
                                v[nt][0] = __fadd_rn(v[nt][0], p[w][nt].x);
                                v[nt][1] = __fadd_rn(v[nt][1], p[w][nt].y);
                                v[nt][2] = __fadd_rn(v[nt][2], p[w][nt].z);
                                v[nt][3] = __fadd_rn(v[nt][3], p[w][nt].w);
                            }
                        }
                }
            }
            if (bias) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = nt * 8 + 2 * t4 + (i & 1);
                        if (n < E) v[nt][i] = __fadd_rn(v[nt][i], bias[n]);
                    }
            }
            select_and_store<NT>(v, tile * 16, min(T, tile * 16 + 16), E, k, g, t4, idx, gate,
                                 logits);
        }
    }
    cp_async_wait_all();
    // no CTA leaves while the reducing warp may still read its partial sums
    sm100::cluster_sync_all();
}

// ---------------------------------------------------------------------------
// Streaming kernel for batches with at least one 16-token tile per SM (where
// the cluster kernel runs at C = 1).  One CTA per SM, and the tokens are cut
// into tiles of hrows = ceil(T / (waves * CTAs)) <= 16 rows, so every SM reads
// nearly the same number of rows (16-row tiles left a third of the SMs with
// half the work at T = 4096).  A producer warp streams each tile's eight k
// ranges into a ring of shared-memory slots with TMA, one copy per slot: x is
// viewed in 3-D as [T rows][d / 64 chunks][64 columns], and a box of hrows rows
// by nbox = min(8, d / 512) chunks lands as hrows rows of nbox * 128 bytes
// (128-byte swizzle; rows past T read as zeros).  Small copies cost: the same
// bytes as 14-row boxes of one chunk each, eight copies per slot, ran slower
// than the cluster kernel.  Consumer warp q owns k range q of every tile, as warp q of the cluster
// kernel does at C = 1: the same W_r staging, the same A fragments (read from
// the swizzled slot instead of global memory), the same MMAs in the same k
// order and the same left-to-right sum over the ranges, so both kernels give a
// token the same bits.  Each consumer warp has its own ring of depth slots,
// so consecutive uses of a slot belong to one warp, which has consumed use u - 1
// before it waits for use u: with one ring shared by all warps, a warp that had
// run ahead could wait for use u of a slot whose use u - 1 had not landed yet,
// and the parity wait passed on the phase before.  The ranges' partial sums of a
// tile go to one of two shared-memory buffers, and an epilogue warp adds them,
// adds the bias and selects the top k while the consumers go on to the next
// tile (mbarriers in both directions; with the selection inside a loop bound by
// a per-tile barrier, a rotating warp doing it, the kernel ran no faster than
// the cluster kernel).  Every mbarrier wait is bounded; an expired one is
// recorded in the workspace status word (when given, with where it gave up in
// the words after it) and the kernel runs on to its end.
namespace stream {
constexpr int kConsumers = kWarps;             // warps 0-7: one per k range
constexpr int kProducer = kConsumers;          // warp 8: TMA
constexpr int kThreads = (kConsumers + 2) * 32;  // warp 9: sums, top k, stores
constexpr int kMaxDepth = 4;                   // ring slots per consumer warp
constexpr int kRowsMax = 16;                   // a slot holds up to 16 rows
constexpr int kBoxesPerStage = 8;              // chunks of 64 columns per slot at most
constexpr int kSmemLimit = 227 * 1024;
}  // namespace stream

struct StreamParams {
    const uint16_t* wg;
    const float* bias;
    int T, d, E, k;
    int hrows;       // rows per token tile (<= 16)
    int ntiles;      // ceil(T / hrows)
    int rb;          // 64-column chunks per k range (d / 512)
    int nbox;        // chunks per slot, min(8, rb); rb is a multiple of it
    int nch;         // ring stages per k range (rb / nbox)
    int depth;       // ring slots per consumer warp (slots = 8 * depth)
    int slot_bytes;  // kRowsMax * nbox * 128
    int32_t* idx;
    float* gate;
    float* logits;
    int* status;     // workspace status word (nullable)
    int clear;       // zero *status before anything else
    uint64_t timeout_ns;
    const uint16_t* gamma;  // RMSNorm_2 weights [d] (norm mode)
    float eps;
    uint16_t* u_out;        // u [T, d] (norm mode)
};

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// First expired wait of the launch: status word 1 = which wait (1 producer on a
// free slot, 2 consumer on a full slot, 3 consumer on a free partial buffer,
// 4 epilogue on a written partial buffer), word 2 = the stage or tile index,
// word 3 = the CTA, word 4 = the barrier's parity waited for.
__device__ __noinline__ void note_expired(int* status, int kind, int index, int parity) {
    if (status && atomicCAS(status + 1, 0, kind) == 0) {
        status[2] = index;
        status[3] = (int)blockIdx.x;
        status[4] = parity;
    }
}

// Barrier 1 among the consumer warps only (norm mode: the row sums of squares of
// a tile meet before any warp scales its range).
__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(stream::kConsumers * 32) : "memory");
}

// kNorm: the block edge's RMSNorm_2 as in router_kernel's norm mode, from the
// tile already in shared memory (one stage per k range, nch == 1): pass A adds
// the squares of the warp's range per row (in k order, then over the quad),
// the eight ranges' sums meet after one consumer barrier and are added in range
// order, and pass B scales the same shared-memory rows, stores u and feeds the
// MMAs -- the same operations in the same order as the cluster kernel, so u and
// the routing have the same bits in both.
template <int NT, bool kNorm>
__global__ void __launch_bounds__(stream::kThreads, 1)
    router_stream_kernel(const __grid_constant__ CUtensorMap tmx, const StreamParams p) {
    using namespace stream;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = sm100::smem_u32(smem_raw);
    const uint32_t s_x = (raw + 1023u) & ~1023u;  // 128-byte swizzle wants 1024-byte rows of 8
    uint8_t* smem = smem_raw + (s_x - raw);
    const int nslots = kConsumers * p.depth;
    uint8_t* s_wp = smem + nslots * p.slot_bytes;
    const uint32_t s_w = sm100::smem_u32(s_wp);
    float4* s_part = reinterpret_cast<float4*>(s_wp + NT * p.d * 16);
    float* s_ss = reinterpret_cast<float*>(s_part + 2 * kConsumers * 32 * NT);  // [2][8][16]
    uint64_t* full = reinterpret_cast<uint64_t*>(s_ss + 2 * kConsumers * 16);
    uint64_t* empty = full + nslots;
    uint64_t* pfull = empty + nslots;  // [2] a tile's partial sums written (one per consumer warp)
    uint64_t* pempty = pfull + 2;      // [2] a tile's partial sums read (the epilogue warp)
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < nslots; ++i) {
            sm100::mbar_init(&full[i], 1);
            sm100::mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            sm100::mbar_init(&pfull[i], kConsumers);
            sm100::mbar_init(&pempty[i], 1);
        }
        sm100::fence_barrier_init();
    }
    if (warp == kProducer && lane == 0) sm100::tma_prefetch_map(&tmx);
    __syncthreads();
    grid_dependency_wait();
    if (p.clear && p.status && blockIdx.x == 0 && threadIdx.x == 0) *p.status = 0;
    bool ok = true;

    if (warp == kProducer) {
        // stage n of consumer q (n = local tile * nch + chunk) goes to slot
        // q * depth + n % depth, its use n / depth; issued tile by tile, range by range
        if (lane == 0) {
            int it = 0;
            for (int tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x, ++it) {
                const int row0 = tile * p.hrows;
                for (int q = 0; q < kConsumers; ++q) {
                    for (int c = 0; c < p.nch; ++c) {
                        const int n = it * p.nch + c;
                        const int slot = q * p.depth + n % p.depth;
                        const int use = n / p.depth;
                        if (use > 0 && !sm100::mbar_wait(&empty[slot], (use - 1) & 1, p.timeout_ns)) {
                            ok = false;
                            note_expired(p.status, 1, n, (use - 1) & 1);
                        }
                        sm100::mbar_arrive_expect_tx(&full[slot],
                                                     (uint32_t)(p.nbox * p.hrows * 128));
                        sm100::tma_load_3d(smem + slot * p.slot_bytes, &tmx, &full[slot], 0,
                                           q * p.rb + c * p.nbox, row0);
                    }
                }
            }
        }
    } else if (warp < kConsumers) {
        const int q = warp;  // this warp's k range
        const int g = lane >> 2;
        const int t4 = lane & 3;
        const int range_kb = (p.d >> 5) / kConsumers;
        const int kb_lo = q * range_kb;
        stage_wr<NT>(s_wp, p.d, 0, kb_lo * 32, range_kb * 32, p.wg, p.E, lane);
        const int lrow = 8 * ((lane & 7) >> 1) + 2 * (lane >> 3) + (lane & 1);
        const uint32_t lane_off = (uint32_t)(w_slot(lrow) * 16);
        // lane (g, t4) reads 8 columns t4*8.. of a 32-column k block from rows g and
        // g + 8 of a slot: row r, chunk b is the 128-byte line r * nbox + b of the
        // slot, whose 16-byte piece u the swizzle moves to u ^ (line & 7); rows g
        // and g + 8 share that key (8 * nbox lines apart)
        const uint32_t pitch = (uint32_t)(p.nbox * 128);
        const uint32_t row_g = (uint32_t)g * pitch, row_g8 = (uint32_t)(g + 8) * pitch;
        int it = 0;
        for (int tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x, ++it) {
            float c[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0.f;
            for (int cc = 0; cc < p.nch; ++cc) {
                const int n = it * p.nch + cc;
                const int slot = q * p.depth + n % p.depth;
                const int par = (n / p.depth) & 1;
                if (!sm100::mbar_wait(&full[slot], par, p.timeout_ns)) {
                    ok = false;
                    note_expired(p.status, 2, n, par);
                }
                if (it == 0 && cc == 0) {  // this warp's W_r rows must have landed
                    cp_async_wait_all();
                    __syncwarp();
                }
                const uint32_t sx = s_x + (uint32_t)(slot * p.slot_bytes);
                const int kb0 = kb_lo + cc * p.nbox * 2;
                float inv0 = 1.0f, inv1 = 1.0f;
                if constexpr (kNorm) {
                    // pass A: this warp's range of rows g and g + 8
                    float ss0 = 0.0f, ss1 = 0.0f;
                    for (int b = 0; b < p.nbox; ++b) {
                        const uint32_t box = sx + (uint32_t)(b * 128);
                        const int key = (g * p.nbox + b) & 7;
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const uint32_t ch = (uint32_t)(((hh * 4 + t4) ^ key) * 16);
                            ss0 = sum_squares8(ld_shared_v4(box + row_g + ch), ss0);
                            ss1 = sum_squares8(ld_shared_v4(box + row_g8 + ch), ss1);
                        }
                    }
                    ss0 = __fadd_rn(ss0, __shfl_xor_sync(0xffffffffu, ss0, 1));
                    ss0 = __fadd_rn(ss0, __shfl_xor_sync(0xffffffffu, ss0, 2));
                    ss1 = __fadd_rn(ss1, __shfl_xor_sync(0xffffffffu, ss1, 1));
                    ss1 = __fadd_rn(ss1, __shfl_xor_sync(0xffffffffu, ss1, 2));
                    float* my_ss = s_ss + ((it & 1) * kConsumers + q) * 16;
                    if (t4 == 0) {
                        my_ss[g] = ss0;
                        my_ss[g + 8] = ss1;
                    }
                    // the buffer alternates per tile: a warp reads buffer it & 1
                    // before it reaches the next tile's barrier, which every
                    // writer of that buffer passes before writing it again
                    consumers_sync();
                    const float* all_ss = s_ss + (it & 1) * kConsumers * 16;
                    float tot0 = all_ss[g], tot1 = all_ss[g + 8];
#pragma unroll
                    for (int w = 1; w < kConsumers; ++w) {
                        tot0 = __fadd_rn(tot0, all_ss[w * 16 + g]);
                        tot1 = __fadd_rn(tot1, all_ss[w * 16 + g + 8]);
                    }
                    inv0 = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot0, (float)p.d), p.eps)));
                    inv1 = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot1, (float)p.d), p.eps)));
                }
                const int r0 = tile * p.hrows + g;
                const bool u0 = kNorm && g < p.hrows && r0 < p.T;
                const bool u1 = kNorm && g + 8 < p.hrows && r0 + 8 < p.T;
                for (int b = 0; b < p.nbox; ++b) {
                    const uint32_t box = sx + (uint32_t)(b * 128);
                    const int key = (g * p.nbox + b) & 7;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint32_t ch = (uint32_t)(((hh * 4 + t4) ^ key) * 16);
                        uint4 a0 = ld_shared_v4(box + row_g + ch);
                        uint4 a1 = ld_shared_v4(box + row_g8 + ch);
                        const int kb = kb0 + b * 2 + hh;
                        if constexpr (kNorm) {
                            // pass B: u = bf16((U * inv) * gamma), stored for the scatter
                            const uint4 gm = __ldg(reinterpret_cast<const uint4*>(p.gamma) + kb * 4 + t4);
                            a0 = rms_scale8(a0, gm, inv0);
                            a1 = rms_scale8(a1, gm, inv1);
                            uint4* urow = reinterpret_cast<uint4*>(p.u_out) + kb * 4 + t4;
                            if (u0) urow[(int64_t)r0 * (p.d / 8)] = a0;
                            if (u1) urow[(int64_t)(r0 + 8) * (p.d / 8)] = a1;
                        }
                        const uint32_t blk = s_w + (uint32_t)(kb * 32 * 16) + lane_off;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            uint32_t bf[4];
                            ldmatrix_x4_trans(blk + (uint32_t)(nt * p.d * 16), bf);
                            mma_bf16_16816(c[nt], a0.x, a1.x, a0.y, a1.y, bf[0], bf[1]);
                            mma_bf16_16816(c[nt], a0.z, a1.z, a0.w, a1.w, bf[2], bf[3]);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive(&empty[slot]);
            }
            // partial sums into buffer it & 1, once the epilogue has read what
            // tile it - 2 left there
            const int pb = it & 1;
            if (it >= 2 && !sm100::mbar_wait(&pempty[pb], ((it >> 1) - 1) & 1, p.timeout_ns)) {
                ok = false;
                note_expired(p.status, 3, it, ((it >> 1) - 1) & 1);
            }
            float4* mine = s_part + ((pb * kConsumers + q) * 32 + lane) * NT;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                mine[nt] = make_float4(c[nt][0], c[nt][1], c[nt][2], c[nt][3]);
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(&pfull[pb]);
        }
        cp_async_wait_all();  // (a warp without tiles still waits for its W_r copies)
    } else {
        // epilogue: the ranges' partial sums of each tile added left to right
        const int g = lane >> 2;
        const int t4 = lane & 3;
        int it = 0;
        for (int tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x, ++it) {
            const int pb = it & 1;
            if (!sm100::mbar_wait(&pfull[pb], (it >> 1) & 1, p.timeout_ns)) {
                ok = false;
                note_expired(p.status, 4, it, (it >> 1) & 1);
            }
            float v[NT][4];
            const float4* part = s_part + (pb * kConsumers * 32 + lane) * NT;
#pragma unroll
            for (int w = 0; w < kConsumers; ++w)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float4 pv = part[w * 32 * NT + nt];
                    if (w == 0) {
                        v[nt][0] = pv.x; v[nt][1] = pv.y; v[nt][2] = pv.z; v[nt][3] = pv.w;
                    } else {
                        v[nt][0] = __fadd_rn(v[nt][0], pv.x);
                        v[nt][1] = __fadd_rn(v[nt][1], pv.y);
                        v[nt][2] = __fadd_rn(v[nt][2], pv.z);
                        v[nt][3] = __fadd_rn(v[nt][3], pv.w);
                    }
                }
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(&pempty[pb]);  // free for tile it + 2
            if (p.bias) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = nt * 8 + 2 * t4 + (i & 1);
                        if (n < p.E) v[nt][i] = __fadd_rn(v[nt][i], p.bias[n]);
                    }
            }
            const int row0 = tile * p.hrows;
            select_and_store<NT>(v, row0, min(p.T, row0 + p.hrows), p.E, p.k, g, t4, p.idx,
                                 p.gate, p.logits);
        }
    }
    if (!ok) record_error(p.status, kDeviceTimeoutBase | kRoleRouter);
}

}  // namespace router

int router_cluster(const moe_shape& s) {
    using namespace router;
    const int ntiles = (s.T + 15) / 16;
    const int sms = device_sm_count();
    const int nkb = s.d / 32;
    // Largest cluster (1, 2, 4 or 8 CTAs per token tile) that keeps the grid
    // within two CTAs per SM and gives every warp at least one k block.
    int C = 1;
    while (C < kMaxCluster && (int64_t)ntiles * (2 * C) <= 2 * sms && 2 * C * kWarps <= nkb) C *= 2;
    return C;
}

namespace {

// Launch plan of the streaming kernel, or false where the cluster kernel runs:
// C > 1, fewer 16-token tiles than SMs, d not a multiple of 512 (a k range must
// be whole 64-column chunks, and up to 8 of them or a multiple of 8), W_r plus
// eight ring slots over the shared memory, or (norm mode) a k range of more than
// one slot.
struct StreamPlan {
    int ctas, hrows, ntiles, rb, nbox, nch, depth, slot_bytes;
    size_t smem;
};

bool stream_plan(const moe_shape& s, int C, bool norm, StreamPlan& pl) {
    using namespace router::stream;
    const int NT = (s.E + 7) / 8;
    if (C != 1 || s.d % 512 != 0) return false;
    const int sms = device_sm_count();
    const int t16 = (s.T + 15) / 16;
    if (sms <= 0 || t16 < sms) return false;
    const int waves = (t16 + sms - 1) / sms;
    pl.ctas = sms;
    pl.hrows = (s.T + waves * sms - 1) / (waves * sms);
    pl.ntiles = (s.T + pl.hrows - 1) / pl.hrows;
    pl.rb = s.d / 512;
    pl.nbox = std::min(kBoxesPerStage, pl.rb);
    if (pl.rb % pl.nbox != 0) return false;
    pl.nch = pl.rb / pl.nbox;
    if (norm && pl.nch != 1) return false;
    pl.slot_bytes = kRowsMax * pl.nbox * 128;
    // alignment slack, W_r planes, two buffers of partial sums, two of row sums
    // of squares, four mbarriers; each slot also takes two mbarriers; at least
    // one slot per warp
    const size_t fixed = 1024 + (size_t)NT * s.d * 16 +
                         (size_t)2 * kConsumers * 32 * NT * sizeof(float4) +
                         (size_t)2 * kConsumers * 16 * sizeof(float) + 4 * sizeof(uint64_t);
    if (fixed >= (size_t)kSmemLimit) return false;
    const size_t per_warp_slot = (size_t)kConsumers * (pl.slot_bytes + 16);
    pl.depth = (int)std::min<size_t>(kMaxDepth, ((size_t)kSmemLimit - fixed) / per_warp_slot);
    if (pl.depth < 1) return false;
    pl.smem = fixed + (size_t)pl.depth * per_warp_slot;
    return true;
}

}  // namespace

int launch_router(const moe_shape& s, const void* x, const void* Wg, const float* bias,
                  int32_t* idx, float* gate, float* logits, cudaStream_t stream, int cluster,
                  const RouterNorm* norm, int* status, bool clear_status) {
    using namespace router;
    if (s.T == 0) return MOE_OK;
    const int NT = (s.E + 7) / 8;
    // The cluster size fixes the order in which the partial sums of a logit are
    // added; a caller that runs one batch in token chunks passes the size chosen
    // for the whole batch so every chunk rounds the same way (both kernels add
    // them in the same order at C = 1).
    const int C = cluster <= 0 ? router_cluster(s) : cluster;
    if (C != 1 && C != 2 && C != 4 && C != 8) return MOE_ERR_INVALID_ARG;
    int* to_clear = clear_status ? status : nullptr;
    StreamPlan pl;
    if (stream_plan(s, C, norm != nullptr, pl)) {
        // x as [T][d / 64][64]: box of hrows rows by nbox 64-column chunks
        CUtensorMap tmx;
        const uint64_t dims[3] = {64, (uint64_t)s.d / 64, (uint64_t)s.T};
        const uint64_t strides[2] = {128, (uint64_t)s.d * 2};
        const uint32_t box[3] = {64, (uint32_t)pl.nbox, (uint32_t)pl.hrows};
        if (!make_bf16_map_3d(&tmx, x, dims, strides, box)) return MOE_ERR_CUDA;
        StreamParams p;
        p.wg = static_cast<const uint16_t*>(Wg);
        p.bias = bias;
        p.T = s.T;
        p.d = s.d;
        p.E = s.E;
        p.k = s.k;
        p.hrows = pl.hrows;
        p.ntiles = pl.ntiles;
        p.rb = pl.rb;
        p.nbox = pl.nbox;
        p.nch = pl.nch;
        p.depth = pl.depth;
        p.slot_bytes = pl.slot_bytes;
        p.idx = idx;
        p.gate = gate;
        p.logits = logits;
        p.status = status;
        p.clear = clear_status ? 1 : 0;
        p.timeout_ns = kDefaultWaitTimeoutNs;
        p.gamma = norm ? static_cast<const uint16_t*>(norm->gamma) : nullptr;
        p.eps = norm ? norm->eps : 0.0f;
        p.u_out = norm ? static_cast<uint16_t*>(norm->u) : nullptr;
        auto run_stream = [&](auto kern) {
            if (!ensure_dynamic_smem(reinterpret_cast<const void*>(kern), (int)pl.smem))
                return MOE_ERR_CUDA;
            return launch_pdl(kern, dim3(pl.ctas), dim3(stream::kThreads), pl.smem, stream, tmx,
                              p) == cudaSuccess
                       ? MOE_OK
                       : MOE_ERR_CUDA;
        };
#define MOE_STREAM_CASE(N)                                                              \
    case N:                                                                             \
        return norm ? run_stream(router_stream_kernel<N, true>)                         \
                    : run_stream(router_stream_kernel<N, false>);
        switch (NT) {
            MOE_STREAM_CASE(1)
            MOE_STREAM_CASE(2)
            MOE_STREAM_CASE(3)
            MOE_STREAM_CASE(4)
            default: return MOE_ERR_UNSUPPORTED;
        }
#undef MOE_STREAM_CASE
    }
    const int nkb = s.d / 32;
    const int rows_cap = ((nkb + C - 1) / C) * 32;
    const size_t smem = (size_t)NT * rows_cap * 16 + (size_t)2 * kWarps * 32 * NT * 16;
    const int ntiles = (s.T + 15) / 16;
    const int sms = device_sm_count();
    const int nclusters = std::max(1, std::min(ntiles, (2 * sms) / C));
    const uint16_t* xp = static_cast<const uint16_t*>(x);
    const uint16_t* wp = static_cast<const uint16_t*>(Wg);
    const uint16_t* gp = norm ? static_cast<const uint16_t*>(norm->gamma) : nullptr;
    const float eps = norm ? norm->eps : 0.0f;
    uint16_t* up = norm ? static_cast<uint16_t*>(norm->u) : nullptr;
    auto run = [&](auto kern) {
        if (!ensure_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem))
            return MOE_ERR_CUDA;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(nclusters * C);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
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
        return cudaLaunchKernelEx(&cfg, kern, xp, wp, bias, s.T, s.d, s.E, s.k, C, idx, gate,
                                  logits, gp, eps, up, to_clear) == cudaSuccess
                   ? MOE_OK
                   : MOE_ERR_CUDA;
    };
#define MOE_ROUTER_CASE(N)                                                              \
    case N:                                                                             \
        return norm ? run(router_kernel<N, true>) : run(router_kernel<N, false>);
    switch (NT) {
        MOE_ROUTER_CASE(1)
        MOE_ROUTER_CASE(2)
        MOE_ROUTER_CASE(3)
        MOE_ROUTER_CASE(4)
        default: return MOE_ERR_UNSUPPORTED;
    }
#undef MOE_ROUTER_CASE
}

}  // namespace moe
