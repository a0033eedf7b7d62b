// expert_gemm.cu -- grouped expert GEMMs on the 5th-generation tensor cores.
//
// The experts of the MoE layer (Mixtral textbook page, section "Прямой проход в
// формулах": Expert_i(u) = (SiLU(u W_gate^i) (.) u W_up^i) W_down^i) run over
// the expert-sorted rows produced by dispatch (section "Алгоритм": each expert
// receives all of its tokens in one call; an expert with no tokens is skipped).
//
// Two launches of one persistent, warp-specialised kernel:
//   GEMM1 (kSwiGLU):  A = x_sorted [R, d],  B = W1[e] | W3[e]  ->  h = SiLU(a) (.) b, bf16
//   GEMM2 (kDown):    A = h        [R, d_ff], B = W2[e]        ->  o (fp32)
//
// Tile: 128 rows (one TMEM lane per row) x 256 accumulator columns.  For GEMM1
// the 256 columns are 128 columns of x W1 followed by the same 128 columns of
// x W3, so the SwiGLU product is formed in the epilogue straight out of TMEM.
// K advances 64 elements (one 128-byte swizzle row) per pipeline stage.
//
// Roles (192 threads, one CTA per SM):
//   warp 0      TMA producer: per stage one copy per weight matrix (a 3-D box
//               filling 64 x 64 MN-major boxes, see make_weight_map), issued
//               first, then the A box [128 x 64] (K-major)
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 2..5  epilogue: tcgen05.ld -> SiLU(.) / convert -> TMA stores of 32 x 32 chunks
// Shared-memory stages are recycled through full/empty mbarriers; the two TMEM
// accumulator buffers (2 x 256 columns) let the epilogue of tile i overlap the
// MMAs of tile i+1.  The producer and MMA stage loops are on the critical path
// (every stage waits for a load round trip), so they are kept short: the abort
// flag is read only after a slow wait, descriptors are derived by addition.
// Tiles are dealt evenly to the CTAs (deal_tiles); the CTA-pair variant for the
// down projection is described further below.
//
// Weights stay in their natural row-major layout ([E, d, d_ff] and
// [E, d_ff, d]); the B operand is read MN-major, which tcgen05 supports for
// 16-bit types, so no repacking pass exists.
//
// Ragged groups: a tile starts at an expert's first row + 128*m and may run
// past the expert's last row into the next expert's rows (or past R, where TMA
// fills zeros); those rows are computed and discarded (stores are predicated).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "combine_math.cuh"
#include "expert_gemm.cuh"
#include "sm100.cuh"

namespace moe {
namespace gemm {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kBoxN = 64;
constexpr int kMaxBoxes = 4;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;                          // 16 KB
constexpr int kBBoxBytes = kBK * kBoxN * 2;                     // 8 KB
constexpr int kStageBytes = kABytes + kMaxBoxes * kBBoxBytes;   // 48 KB
constexpr int kAccCols = 256;
constexpr int kTmemCols = 2 * kAccCols;
constexpr int kThreads = 192;
constexpr int kMaxE = 32;
constexpr int kEpiBufBytes = 4096;                              // 32 rows x 128 bytes
constexpr int kEpiWarpBytes = 2 * kEpiBufBytes;                 // two staging buffers
constexpr int kEpiBytes = 4 * kEpiWarpBytes;                    // four epilogue warps
constexpr int kOutBox = 32;                                     // output box: 32 x 32
constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + kEpiBytes + 1024;

struct Params {
    const int32_t* offsets;  // [E+1]
    void* out;               // GEMM1: bf16 h [R, n_out]; GEMM2: float o [R, n_out]
    int* err;                // device status word
    uint64_t timeout_ns;
    int E;
    int K;                   // contraction length
    int n_out;               // output columns
    int n_tile_out;          // output columns per tile
    int n_boxes;             // B boxes per stage (MMA N = 64 * n_boxes)
    int stall_after;         // test hook: producer stops after this many stages (-1: never)
    int group_m;             // m-tiles per rasterisation group (see decode_tile_rows)
    const float* bias_a;     // GEMM1: b1 [E, n_out]; GEMM2: b2 [E, n_out]; or nullptr
    const float* bias_b;     // GEMM1: b3 [E, n_out]; or nullptr
    int halves_inline;       // pair kernel: half tiles in place (1) or after all full tiles (0)
    // GEMM2 on CTA pairs with the combine fused (y non-null): besides o, each
    // token's 128-column chunks of y, finished by whichever of its k row tiles
    // stores last (see finish_tokens)
    const int32_t* perm_tok;  // [R] token of each sorted row
    const int32_t* inv;       // [T, k] sorted row of each (token, slot)
    const float* gate;        // [T, k]
    const void* residual;     // [T, n_out] bf16 added before the rounding, or nullptr
    void* y;                  // [T, n_out] bf16, or nullptr: o only
    int* cnt;                 // [T, n_out / 128] o stores done per chunk, zero at launch
    int k;
};

// Tiles are dealt round-robin to `active` workers (CTAs, or CTA pairs): the
// fewest that still need no more rounds than all `launched` workers would, so
// every active worker gets the same number of tiles (+-1) and no final round
// runs a few tiles on a few SMs while the rest idle.  A worker at or beyond
// `active` gets no tile (first tile = total).
struct TileDeal {
    int first, stride;
};
__device__ __forceinline__ TileDeal deal_tiles(int worker, int launched, int total) {
    const int rounds = (total + launched - 1) / launched;
    const int active = rounds > 0 ? (total + rounds - 1) / rounds : 0;
    TileDeal d;
    d.first = worker < active ? worker : total;
    d.stride = active > 0 ? active : 1;
    return d;
}

// Per-stage wait: when the phase completes within try_wait's own suspend window
// the abort flag is not read; otherwise a bounded wait, then the flag.
__device__ __forceinline__ bool stage_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns,
                                           volatile int& abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait(bar, parity, timeout_ns) && !abort_flag;
}

struct TileInfo {
    int e, row0, rows, n0;
};

// Tile t of the expert-major enumeration: expert e owns tiles
// [n_tiles * mt_prefix[e], n_tiles * mt_prefix[e+1]).  Within an expert the
// m-tiles are walked in groups of `group_m` (the last group may be smaller);
// within a group the order is n-major with m fastest.  Tiles that run at the
// same time then share weight tiles, and a group's activation rows -- sized on
// the host to sit in L2 next to the weight stream -- are read from DRAM once
// for all column tiles instead of once per few column tiles.
__device__ __forceinline__ TileInfo decode_tile_rows(int t, const int* mt_prefix, const int* off,
                                                     int n_tiles, int n_tile_out, int tile_rows,
                                                     int group_m) {
    TileInfo ti;
    int e = 0;
    while (t >= n_tiles * mt_prefix[e + 1]) ++e;
    const int local = t - n_tiles * mt_prefix[e];
    const int mt = mt_prefix[e + 1] - mt_prefix[e];
    const int g = local / (group_m * n_tiles);
    const int m0 = g * group_m;
    const int gm = min(group_m, mt - m0);
    const int r = local - g * group_m * n_tiles;
    const int n = r / gm;
    const int m = m0 + (r - n * gm);
    ti.e = e;
    ti.row0 = off[e] + m * tile_rows;
    ti.rows = min(tile_rows, off[e + 1] - ti.row0);
    ti.n0 = n * n_tile_out;
    return ti;
}

// Epilogue output path.  A warp owns 32 rows of the tile (one TMEM lane quarter)
// and writes them 32 columns at a time.  When all 32 rows belong to the tile's
// expert, the chunk is staged in shared memory in the output tensor map's
// swizzled layout (one row per lane; the swizzle spreads the lanes' 16-byte
// writes over all banks) and leaves as one TMA store, so global memory sees
// whole rows instead of 32 scattered 16-byte pieces per instruction.  Each warp
// alternates between two staging buffers; before refilling one, lane 0 waits
// until the store issued from it has finished reading shared memory.  Warps
// whose rows run past the expert (the last tile of each expert) store row by
// row with predication instead, since a tensor-map store cannot skip rows.
struct EpiStage {
    uint8_t* base;  // this warp's two buffers, 1024-byte aligned
    uint32_t next;  // buffer to fill next
};

// Hands out the next staging buffer once the store that last read it is done.
__device__ __forceinline__ uint8_t* epi_acquire(EpiStage& st, int lane) {
    uint8_t* buf = st.base + st.next * kEpiBufBytes;
    if (lane == 0) bulk_wait_group_read<1>();
    __syncwarp();
    return buf;
}

// Publishes a filled buffer to the TMA unit and stores it at (x, y).
__device__ __forceinline__ void epi_release(EpiStage& st, const CUtensorMap* map, uint8_t* buf,
                                            int x, int y, int lane) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(map, buf, x, y);
        bulk_commit_group();
    }
    st.next ^= 1u;
}

// r[j] += bias[j] for 32 consecutive float32 columns (the same for every lane:
// the loads are broadcasts).  Float32 addition, as the bias of a Linear layer
// is added to its float32 accumulator.
__device__ __forceinline__ void add_bias_32(uint32_t (&r)[32], const float* bias) {
    const float4* b4 = reinterpret_cast<const float4*>(bias);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float4 b = __ldg(b4 + j);
        r[4 * j + 0] = __float_as_uint(__fadd_rn(__uint_as_float(r[4 * j + 0]), b.x));
        r[4 * j + 1] = __float_as_uint(__fadd_rn(__uint_as_float(r[4 * j + 1]), b.y));
        r[4 * j + 2] = __float_as_uint(__fadd_rn(__uint_as_float(r[4 * j + 2]), b.z));
        r[4 * j + 3] = __float_as_uint(__fadd_rn(__uint_as_float(r[4 * j + 3]), b.w));
    }
}

// 2^x by the special-function unit's approximation, without flushing subnormal
// results to zero (ex2.approx.f32, no .ftz).
__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// SiLU(a) * b in float32, with sigma(a) = 1 / (1 + e^-a) formed from
// t = e^-|a| = 2^(-|a| log2 e), which lies in (0, 1]: sigma = 1 / (1 + t) for
// a >= 0 and t / (1 + t) for a < 0.  The divisor 1 + t stays in (1, 2] for
// every a, where the fast division is accurate (to two float32 ulps; with the
// plain form a / (1 + e^-a) the divisor exceeds 2^126 once a < -87.3, where the
// fast division returns 0), and t underflows gradually rather than overflowing.
// Relative error: the rounding of -|a| log2 e moves t by up to |a| 2^-24
// relative, about 2^-17 at |a| = 100, far below the bf16 rounding of h that
// follows.
__device__ __forceinline__ float silu_times(float a, float b) {
    constexpr float kLog2e = 1.4426950408889634f;
    const float t = exp2_approx(-fabsf(a) * kLog2e);
    const float sigma = __fdividef(a >= 0.0f ? 1.0f : t, 1.0f + t);
    return a * sigma * b;
}

// GEMM1 epilogue of one TMEM lane (= one row): columns [0, hcols) from taddr
// hold a = x W1 and columns [b_off, b_off + hcols) hold b = x W3 for the same
// output columns; h = SiLU(a) * b (silu_times).  hrow points at the row's
// first output column x0.  With `tma` the warp's 32 rows go out through `map`
// (bf16, 64-byte rows, 64-byte swizzle) at (x0 + c, y0).  ba / bb (nullable)
// are the biases of output column x0 for a and b.
__device__ __forceinline__ void epilogue_swiglu(uint32_t taddr, uint32_t b_off, bool valid,
                                                bool tma, __nv_bfloat16* hrow, int hcols,
                                                const CUtensorMap* map, EpiStage& st, int x0,
                                                int y0, int lane, const float* ba,
                                                const float* bb) {
#pragma unroll 1
    for (int c = 0; c < hcols; c += 32) {
        uint32_t ra[32], rb[32];
        tmem_ld_32cols(taddr + c, ra);
        tmem_ld_32cols(taddr + b_off + c, rb);
        tmem_ld_wait();
        if (ba) add_bias_32(ra, ba + c);
        if (bb) add_bias_32(rb, bb + c);
        if (valid || tma) {
            uint32_t packed[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float a0 = __uint_as_float(ra[2 * j]);
                const float a1 = __uint_as_float(ra[2 * j + 1]);
                const float b0 = __uint_as_float(rb[2 * j]);
                const float b1 = __uint_as_float(rb[2 * j + 1]);
                // fast division on a divisor in (1, 2] (silu_times): the epilogue
                // warps share issue slots with the producer and MMA threads, and
                // the IEEE division cost GEMM1 0.6 %
                const float h0 = silu_times(a0, b0);
                const float h1 = silu_times(a1, b1);
                packed[j] = pack_bf16x2(h0, h1);
            }
            if (tma) {
                uint8_t* buf = epi_acquire(st, lane);
                uint8_t* rowp = buf + lane * 64;
                const int sw = (lane >> 1) & 3;  // 64-byte swizzle: chunk ^= address bits 7..8
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    *reinterpret_cast<uint4*>(rowp + ((j ^ sw) << 4)) =
                        make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2],
                                   packed[4 * j + 3]);
                epi_release(st, map, buf, x0 + c, y0, lane);
            } else {
                uint4* dst = reinterpret_cast<uint4*>(hrow + c);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2],
                                        packed[4 * j + 3]);
            }
        }
    }
}

// GEMM2 epilogue of one TMEM lane: `ncols` fp32 columns stored as they are
// (plus the bias `bo` of the tile's first column, when given).  With `tma` the
// warp's rows go out through `map` (fp32, 128-byte rows, 128-byte swizzle) at
// (x0 + c, y0).
__device__ __forceinline__ void epilogue_store_f32(uint32_t taddr, bool valid, bool tma,
                                                   float* orow, int ncols, const CUtensorMap* map,
                                                   EpiStage& st, int x0, int y0, int lane,
                                                   const float* bo) {
#pragma unroll 1
    for (int c = 0; c < ncols; c += 32) {
        uint32_t r[32];
        tmem_ld_32cols(taddr + c, r);
        tmem_ld_wait();
        if (bo) add_bias_32(r, bo + c);
        if (tma) {
            uint8_t* buf = epi_acquire(st, lane);
            uint8_t* rowp = buf + lane * 128;
            const int sw = lane & 7;  // 128-byte swizzle: chunk ^= address bits 7..9
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4*>(rowp + ((j ^ sw) << 4)) =
                    make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
            epi_release(st, map, buf, x0 + c, y0, lane);
        } else if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                dst[j] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
        }
    }
}

__device__ __forceinline__ void cp_async_cg16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_ca8(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The combine fused into the down projection's epilogue.  A warp has just
// stored o for its 32 rows (one per lane) and `ncols` columns from x0 (1 or 2
// chunks of 128).  A (token, chunk) of y needs the o rows of all k of the
// token's slots, stored by k row tiles in any order.  Once its own stores are
// complete and visible, each lane counts its chunks done with one atomic add
// per chunk; a lane whose add is the k-th holds the token's last rows, and the
// warp then forms those chunks of y with the combine kernel's arithmetic (so y
// has the same bits as with the separate combine).  The warp works on 32 / LPI
// chunks at a time, LPI lanes each (128 / LPI columns a lane), so that the
// chunks' latency chains overlap; their k rows come from L2 through
// asynchronous copies into the warp's idle staging buffers (`stage`,
// kEpiWarpBytes), as many chunks at once as fit, then each lane combines the
// columns it fetched.  Nothing waits on another CTA.  Every slot of a routed
// token has a row (the router always selects k experts), so k adds finish it.
template <int KMAX, int LPI>
__device__ __noinline__ void finish_tokens(const Params& p, uint8_t* stage, bool valid, bool tma,
                                           int64_t grow, int x0, int ncols, int lane) {
    constexpr int CPL = 128 / LPI;   // columns per lane
    constexpr int IPS = 32 / LPI;    // chunks per warp step
    // the warp's TMA stores (issued by lane 0) complete: their rows are in
    // memory and the staging buffers are free
    if (lane == 0) {
        bulk_wait_group<0>();
        if (tma) fence_proxy_async_global();
    }
    __syncwarp();
    __threadfence();  // this warp's o stores before its counts
    const int chunks = p.n_out >> 7;
    const int tok = valid ? __ldg(p.perm_tok + grow) : 0;
    int old[2] = {-1, -1};
#pragma unroll
    for (int j = 0; j < 2; ++j)
        if (valid && j * 128 < ncols)
            old[j] = atomicAdd(p.cnt + (int64_t)tok * chunks + (x0 >> 7) + j, 1);
    const unsigned m0 = __ballot_sync(0xffffffffu, old[0] == p.k - 1);
    const unsigned m1 = __ballot_sync(0xffffffffu, old[1] == p.k - 1);
    if ((m0 | m1) == 0u) return;
    __threadfence();  // the other tiles' counts before their rows
    // each lane's token's sorted rows and gates, handed out by shuffles
    int my_rows[KMAX];
    float my_gs[KMAX];
    const bool any = ((m0 | m1) >> lane) & 1u;
#pragma unroll
    for (int s = 0; s < KMAX; ++s) {
        const bool in = any && s < p.k;
        my_rows[s] = in ? __ldg(p.inv + (int64_t)tok * p.k + s) : -1;
        my_gs[s] = in ? __ldg(p.gate + (int64_t)tok * p.k + s) : 0.f;
    }
    // the chunk list (lane | chunk << 5), chunk 0's in lane order first, in the
    // last 256 bytes of the staging buffers
    constexpr int kListBytes = 256;
    int* list = reinterpret_cast<int*>(stage + kEpiWarpBytes - kListBytes);
    const unsigned lt = (1u << lane) - 1u;
    const int n0 = __popc(m0);
    const int nitems = n0 + __popc(m1);
    if ((m0 >> lane) & 1u) list[__popc(m0 & lt)] = lane;
    if ((m1 >> lane) & 1u) list[n0 + __popc(m1 & lt)] = lane | 32;
    __syncwarp();
    const float* o = static_cast<const float*>(p.out);
    const __nv_bfloat16* res = static_cast<const __nv_bfloat16*>(p.residual);
    __nv_bfloat16* y = static_cast<__nv_bfloat16*>(p.y);
    // per chunk: k rows of 128 float32, then 128 bf16 of residual
    const int item_bytes = p.k * 512 + (res ? 256 : 0);
    const int per_batch = (kEpiWarpBytes - kListBytes) / item_bytes;
    const uint32_t sbase = smem_u32(stage);
    const int g = lane / LPI;          // this lane's chunk within a step
    const int qc = (lane % LPI) * CPL;  // and its first column within the chunk
#pragma unroll 1
    for (int base = 0; base < nitems; base += per_batch) {
        const int nb = min(per_batch, nitems - base);
        // issue: the batch's chunks' rows (and residual), IPS chunks a step
#pragma unroll 1
        for (int u0 = 0; u0 < nb; u0 += IPS) {
            const int u = u0 + g;
            const int e = u < nb ? list[base + u] : 0;
            const int src = e & 31;
            const int col = x0 + (e >> 5) * 128 + qc;
            const uint32_t at = sbase + (uint32_t)(u * item_bytes);
#pragma unroll
            for (int s = 0; s < KMAX; ++s) {
                if (s >= p.k) break;
                const int row = __shfl_sync(0xffffffffu, my_rows[s], src);
                if (u < nb && row >= 0) {
                    const float* from = o + (int64_t)row * p.n_out + col;
#pragma unroll
                    for (int c = 0; c < CPL / 4; ++c)
                        cp_async_cg16(at + s * 512 + qc * 4 + c * 16, from + c * 4);
                }
            }
            if (res) {
                const int t = __shfl_sync(0xffffffffu, tok, src);
                if (u < nb) {
                    const __nv_bfloat16* from = res + (int64_t)t * p.n_out + col;
                    const uint32_t rat = at + p.k * 512 + qc * 2;
                    if constexpr (CPL >= 8) {
#pragma unroll
                        for (int c = 0; c < CPL / 8; ++c) cp_async_cg16(rat + c * 16, from + c * 8);
                    } else {
                        cp_async_ca8(rat, from);
                    }
                }
            }
        }
        cp_async_wait_all();  // each lane reads back only what it fetched
        // combine: the same chunks, the same lanes
#pragma unroll 1
        for (int u0 = 0; u0 < nb; u0 += IPS) {
            const int u = u0 + g;
            const int e = u < nb ? list[base + u] : 0;
            const int src = e & 31;
            const int col = x0 + (e >> 5) * 128 + qc;
            const int t = __shfl_sync(0xffffffffu, tok, src);
            const uint8_t* at = stage + u * item_bytes;
            int rows[KMAX];
            float gs[KMAX];
            float v[KMAX][CPL];
#pragma unroll
            for (int s = 0; s < KMAX; ++s) {
                rows[s] = __shfl_sync(0xffffffffu, my_rows[s], src);
                gs[s] = __shfl_sync(0xffffffffu, my_gs[s], src);
                if (u < nb && s < p.k && rows[s] >= 0) {
#pragma unroll
                    for (int c = 0; c < CPL / 4; ++c) {
                        const float4 f =
                            *reinterpret_cast<const float4*>(at + s * 512 + qc * 4 + c * 16);
                        v[s][4 * c] = f.x;
                        v[s][4 * c + 1] = f.y;
                        v[s][4 * c + 2] = f.z;
                        v[s][4 * c + 3] = f.w;
                    }
                }
            }
            if (u >= nb) continue;
            float r[CPL], out[CPL];
            if (res) {
#pragma unroll
                for (int c = 0; c < CPL / 2; ++c) {
                    const uint32_t w =
                        *reinterpret_cast<const uint32_t*>(at + p.k * 512 + qc * 2 + c * 4);
                    r[2 * c] = bf16_lo(w);
                    r[2 * c + 1] = bf16_hi(w);
                }
            }
            combine_columns<KMAX, CPL>(v, gs, rows, p.k, res != nullptr, r, out);
            uint32_t packed[CPL / 2];
#pragma unroll
            for (int c = 0; c < CPL / 2; ++c) packed[c] = pack_bf16x2(out[2 * c], out[2 * c + 1]);
            __nv_bfloat16* dst = y + (int64_t)t * p.n_out + col;
            if constexpr (CPL >= 8) {
#pragma unroll
                for (int c = 0; c < CPL / 8; ++c)
                    reinterpret_cast<uint4*>(dst)[c] = make_uint4(
                        packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
            } else {
                *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
            }
        }
    }
}

template <bool kSwiGLU>
__global__ void __launch_bounds__(kThreads, 1)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmB1,
                       const __grid_constant__ CUtensorMap tmOut, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    __shared__ uint64_t full_bar[kStages];
    __shared__ uint64_t empty_bar[kStages];
    __shared__ uint64_t acc_full[2];
    __shared__ uint64_t acc_empty[2];
    __shared__ uint64_t drain_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int s_off[kMaxE + 1];
    __shared__ int s_mt[kMaxE + 1];
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
        }
        mbar_init(&drain_bar, 1);
        fence_barrier_init();
        s_abort = 0;
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tmA);
        tma_prefetch_map(&tmB0);
        if (kSwiGLU) tma_prefetch_map(&tmB1);
        tma_prefetch_map(&tmOut);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    // The set-up above overlaps the previous kernel's tail; the offsets and the
    // A rows are its output.
    grid_dependency_wait();
    if (threadIdx.x == 0) {
        // m-tile prefix over experts (E <= 32, serial)
        int acc = 0;
        s_mt[0] = 0;
        for (int e = 0; e <= p.E; ++e) s_off[e] = p.offsets[e];
        for (int e = 0; e < p.E; ++e) {
            const int cnt = max(0, s_off[e + 1] - s_off[e]);
            acc += (cnt + kBM - 1) / kBM;
            s_mt[e + 1] = acc;
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = tmem_slot;

    const int n_tiles = p.n_out / p.n_tile_out;
    const int total_tiles = s_mt[p.E] * n_tiles;
    const int kb_count = p.K / kBK;
    const TileDeal deal = deal_tiles(blockIdx.x, gridDim.x, total_tiles);

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_parity = 0;
            int issued = 0;
            bool ok = true;
            const uint32_t tx_bytes = kABytes + p.n_boxes * kBBoxBytes;
            for (int t = deal.first; t < total_tiles && ok; t += deal.stride) {
                const TileInfo ti = decode_tile_rows(t, s_mt, s_off, n_tiles, p.n_tile_out, kBM, p.group_m);
                const int wrow0 = ti.e * p.K;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (p.stall_after >= 0 && issued >= p.stall_after) {
                        ok = false;  // test hook: behave like a producer that died
                        break;
                    }
                    if (!stage_wait(&empty_bar[stage], phase ^ 1u, p.timeout_ns, s_abort)) {
                        record_error(p.err, kDeviceTimeoutBase | kRoleProducer);
                        ok = false;
                        break;
                    }
                    uint8_t* sA = smem + stage * kStageBytes;
                    uint8_t* sB = sA + kABytes;
                    mbar_arrive_expect_tx(&full_bar[stage], tx_bytes);
                    const int wrow = wrow0 + kb * kBK;
                    // Weight maps are 3-D views [chunk][row][64 columns] whose box
                    // spans all the chunks of one copy: one load per matrix.
                    if (kSwiGLU) {
                        // W1 columns [n0, n0 + half chunks) then the same W3 columns
                        const int half = p.n_boxes / 2;
                        tma_load_3d(sB, &tmB0, &full_bar[stage], 0, wrow, ti.n0 / kBoxN);
                        tma_load_3d(sB + half * kBBoxBytes, &tmB1, &full_bar[stage], 0, wrow,
                                    ti.n0 / kBoxN);
                    } else {
                        tma_load_3d(sB, &tmB0, &full_bar[stage], 0, wrow, ti.n0 / kBoxN);
                    }
                    tma_load_2d(sA, &tmA, &full_bar[stage], kb * kBK, ti.row0);
                    issued_mask |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) s_abort = 1;
            // Every copy this thread issued must land before the CTA may exit.
            for (int s = 0; s < kStages; ++s)
                if (issued_mask & (1u << s))
                    (void)mbar_wait(&full_bar[s], (issued_parity >> s) & 1u, p.timeout_ns);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            const uint32_t idesc = idesc_bf16_f32(kBM, p.n_boxes * kBoxN, false, true);
            // Descriptors of stage 0, K step 0; a stage / K step only moves the
            // start-address field (address >> 4, no carry below 256 KB).
            const uint64_t adesc0 = desc_kmajor_sw128(smem_u32(smem));
            const uint64_t bdesc0 = desc_mnmajor_sw128(smem_u32(smem) + kABytes, kBBoxBytes);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = deal.first; t < total_tiles && ok; t += deal.stride) {
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, p.timeout_ns) || s_abort) {
                    record_error(p.err, kDeviceTimeoutBase | kRoleMma);
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * kAccCols;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!stage_wait(&full_bar[stage], phase, p.timeout_ns, s_abort)) {
                        record_error(p.err, kDeviceTimeoutBase | kRoleMma);
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint64_t soff = (uint64_t)((uint32_t)(stage * kStageBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        tc_mma_bf16(d_tmem, adesc0 + soff + kk * (32 >> 4),
                                    bdesc0 + soff + kk * (2048 >> 4), idesc, (kb | kk) != 0);
                    tc_commit(&empty_bar[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(&acc_full[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok) s_abort = 1;
            // Wait for every MMA this thread issued before TMEM is released.
            tc_commit(&drain_bar);
            (void)mbar_wait(&drain_bar, 0, p.timeout_ns);
        }
    } else {
        // ---------------------------------------------------- epilogue (warps 2..5)
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int row_in_tile = q * 32 + lane;
        EpiStage st{smem + kStages * kStageBytes + q * kEpiWarpBytes, 0u};
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = deal.first; t < total_tiles; t += deal.stride) {
            const TileInfo ti = decode_tile_rows(t, s_mt, s_off, n_tiles, p.n_tile_out, kBM, p.group_m);
            const bool got = mbar_wait(&acc_full[acc], acc_phase, p.timeout_ns);
            if (!got || s_abort) {
                if (!got) record_error(p.err, kDeviceTimeoutBase | kRoleEpilogue);
                s_abort = 1;
                break;
            }
            tc_fence_after_sync();
            const uint32_t taddr = tmem_base + acc * kAccCols + ((uint32_t)(q * 32) << 16);
            const bool valid = row_in_tile < ti.rows;
            const bool tma = q * 32 + 32 <= ti.rows;  // warp-uniform: all 32 rows are the expert's
            const int64_t grow = (int64_t)ti.row0 + row_in_tile;
            const int y0 = ti.row0 + q * 32;
            const int64_t boff = (int64_t)ti.e * p.n_out + ti.n0;
            const float* ba = p.bias_a ? p.bias_a + boff : nullptr;
            const float* bb = p.bias_b ? p.bias_b + boff : nullptr;
            if (kSwiGLU)
                epilogue_swiglu(taddr, (uint32_t)p.n_tile_out, valid, tma,
                                reinterpret_cast<__nv_bfloat16*>(p.out) + grow * p.n_out + ti.n0,
                                p.n_tile_out, &tmOut, st, ti.n0, y0, lane, ba, bb);
            else
                epilogue_store_f32(taddr, valid, tma,
                                   reinterpret_cast<float*>(p.out) + grow * p.n_out + ti.n0,
                                   p.n_boxes * kBoxN, &tmOut, st, ti.n0, y0, lane, ba);
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        // The staging buffers must outlive every store that reads them.
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------- CTA-pair kernel
// Same roles, but a cluster of two CTAs on two SMs shares each tile's MMAs
// (tcgen05.mma.cta_group::2): CTA rank r holds its share of the A rows and half
// of the B columns, and receives its own rows of D in its TMEM.  Per CTA a
// stage is 32 KB (A 16 KB + half of B 16 KB), so six stages fit, and each SM
// reads half as many B bytes per MMA as a single CTA with the same tile.
//
// Tile kinds.  An expert's rows are cut into "full" tiles of 256 rows (M = 256:
// 128 rows per CTA; the last one may be ragged) and, when the last remainder
// is at most 128 rows, one "half" tile of 128 rows (M = 128: 64 rows per CTA,
// loaded through a 64-row A box), which does half a full tile's MMA work
// instead of padding the remainder to 256 rows.
//
// TMEM layout of one accumulator (256 columns) in each CTA:
//   full tile: lane l = row l of the CTA's 128 rows, column c = MMA column c;
//   half tile: lane l = row l % 64 of the CTA's 64 rows, MMA columns
//              128 (l / 64) + c in columns c < 128.
// B columns: GEMM2 (N = 256 output columns) -- CTA r holds output columns
// [128 r, 128 r + 128) of the tile.  GEMM1 (128 h columns per tile) -- CTA r
// holds W1 columns [64 r, 64 r + 64) and then the same W3 columns, so MMA
// column order is a(0..63) b(0..63) a(64..127) b(64..127): in both tile kinds
// every lane holds a and b of the same h columns, 64 columns apart.
//
// Dealing (identical in every role and both CTAs): all tiles round-robin over
// the P pairs, full tiles first, then half tiles (see deal_pair_tile).
//
// Synchronisation: both CTAs' TMA loads count their bytes on the leader's
// (rank 0) full barrier, which only the leader arms with the bytes of both;
// the leader's single MMA thread commits each consumed stage to the empty
// barriers of both CTAs and each finished accumulator to the acc_full barriers
// of both (one multicast commit each); the epilogue warps of both CTAs arrive on the leader's acc_empty
// barrier (count 8).  Cluster barriers at start (barrier initialisation) and
// end (before the pair frees its tensor memory) are reached by every thread of
// both CTAs unconditionally; every mbarrier wait in between is bounded.
constexpr int kPM = 256;                                       // rows per full pair tile
constexpr int kPHalf = 128;                                    // rows per half pair tile
constexpr int kPairStages = 6;
constexpr int kPairBBoxes = 2;                                 // B boxes per CTA per stage
constexpr int kPairStageBytes = kABytes + kPairBBoxes * kBBoxBytes;   // 32 KB
constexpr size_t kPairSmemBytes = (size_t)kPairStages * kPairStageBytes + kEpiBytes + 1024;
constexpr int kPairMinRows = 512;
// Rounds of GEMM2 pair tiles from which the combine runs in GEMM2's epilogue.
// The finishing of a pair's last tile is not hidden behind a next tile: with
// one round (the quarter-width batch) GEMM2 grew by 22 us against an 8 us
// combine; at the Mixtral prefill batch (7 rounds) the step measured 8-18 us
// shorter than with the separate combine, at the skewed 16384-token batch
// (28 rounds) 40-95 us.
constexpr int kFuseMinRounds = 4;
constexpr int kPairMinRounds = 8;
constexpr int kInlineHalfRounds = 16;

// Tile of the pair enumeration, in one of two orders.
//  - Half tiles last (halves_inline = 0): ids [0, F) are full tiles
//    (expert-major, in the rasterisation groups of decode_tile_rows over
//    s_full), ids [F, F + H) half tiles (expert-major, n fastest).  Dealt
//    round-robin, the half tiles then go first to the pairs that got one full
//    tile fewer: the better balance when there are few rounds of tiles.
//  - Half tiles in place (halves_inline = 1): an expert's half m-tile is its
//    last m-tile (decode_tile_rows over s_mt = full + half m-tiles), so the half
//    tile of column n runs right after the full tiles of column n, while that
//    column's weight slice is still in L2; a tile of at most 128 rows is a half
//    tile.  The better DRAM traffic when there are many rounds of tiles.
struct PairTile {
    TileInfo ti;
    bool half;
};

__device__ __forceinline__ PairTile decode_pair_tile(int id, int F, const int* s_full,
                                                     const int* s_half, const int* s_mt,
                                                     const int* off, int n_tiles, int n_tile_out,
                                                     int group_m, bool inline_halves) {
    PairTile pt;
    if (inline_halves) {
        pt.ti = decode_tile_rows(id, s_mt, off, n_tiles, n_tile_out, kPM, group_m);
        pt.half = pt.ti.rows <= kPHalf;
    } else if (id < F) {
        pt.ti = decode_tile_rows(id, s_full, off, n_tiles, n_tile_out, kPM, group_m);
        pt.half = false;
    } else {
        const int j = id - F;
        const int hm = j / n_tiles;
        int e = 0;
        while (hm >= s_half[e + 1]) ++e;
        pt.ti.e = e;
        pt.ti.row0 = off[e] + (s_full[e + 1] - s_full[e]) * kPM;
        pt.ti.rows = off[e + 1] - pt.ti.row0;
        pt.ti.n0 = (j - hm * n_tiles) * n_tile_out;
        pt.half = true;
    }
    return pt;
}

// The i-th tile (id) dealt to pair p of P, or -1 past its last: the tiles go
// round-robin in enumeration order, full tiles first, then half tiles.  A half
// tile has half the MMA work of a full one but the same B bytes per stage, so
// it takes about 0.7 of a full tile's time; dealing the half tiles after all
// full tiles hands them to the pairs with one full tile fewer first, and no
// pair runs two half tiles where a full tile would have done.
__device__ __forceinline__ int deal_pair_tile(int i, int p, int P, int F, int H) {
    const int id = p + i * P;
    return id < F + H ? id : -1;
}

template <bool kSwiGLU>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    expert_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmA64,
                            const __grid_constant__ CUtensorMap tmB0,
                            const __grid_constant__ CUtensorMap tmB1,
                            const __grid_constant__ CUtensorMap tmOut,
                            const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    __shared__ uint64_t full_bar[kPairStages];
    __shared__ uint64_t empty_bar[kPairStages];
    __shared__ uint64_t acc_full[2];
    __shared__ uint64_t acc_empty[2];
    __shared__ uint64_t drain_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int s_off[kMaxE + 1];
    __shared__ int s_full[kMaxE + 1];
    __shared__ int s_half[kMaxE + 1];
    __shared__ int s_mt[kMaxE + 1];
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 8);
        }
        mbar_init(&drain_bar, 1);
        fence_barrier_init();
        s_abort = 0;
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tmA);
        tma_prefetch_map(&tmA64);
        tma_prefetch_map(&tmB0);
        if (kSwiGLU) tma_prefetch_map(&tmB1);
        tma_prefetch_map(&tmOut);
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    grid_dependency_wait();
    if (threadIdx.x == 0) {
        // full m-tiles (256 rows; a remainder above 128 rows is a ragged full
        // tile) and half m-tiles (a remainder of 1..128 rows) per expert
        int nf = 0, nh = 0;
        s_full[0] = 0;
        s_half[0] = 0;
        s_mt[0] = 0;
        for (int e = 0; e <= p.E; ++e) s_off[e] = p.offsets[e];
        for (int e = 0; e < p.E; ++e) {
            const int cnt = max(0, s_off[e + 1] - s_off[e]);
            const int rem = cnt % kPM;
            nf += cnt / kPM + (rem > kPHalf ? 1 : 0);
            nh += (rem > 0 && rem <= kPHalf) ? 1 : 0;
            s_full[e + 1] = nf;
            s_half[e + 1] = nh;
            s_mt[e + 1] = nf + nh;
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync_all();  // the peer's barriers are initialised before anyone signals them
    tc_fence_after_sync();
    const uint32_t tmem_base = tmem_slot;

    const int n_tiles = p.n_out / p.n_tile_out;
    const bool inl = p.halves_inline != 0;
    // for the deal, in-place half tiles count among the F tiles (no separate H)
    const int F = (inl ? s_mt[p.E] : s_full[p.E]) * n_tiles;
    const int H = inl ? 0 : s_half[p.E] * n_tiles;
    const int kb_count = p.K / kBK;
    const int boxes = p.n_boxes;  // B boxes per CTA per stage

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer (both CTAs)
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_parity = 0;
            int issued = 0;
            bool ok = true;
            const uint32_t leader_full0 = map_to_cta(smem_u32(&full_bar[0]), 0);
            for (int i = 0; ok; ++i) {
                const int id = deal_pair_tile(i, pair, npairs, F, H);
                if (id < 0) break;
                const PairTile pt = decode_pair_tile(id, F, s_full, s_half, s_mt, s_off, n_tiles,
                                                     p.n_tile_out, p.group_m, inl);
                const CUtensorMap* am = pt.half ? &tmA64 : &tmA;
                const int my_row0 = pt.ti.row0 + (int)rank * (pt.half ? kPHalf / 2 : kBM);
                const uint32_t tx_pair =
                    2u * ((pt.half ? kABytes / 2 : kABytes) + boxes * kBBoxBytes);
                const int wrow0 = pt.ti.e * p.K;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (p.stall_after >= 0 && issued >= p.stall_after) {
                        ok = false;  // test hook: both producers stop at the same stage
                        break;
                    }
                    if (!stage_wait(&empty_bar[stage], phase ^ 1u, p.timeout_ns, s_abort)) {
                        record_error(p.err, kDeviceTimeoutBase | kRoleProducer);
                        ok = false;
                        break;
                    }
                    uint8_t* sA = smem + stage * kPairStageBytes;
                    uint8_t* sB = sA + kABytes;
                    const uint32_t bar = leader_full0 + stage * (uint32_t)sizeof(uint64_t);
                    if (leader) mbar_arrive_expect_tx(&full_bar[stage], tx_pair);
                    const int wrow = wrow0 + kb * kBK;
                    if (kSwiGLU) {
                        // 64 W1 columns and the same 64 W3 columns of this CTA's half
                        const int chunk = (pt.ti.n0 + (int)rank * kBoxN) / kBoxN;
                        tma_load_3d_pair(sB, &tmB0, bar, 0, wrow, chunk);
                        tma_load_3d_pair(sB + kBBoxBytes, &tmB1, bar, 0, wrow, chunk);
                    } else {
                        const int c0 = pt.ti.n0 + (int)rank * boxes * kBoxN;
                        tma_load_3d_pair(sB, &tmB0, bar, 0, wrow, c0 / kBoxN);
                    }
                    tma_load_2d_pair(sA, am, bar, kb * kBK, my_row0);
                    issued_mask |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    ++issued;
                    if (++stage == kPairStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) s_abort = 1;
            // The leader's full barriers count the bytes of both CTAs: once every
            // phase the leader armed has completed, no copy of either CTA is in flight.
            if (leader)
                for (int s = 0; s < kPairStages; ++s)
                    if (issued_mask & (1u << s))
                        (void)mbar_wait(&full_bar[s], (issued_parity >> s) & 1u, p.timeout_ns);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------ MMA issuer (leader only)
            const uint32_t idesc_full = idesc_bf16_f32(kPM, 2 * boxes * kBoxN, false, true);
            const uint32_t idesc_half = idesc_bf16_f32(kPHalf, 2 * boxes * kBoxN, false, true);
            const uint64_t adesc0 = desc_kmajor_sw128(smem_u32(smem));
            const uint64_t bdesc0 = desc_mnmajor_sw128(smem_u32(smem) + kABytes, kBBoxBytes);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int id = deal_pair_tile(i, pair, npairs, F, H);
                if (id < 0) break;
                const bool half = inl ? decode_tile_rows(id, s_mt, s_off, n_tiles, p.n_tile_out,
                                                         kPM, p.group_m).rows <= kPHalf
                                      : id >= F;
                const uint32_t idesc = half ? idesc_half : idesc_full;
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, p.timeout_ns) || s_abort) {
                    record_error(p.err, kDeviceTimeoutBase | kRoleMma);
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * kAccCols;
                // The next stage's barrier is looked at before this stage's MMAs
                // are issued, so its wait overlaps them (measured faster here,
                // not on the single-CTA kernel).
                bool ready = mbar_try_wait(&full_bar[stage], phase);
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!ready && !stage_wait(&full_bar[stage], phase, p.timeout_ns, s_abort)) {
                        record_error(p.err, kDeviceTimeoutBase | kRoleMma);
                        ok = false;
                        break;
                    }
                    const int cur = stage;
                    if (++stage == kPairStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    ready = kb + 1 < kb_count && mbar_try_wait(&full_bar[stage], phase);
                    const uint64_t soff = (uint64_t)((uint32_t)(cur * kPairStageBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        tc_mma_bf16_pair(d_tmem, adesc0 + soff + kk * (32 >> 4),
                                         bdesc0 + soff + kk * (2048 >> 4), idesc, (kb | kk) != 0);
                    tc_commit_pair_mc(smem_u32(&empty_bar[cur]), 0x3);
                }
                if (!ok) break;
                tc_commit_pair_mc(smem_u32(&acc_full[acc]), 0x3);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok) s_abort = 1;
            tc_commit_pair(smem_u32(&drain_bar));
            (void)mbar_wait(&drain_bar, 0, p.timeout_ns);
        }
    } else {
        // ---------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;
        EpiStage st{smem + kPairStages * kPairStageBytes + q * kEpiWarpBytes, 0u};
        int acc = 0;
        uint32_t acc_phase = 0;
        const uint32_t leader_acc_empty0 = map_to_cta(smem_u32(&acc_empty[0]), 0);
        for (int i = 0;; ++i) {
            const int id = deal_pair_tile(i, pair, npairs, F, H);
            if (id < 0) break;
            const PairTile pt = decode_pair_tile(id, F, s_full, s_half, s_mt, s_off, n_tiles,
                                                 p.n_tile_out, p.group_m, inl);
            const bool got = mbar_wait(&acc_full[acc], acc_phase, p.timeout_ns);
            if (!got || s_abort) {
                if (!got) record_error(p.err, kDeviceTimeoutBase | kRoleEpilogue);
                s_abort = 1;
                break;
            }
            tc_fence_after_sync();
            const uint32_t taddr = tmem_base + acc * kAccCols + ((uint32_t)(q * 32) << 16);
            // this warp's rows of the tile and the MMA columns its lanes hold
            const int warp_row0 = pt.half ? (int)rank * (kPHalf / 2) + (q & 1) * 32
                                          : (int)rank * kBM + q * 32;
            const int col_half = pt.half ? (q >> 1) : 0;  // half tile: which 128 MMA columns
            const int row_in_tile = warp_row0 + lane;
            const bool valid = row_in_tile < pt.ti.rows;
            const bool tma = warp_row0 + 32 <= pt.ti.rows;  // warp-uniform
            const int64_t grow = (int64_t)pt.ti.row0 + row_in_tile;
            const int y0 = pt.ti.row0 + warp_row0;
            const int64_t boff = (int64_t)pt.ti.e * p.n_out;
            if (kSwiGLU) {
                // h columns [x0, x0 + 64): a in TMEM columns [c0, c0 + 64), b 64 further
                for (int seg = 0; seg < (pt.half ? 1 : 2); ++seg) {
                    const int part = pt.half ? col_half : seg;
                    const int x0 = pt.ti.n0 + part * 64;
                    epilogue_swiglu(taddr + (uint32_t)((pt.half ? 0 : part) * 128), 64u, valid,
                                    tma,
                                    reinterpret_cast<__nv_bfloat16*>(p.out) + grow * p.n_out + x0,
                                    64, &tmOut, st, x0, y0, lane,
                                    p.bias_a ? p.bias_a + boff + x0 : nullptr,
                                    p.bias_b ? p.bias_b + boff + x0 : nullptr);
                }
            } else {
                const int ncols = pt.half ? boxes * kBoxN : 2 * boxes * kBoxN;
                const int x0 = pt.ti.n0 + col_half * boxes * kBoxN;
                epilogue_store_f32(taddr, valid, tma,
                                   reinterpret_cast<float*>(p.out) + grow * p.n_out + x0, ncols,
                                   &tmOut, st, x0, y0, lane,
                                   p.bias_a ? p.bias_a + boff + x0 : nullptr);
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_acc_empty0 + acc * (uint32_t)sizeof(uint64_t));
            if (!kSwiGLU && p.y) {  // the accumulator is free again: finish tokens meanwhile
                const int ncols = pt.half ? boxes * kBoxN : 2 * boxes * kBoxN;
                const int x0 = pt.ti.n0 + col_half * boxes * kBoxN;
                if (p.k <= 2)
                    finish_tokens<2, 8>(p, st.base, valid, tma, grow, x0, ncols, lane);
                else
                    finish_tokens<8, 32>(p, st.base, valid, tma, grow, x0, ncols, lane);
            }
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }

    tc_fence_before_sync();
    __syncwarp();
    __syncthreads();
    cluster_sync_all();  // both CTAs are done with the pair's MMAs and tensor memory
    tc_fence_after_sync();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 2-D bf16 tensor map over a row-major [rows, cols] matrix with a
// [box_rows, 64]-element box and 128-byte swizzle.
static bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                     uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Weight map: a row-major [rows, cols] bf16 matrix viewed in 3-D as
// [cols / 64 chunks][rows][64 columns] (chunk stride 128 bytes, row stride
// cols * 2), box {64, 64 rows, chunks}, 128-byte swizzle.  One copy of the box
// fills `chunks` consecutive 8 KB shared-memory boxes, each laid out exactly as
// a 2-D {64, 64} box would be.
static bool make_weight_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                            uint32_t chunks) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {64, rows, cols / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, (cuuint32_t)kBK, chunks};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Output map for the epilogue's TMA stores: a row-major [rows, cols] matrix of
// bf16 (h) or fp32 (o) with a 32 x 32-element box; the box rows are 64 or 128
// bytes, swizzled in shared memory with the matching 64- or 128-byte pattern.
static bool make_out_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                         bool f32) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const uint64_t esize = f32 ? 4 : 2;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * esize};
    cuuint32_t box[2] = {kOutBox, kOutBox};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <bool kSwiGLU>
static int launch(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                  const CUtensorMap& out, const Params& p, int max_tiles, cudaStream_t stream) {
    auto kern = expert_gemm_kernel<kSwiGLU>;
    static int configured_device = -1;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (configured_device != dev) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes) != cudaSuccess)
            return MOE_ERR_CUDA;
        configured_device = dev;
    }
    const int grid = max(1, min(device_sm_count(), max_tiles));
    return launch_pdl(kern, dim3(grid), dim3(kThreads), kSmemBytes, stream, a, b0, b1, out, p) ==
                   cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

// Number of CTA pairs that can be resident at once (clusters must fit inside a
// GPC, so this can be below half the SM count); cached per device.
template <bool kSwiGLU>
static int max_pairs() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cached[dev] == 0) {
        auto kern = expert_gemm_pair_kernel<kSwiGLU>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kPairSmemBytes) != cudaSuccess)
            return 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * 74, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kPairSmemBytes;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        int n = 0;
        // The kernel carries its cluster shape (2,1,1); ask without and, should the
        // runtime want it spelled out, with the matching launch attribute.
        if (cudaOccupancyMaxActiveClusters(&n, (void*)kern, &cfg) != cudaSuccess || n <= 0) {
            (void)cudaGetLastError();
            cfg.attrs = &attr;
            cfg.numAttrs = 1;
            n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, (void*)kern, &cfg) != cudaSuccess || n <= 0) {
                (void)cudaGetLastError();
                return 0;
            }
        }
        cached[dev] = n;
    }
    return cached[dev];
}

template <bool kSwiGLU>
static int launch_pair(const CUtensorMap& a, const CUtensorMap& a64, const CUtensorMap& b0,
                       const CUtensorMap& b1, const CUtensorMap& out, const Params& p,
                       int max_tiles, cudaStream_t stream) {
    const int pairs = max_pairs<kSwiGLU>();  // also sets the shared-memory attribute
    if (pairs <= 0) return MOE_ERR_CUDA;
    const int grid = 2 * max(1, min(pairs, max_tiles));
    return launch_pdl(expert_gemm_pair_kernel<kSwiGLU>, dim3(grid), dim3(kThreads),
                      kPairSmemBytes, stream, a, a64, b0, b1, out, p) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

}  // namespace gemm

// The fused combine counts whole 128-column chunks per warp: it needs GEMM2 on
// CTA pairs with 256-column tiles (each warp then stores 1 or 2 whole chunks).
bool combine_fusable(const moe_shape& s) {
    return (int64_t)s.T * s.k >= gemm::kPairMinRows && s.d % 256 == 0;
}

// The combine is fused only when GEMM2 has several rounds of pair tiles
// (kFuseMinRounds).
bool combine_fused(const moe_shape& s) {
    if (!combine_fusable(s)) return false;
    const int64_t tiles = ((int64_t)s.T * s.k / gemm::kPM) * (s.d / 256);
    return tiles >= (int64_t)gemm::kFuseMinRounds * std::max(1, device_sm_count() / 2);
}

int expert_gemms(const moe_shape& s, const void* x_sorted, const int32_t* offsets, const void* W1,
                 const void* W3, const void* W2, void* h, float* o, int* err,
                 uint64_t timeout_ns, int stall_after, cudaStream_t stream,
                 void* mid_event, const float* b1, const float* b3, const float* b2,
                 const FusedCombine* fuse) {
    using namespace gemm;
    const int R = s.T * s.k;
    if (R == 0) return MOE_OK;
    CUtensorMap mx, mh, mx64, mh64, m1, m3, m2, oh, oo;
    if (!make_map(&mx, x_sorted, (uint64_t)R, (uint64_t)s.d, kBM) ||
        !make_map(&mh, h, (uint64_t)R, (uint64_t)s.d_ff, kBM) ||
        !make_map(&mx64, x_sorted, (uint64_t)R, (uint64_t)s.d, kPHalf / 2) ||
        !make_map(&mh64, h, (uint64_t)R, (uint64_t)s.d_ff, kPHalf / 2) ||
        !make_out_map(&oh, h, (uint64_t)R, (uint64_t)s.d_ff, false) ||
        !make_out_map(&oo, o, (uint64_t)R, (uint64_t)s.d, true))
        return MOE_ERR_CUDA;
    // The down projection runs on CTA pairs (256-row full tiles, 128-row half
    // tiles for remainders of at most 128 rows) once there are at least
    // kPairMinRows routed rows.  GEMM1 does when its pair tiles fill at least
    // kPairMinRounds rounds of the pairs: with fewer, the single CTA's 128-row
    // tiles quantise better (measured: the quarter-width batch, R = 2048, three
    // pair rounds, ran 4 % slower on pairs; the Mixtral prefill batch, 48
    // rounds, 8 % faster).  Decode-sized work runs on single CTAs, where every
    // tile streams its own weight slice.
    const bool pairs2 = R >= kPairMinRows;
    const int64_t pair_tiles1 = ((int64_t)R / kPM) * (s.d_ff / 128);
    const bool pairs1 = pairs2 && pair_tiles1 >= (int64_t)kPairMinRounds * max_pairs<true>();
    // upper bound on the number of tiles of either kind
    auto mtiles = [&](int tile_rows) { return (R + tile_rows - 1) / tile_rows + 2 * s.E; };
    // m-tiles per rasterisation group: as many as keep the group's activation
    // rows (tile_rows x K bf16 each) within 32 MB of the 126 MB L2, and at
    // least 2048 rows.  About 74 tiles run at once; a group of g m-tiles spreads
    // them over 74 / g column tiles, whose weight slices are read from DRAM once
    // per group, so the traffic is least near g = 8-16.  Measured DRAM bytes of
    // the skewed batch (same box): GEMM1 (K = 4096) 6.2 GB with 16 m-tiles, 7.0
    // with 8, 11.3 with 4; GEMM2 (K = 14336) 6.2 GB with 8, 6.9 with 4 (the
    // 32 MB budget alone).  The step time moved by less than 1 %.
    auto group_rows = [](int tile_rows, int K) {
        const int64_t per_tile = (int64_t)tile_rows * K * 2;
        const int by_bytes = (int)std::max<int64_t>(1, (int64_t(32) << 20) / per_tile);
        return std::max(by_bytes, 2048 / tile_rows);
    };

    Params p1{};
    p1.offsets = offsets;
    p1.out = h;
    p1.err = err;
    p1.timeout_ns = timeout_ns;
    p1.E = s.E;
    p1.K = s.d;
    p1.n_out = s.d_ff;
    // GEMM1 tiles cover 128 h columns: on one CTA 2 weight boxes of W1 and 2 of
    // W3; on a pair each CTA 1 box of W1 and the same columns of W3.  Narrower
    // 64-column tiles, which balance small batches across the SMs better, were
    // measured slower at decode: every tile also streams a full 128-row A tile.
    p1.n_tile_out = 128;
    p1.n_boxes = pairs1 ? 2 : 4;  // per CTA
    p1.stall_after = stall_after;
    p1.group_m = group_rows(pairs1 ? kPM : kBM, s.d);
    p1.bias_a = b1;
    p1.bias_b = b3;
    // Half tiles go in place (next to their column's full tiles, sharing the
    // weight slice in L2) when the launch has many rounds of pair tiles, and
    // last (for balance) when it has few: GEMM1 at the prefill batch runs ~48
    // rounds, GEMM2 ~7, GEMM2 at the skewed batch ~28.
    auto inline_halves = [&](int n_cols_per_tile, int n_out) {
        const int64_t rounds = ((int64_t)R / kPM) * (n_out / n_cols_per_tile) /
                               std::max(1, max_pairs<true>());
        return rounds >= kInlineHalfRounds ? 1 : 0;
    };
    p1.halves_inline = inline_halves(128, s.d_ff);
    // weight boxes: W1 / W3 chunks per copy = half of the CTA's B boxes
    const uint32_t ch1 = (uint32_t)p1.n_boxes / 2;
    if (!make_weight_map(&m1, W1, (uint64_t)s.E * s.d, (uint64_t)s.d_ff, ch1) ||
        !make_weight_map(&m3, W3, (uint64_t)s.E * s.d, (uint64_t)s.d_ff, ch1))
        return MOE_ERR_CUDA;
    const int t1 = mtiles(pairs1 ? kPM : kBM) * (s.d_ff / p1.n_tile_out);
    int rc = pairs1 ? launch_pair<true>(mx, mx64, m1, m3, oh, p1, t1, stream)
                    : launch<true>(mx, m1, m3, oh, p1, t1, stream);
    if (rc != MOE_OK) return rc;
    if (mid_event && cudaEventRecord(static_cast<cudaEvent_t>(mid_event), stream) != cudaSuccess)
        return MOE_ERR_CUDA;

    Params p2 = p1;
    p2.out = o;
    p2.K = s.d_ff;
    p2.n_out = s.d;
    p2.n_tile_out = (s.d % 256 == 0) ? 256 : 128;
    p2.n_boxes = p2.n_tile_out / kBoxN / (pairs2 ? 2 : 1);
    p2.stall_after = stall_after;
    p2.group_m = group_rows(pairs2 ? kPM : kBM, s.d_ff);
    p2.bias_a = b2;
    p2.bias_b = nullptr;
    p2.halves_inline = inline_halves(p2.n_tile_out, s.d);
    p2.k = s.k;
    if (fuse && combine_fusable(s)) {
        p2.perm_tok = fuse->perm_tok;
        p2.inv = fuse->inv;
        p2.gate = fuse->gate;
        p2.residual = fuse->residual;
        p2.y = fuse->y;
        p2.cnt = fuse->cnt;
    }
    if (!make_weight_map(&m2, W2, (uint64_t)s.E * s.d_ff, (uint64_t)s.d, (uint32_t)p2.n_boxes))
        return MOE_ERR_CUDA;
    const int t2 = mtiles(pairs2 ? kPM : kBM) * (s.d / p2.n_tile_out);
    return pairs2 ? launch_pair<false>(mh, mh64, m2, m2, oo, p2, t2, stream)
                  : launch<false>(mh, m2, m2, oo, p2, t2, stream);
}

}  // namespace moe
