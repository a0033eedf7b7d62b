// combine_math.cuh -- the arithmetic of a token's output columns, shared by the
// combine kernel and the down projection's epilogue (which finishes a token's
// columns itself when the combine is fused into it), so both give the same bits.
//
// Mixtral textbook page, section "Алгоритм": a token's output is the sum of its
// k gate-weighted expert outputs.  Here the products are rounded to float32
// separately and added in slot order (no fused multiply-add; a slot whose row
// is negative is skipped), the residual of the block edge is added last in
// float32, and the result is rounded once to bf16 (nearest even).  Every column
// is computed on its own, so how the columns are grouped into threads does not
// change a bit.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"

namespace moe {

// out[j] = g[0] v[0][j] + g[1] v[1][j] + ... over the slots s < k with
// rows[s] >= 0, in slot order (0 when there is none), then + res[j] when
// has_residual.
template <int KMAX, int N>
__device__ __forceinline__ void combine_columns(const float (&v)[KMAX][N], const float (&g)[KMAX],
                                                const int (&rows)[KMAX], int k, bool has_residual,
                                                const float (&res)[N], float (&out)[N]) {
    bool first = true;
#pragma unroll
    for (int s = 0; s < KMAX; ++s) {
        if (s >= k || rows[s] < 0) continue;
#pragma unroll
        for (int j = 0; j < N; ++j) {
            const float p = __fmul_rn(g[s], v[s][j]);
            out[j] = first ? p : __fadd_rn(out[j], p);
        }
        first = false;
    }
    if (first) {
#pragma unroll
        for (int j = 0; j < N; ++j) out[j] = 0.f;
    }
    if (has_residual) {  // H = U + MoE(.): one more float32 addition before the rounding
#pragma unroll
        for (int j = 0; j < N; ++j) out[j] = __fadd_rn(res[j], out[j]);
    }
}

}  // namespace moe
