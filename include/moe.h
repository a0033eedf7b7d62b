/*
 * moe.h -- C ABI of the B200 (sm_100a) Mixtral sparse-MoE feed-forward layer.
 *
 * The layer (Mixtral textbook page, llm-arch-research, section "Прямой проход в
 * формулах", the MoE equation; the same formula in section "Научный вклад"):
 *
 *     g = u W_r,   S = TopK(g, k),   w_i = exp(g_i) / sum_{j in S} exp(g_j),
 *     MoE(u) = sum_{i in S} w_i * (SiLU(u W1_i) (.) (u W3_i)) W2_i
 *
 * computed, as in that page's section "Алгоритм" (algorithm), as a loop over
 * experts rather than tokens: route every token, list each expert's tokens
 * (dispatch), run each expert once over its rows, and add each token's k
 * gate-weighted expert outputs (combine).  No capacity limit, no dropped
 * tokens: every token gets exactly k terms and the experts process T*k rows.
 *
 * Conventions for every entry point
 *  - Layouts are row-major and dense.  bf16 tensors are passed as raw 16-bit
 *    storage (void*).  Shapes:
 *        x        [T, d]        bf16   tokens (already normalised: the layer input u)
 *        Wg       [d, E]        bf16   router W_r (E fastest)
 *        bias     [E]           float  optional router bias (nullable)
 *        W1, W3   [E, d, d_ff]  bf16   gate / up projections (u W1_e, u W3_e)
 *        W2       [E, d_ff, d]  bf16   down projection
 *        y        [T, d]        bf16   layer output
 *  - Every pointer except `stream` is DEVICE memory owned by the caller, except
 *    in the host-I/O entry points (moe_forward_hostio, moe_forward_hostio_batches
 *    and their test hooks) where x and y are HOST memory.  The library never
 *    allocates or frees memory and never synchronises, except
 *    moe_read_device_status (documented there).  All work is enqueued
 *    asynchronously on `stream` (a cudaStream_t; NULL = legacy default stream)
 *    on the current device.
 *  - Every pointer must be 16-byte aligned.
 *  - Arguments are checked on the host before anything is launched; a failed
 *    check returns a non-zero status and launches nothing (the counterpart of
 *    the ValueError the page's MoE constructor raises for a top_k_experts
 *    outside 1..num_experts, section "Mixtral" / "Конфигурация").
 *  - Supported shapes: T >= 0 (T == 0 is a no-op), 1 <= k <= E <= 32, k <= 8,
 *    d and d_ff multiples of 128, T*k*max(d, d_ff) < 2^31, and
 *    16 * d * ceil(E/8) <= 163840 (router tile in shared memory).
 *
 * Precision: bf16 inputs, fp32 accumulation on tensor cores; router logits,
 * gates and expert outputs o in fp32; the SwiGLU product h stored in bf16 (the
 * down projection's tensor-core input); y rounded once to bf16 (nearest-even).
 * Top-k ties go to the lower expert index; slot 0 holds the largest logit.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,    /* null / misaligned pointer, k outside 1..E, negative size */
    MOE_ERR_UNSUPPORTED = 2,    /* legal shape the library does not handle (see limits above) */
    MOE_ERR_WORKSPACE = 3,      /* workspace smaller than the matching *_workspace_bytes */
    MOE_ERR_CUDA = 4,           /* a CUDA runtime/driver call or launch failed */
    MOE_ERR_DEVICE_TIMEOUT = 5  /* a bounded device-side wait expired (see moe_read_device_status) */
} moe_status;

typedef struct {
    int32_t T;     /* tokens (batch * seq_len, the page's N = batch * seq_len) */
    int32_t d;     /* model width (emb_size) */
    int32_t d_ff;  /* expert hidden width (intermediate_size) */
    int32_t E;     /* experts (num_experts) */
    int32_t k;     /* experts per token (top_k_experts) */
} moe_shape;

/* Human-readable name of a status code (static string, never NULL). */
const char* moe_status_string(int status);

/* Checks a shape against the limits above without touching the GPU. */
int moe_check_shape(moe_shape s);

/* Bytes of workspace moe_expert_swiglu needs for shape s (status word and
 * scheduling state). */
size_t moe_expert_workspace_bytes(moe_shape s);

/* Bytes of workspace moe_forward / moe_forward_hostio need for shape s (every
 * intermediate of the layer plus the moe_expert_swiglu workspace). */
size_t moe_forward_workspace_bytes(moe_shape s);

/* Number of kernels one moe_forward (or moe_block_forward) of shape s launches
 * on the current device: router, dispatch index, dispatch scatter, the two
 * expert GEMMs, and the combine unless the down projection forms y itself
 * (4 or more rounds of its CTA-pair tiles on this device's SMs).  0 for
 * T == 0; a negative status (-MOE_ERR_...) for a shape moe_forward rejects.
 * Queries the device's SM count; launches nothing. */
int moe_forward_kernel_count(moe_shape s);

/*
 * moe_route -- router, top-k and softmax over the selected k.
 * Page: section "Прямой проход в формулах" (g = u W_r, S = TopK(g, k), w_i) and
 * section "MoE изнутри" (softmax over the k selected logits, in float32).
 *   x [T,d] bf16, Wg [d,E] bf16, bias [E] float or NULL  (in)
 *   idx [T,k] int32   expert ids, slot 0 = largest logit, ties -> lower id (out)
 *   gate [T,k] float  w_i of the selected experts, summing to 1 (out)
 *   logits [T,E] float  g (+ bias) in float32, or NULL (out)
 */
int moe_route(moe_shape s, const void* x, const void* Wg, const float* bias, int32_t* idx,
              float* gate, float* logits, void* stream);

/*
 * moe_dispatch -- per-expert token lists (the dispatch step of section
 * "Алгоритм": for each expert, the (token, slot) pairs whose top-k list names
 * that expert, in ascending token order).
 *   idx [T,k] int32 (in), x [T,d] bf16 (in)
 *   offsets [E+1] int32: rows of expert e are offsets[e] .. offsets[e+1]-1 (out)
 *   perm_tok [T*k] int32: token of each sorted row (out)
 *   inv [T,k] int32: sorted row of each (token, slot); -1 if idx was outside 0..E-1 (out)
 *   x_sorted [T*k,d] bf16: x_sorted[r] = x[perm_tok[r]] (out)
 * Entries of idx outside 0..E-1 get no row; then offsets[E] < T*k.
 */
int moe_dispatch(moe_shape s, const int32_t* idx, const void* x, int32_t* offsets,
                 int32_t* perm_tok, int32_t* inv, void* x_sorted, void* stream);

/*
 * moe_expert_swiglu -- Expert_e(X[tok]) for every expert e over its rows
 * (section "Алгоритм"; expert = SwiGLU of section "Прямой проход в формулах").
 *   x_sorted [T*k,d] bf16, offsets [E+1] int32 (from moe_dispatch) (in)
 *   W1, W3 [E,d,d_ff] bf16, W2 [E,d_ff,d] bf16 (in)
 *   h [T*k,d_ff] bf16: SiLU(x W1_e) (.) (x W3_e), rounded to bf16 (out)
 *   o [T*k,d] float:   h W2_e (out)
 *   ws: >= moe_expert_workspace_bytes(s) bytes of device memory (scratch)
 * Rows at or beyond offsets[E] are left untouched; an expert without rows
 * costs nothing.  Each row's h and o are accumulated in one fixed order
 * whatever the other rows are, so running an expert's rows alone gives the
 * same bits.  A device wait that expires leaves o/h incomplete and is
 * reported by moe_read_device_status(ws).
 */
int moe_expert_swiglu(moe_shape s, const void* x_sorted, const int32_t* offsets, const void* W1,
                      const void* W3, const void* W2, void* h, float* o, void* ws,
                      size_t ws_bytes, void* stream);

/*
 * moe_expert_swiglu_bias -- moe_expert_swiglu for the layer built with bias on
 * its Linear layers (Mixtral textbook page, section "Подсчёт параметров": the
 * teaching configuration puts a bias on every Linear):
 *     h = SiLU(x W1_e + b1_e) (.) (x W3_e + b3_e),   o = h W2_e + b2_e
 *   b1, b3 [E,d_ff] float, b2 [E,d] float (in; each may be NULL = no bias)
 * The biases are added in float32 to the float32 accumulators, before SiLU and
 * the product (b1, b3) and before o is stored (b2).  Everything else as for
 * moe_expert_swiglu.
 */
int moe_expert_swiglu_bias(moe_shape s, const void* x_sorted, const int32_t* offsets,
                           const void* W1, const void* W3, const void* W2, const float* b1,
                           const float* b3, const float* b2, void* h, float* o, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * moe_expert_swiglu_stall_test -- test hook for the error path of the bounded
 * device waits (no counterpart on the pages).  Runs moe_expert_swiglu with its
 * TMA producer stopping after `stall_after` (>= 0) pipeline stages, as if it had
 * died, and every device wait bounded by `timeout_ns` (1e3 .. 2e9).  The waiting
 * roles give up after timeout_ns, drain their copies and MMAs, free tensor
 * memory and return; moe_read_device_status(ws) then reports
 * MOE_ERR_DEVICE_TIMEOUT and the CUDA context stays usable.  h and o are left
 * incomplete.
 */
int moe_expert_swiglu_stall_test(moe_shape s, const void* x_sorted, const int32_t* offsets,
                                 const void* W1, const void* W3, const void* W2, void* h, float* o,
                                 void* ws, size_t ws_bytes, int stall_after,
                                 uint64_t timeout_ns, void* stream);

/*
 * moe_combine -- y[t] = sum over slots s (in slot order) of gate[t,s] * o[inv[t,s]]
 * (the combine step of section "Алгоритм": each token's output accumulates the
 * gate-weighted outputs of the experts it was sent to, k terms per token).
 * Products and sums in float32 without fused multiply-add; y rounded to bf16.
 *   o [T*k,d] float, inv [T,k] int32, gate [T,k] float (in);  y [T,d] bf16 (out)
 * Slots with inv < 0 are skipped.
 */
int moe_combine(moe_shape s, const float* o, const int32_t* inv, const float* gate, void* y,
                void* stream);

/*
 * moe_forward -- the whole layer: route, dispatch, experts, combine.
 * Page: the MoE equation of section "Прямой проход в формулах"
 * (MoE(u) = sum_{i in S} w_i Expert_i(u)), computed in the order of section
 * "Алгоритм" (route every token, then one pass per expert over its tokens,
 * then k gate-weighted terms per token).
 *   x, Wg, bias (nullable), W1, W3, W2 as above (in);  y [T,d] bf16 (out)
 *   idx_out [T,k] int32, gate_out [T,k] float: copies of the routing, or NULL
 *   ws: >= moe_forward_workspace_bytes(s) bytes of device memory
 * y has the bits of moe_route -> moe_dispatch -> moe_expert_swiglu -> moe_combine
 * on the same inputs; at large batches (4 or more rounds of the down
 * projection's CTA-pair tiles) the combine runs inside that GEMM's epilogue.
 */
int moe_forward(moe_shape s, const void* x, const void* Wg, const float* bias, const void* W1,
                const void* W3, const void* W2, void* y, int32_t* idx_out, float* gate_out,
                void* ws, size_t ws_bytes, void* stream);

/*
 * moe_forward_bias -- moe_forward with the biases of the expert Linear layers
 * (b1, b3 [E,d_ff], b2 [E,d] float, each nullable; see moe_expert_swiglu_bias).
 * Page: section "Подсчёт параметров" (the teaching configuration puts a bias on
 * every Linear, so each expert computes SiLU(u W1 + b1) (.) (u W3 + b3) W2 + b2).
 * The router bias is `bias`, as for moe_forward.
 */
int moe_forward_bias(moe_shape s, const void* x, const void* Wg, const float* bias,
                     const void* W1, const void* W3, const void* W2, const float* b1,
                     const float* b3, const float* b2, void* y, int32_t* idx_out,
                     float* gate_out, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_forward_profiled -- moe_forward (no idx/gate copies) that also records
 * seven caller-created CUDA events (cudaEvent_t handles) on `stream` between its
 * launches: events[0] before the router, [1] after the router, [2] after the
 * dispatch index kernel, [3] after the dispatch scatter, [4] after GEMM1
 * (x W1 | x W3 -> h), [5] after GEMM2 (h W2 -> o), [6] after the combine
 * (right after [5] when the batch is large enough for the combine to run in
 * GEMM2's epilogue: at least 4 rounds of its CTA-pair tiles).
 * n_events must be 7.  Measurement hook with no counterpart on the pages.
 */
int moe_forward_profiled(moe_shape s, const void* x, const void* Wg, const float* bias,
                         const void* W1, const void* W3, const void* W2, void* y, void* ws,
                         size_t ws_bytes, void* const* events, int n_events, void* stream);

/*
 * moe_block_forward -- the MoE half of a decoder block with its edges
 * (Mixtral textbook page, section "Прямой проход в формулах"):
 *     H = U + MoE(RMSNorm_2(U)),   RMSNorm(z) = z / sqrt(mean_j z_j^2 + eps) (.) gamma
 *   U [T,d] bf16: the residual stream after attention (in)
 *   gamma [d] bf16: RMSNorm_2 scale; eps >= 0 (rms_norm_eps, 1e-5 for Mixtral) (in)
 *   Wg, bias, W1, W3, W2 as for moe_forward (in);  H [T,d] bf16 (out)
 *   ws: >= moe_block_workspace_bytes(s) bytes of device memory
 * The normalised rows are rounded to bf16 (the layer's input); the router
 * computes them while it reads U and leaves them in the workspace, at byte
 * offset moe_forward_workspace_bytes(s) ([T,d] bf16), for the dispatch.  The
 * residual is added in float32 to the combined expert outputs before the one
 * rounding of H.
 */
size_t moe_block_workspace_bytes(moe_shape s);
int moe_block_forward(moe_shape s, const void* U, const void* gamma, float eps, const void* Wg,
                      const float* bias, const void* W1, const void* W3, const void* W2, void* H,
                      void* ws, size_t ws_bytes, void* stream);

/*
 * moe_forward_hostio -- moe_forward with x and y in HOST memory (pinned memory
 * gives asynchronous copies): copies x into the workspace, runs the layer and
 * copies y back; everything is ordered after earlier work on `stream`, and
 * `stream` is ordered after the last copy, so the caller synchronises `stream`
 * before reading y.  Weights stay on the device.  Batches of 2048 tokens or
 * more are split into three token chunks (T/8 rounded down to a multiple of 64
 * tokens, the rest, and T/8 again) whose copies run on two library-owned copy
 * streams (created once per device) while the other chunks compute, so only
 * the first chunk's upload and the last chunk's download are not overlapped:
 * the layer is independent per token, so y is the same bit for bit.  Calls
 * from several host threads on one device are enqueued one at a time.
 *   ws: >= moe_forward_workspace_bytes(s) + T*d*2 (x staging) + T*d*2 (y staging)
 *       bytes; moe_forward_hostio_workspace_bytes gives the exact figure.
 */
size_t moe_forward_hostio_workspace_bytes(moe_shape s);
int moe_forward_hostio(moe_shape s, const void* x_host, const void* Wg, const float* bias,
                       const void* W1, const void* W3, const void* W2, void* y_host, void* ws,
                       size_t ws_bytes, void* stream);

/*
 * moe_forward_hostio_batches -- moe_forward over n_batches independent batches
 * of T tokens each with the same weights, batch b read from the host buffer
 * x_host[b] and written to the host buffer y_host[b] (pinned memory gives
 * asynchronous copies); the loop of a server that feeds the layer a queue of
 * batches.  Each batch runs the whole layer once (the weights are streamed once
 * per batch, not once per token chunk), on `stream`; for small batches
 * (T*k*d*d_ff < 2^34, e.g. decode-sized ones) odd batches run on a second,
 * library-owned compute stream with their own part of ws, so two consecutive
 * batches' short kernels overlap; batch
 * b+1's upload and batch b-1's download run on the library's two copy streams
 * while batch b computes, through two staging slots each for x and y in ws, so
 * only the first upload and the last download are not overlapped.  y_host[b]
 * equals moe_forward on x_host[b] bit for bit.  Everything is ordered after
 * earlier work on `stream`, and `stream` after the last download and the
 * second compute stream's last layer.  The status word (at the start of ws) is
 * cleared once, before the first batch, and every layer reports into it, so an
 * expired wait in any batch stays reported.
 *   x_host, y_host: arrays of n_batches host pointers (none null), each buffer
 *       T*d bf16, row-major; a buffer may appear more than once (the caller
 *       owns the data order: y_host[b] is written when batch b's download runs).
 *   ws: >= moe_forward_workspace_bytes(s) (twice for small batches) + 2
 *       x-staging + 2 y-staging slots of T*d*2 bytes;
 *       moe_forward_hostio_batches_workspace_bytes gives the figure.
 * Errors: MOE_ERR_INVALID_ARG for n_batches < 1 or a null array or entry,
 * MOE_ERR_WORKSPACE for a short ws; T == 0 enqueues nothing.
 */
size_t moe_forward_hostio_batches_workspace_bytes(moe_shape s);
int moe_forward_hostio_batches(moe_shape s, int n_batches, const void* const* x_host,
                               const void* Wg, const float* bias, const void* W1,
                               const void* W3, const void* W2, void* const* y_host, void* ws,
                               size_t ws_bytes, void* stream);

/*
 * moe_forward_hostio_batches_stall_test -- test hook for the error path of the
 * queue of batches (no counterpart on the pages).  Runs
 * moe_forward_hostio_batches with the expert kernels' TMA producer of batch
 * `stall_batch` (0 = first; past the last stalls nothing) stopping after
 * `stall_after` (>= 0) pipeline stages, and that batch's device waits bounded
 * by `timeout_ns` (1e3 .. 2e9).  The status word is cleared once, before the
 * first batch, so moe_read_device_status(ws) reports MOE_ERR_DEVICE_TIMEOUT
 * whichever batch's wait expired; that batch's y is incomplete, the others'
 * are right, and the CUDA context stays usable.
 */
int moe_forward_hostio_batches_stall_test(moe_shape s, int n_batches,
                                          const void* const* x_host, const void* Wg,
                                          const float* bias, const void* W1, const void* W3,
                                          const void* W2, void* const* y_host, void* ws,
                                          size_t ws_bytes, int stall_batch, int stall_after,
                                          uint64_t timeout_ns, void* stream);

/*
 * moe_forward_hostio_stall_test -- test hook for the error path of the chunked
 * host-I/O pipeline (no counterpart on the pages).  Runs moe_forward_hostio with
 * the expert kernels' TMA producer of token chunk `stall_chunk` (0 = first;
 * batches of 2048+ tokens run as three chunks, smaller ones as one; a chunk index
 * past the last stalls nothing) stopping after `stall_after` (>= 0) pipeline
 * stages, and that chunk's device waits bounded by `timeout_ns` (1e3 .. 2e9).
 * The status word is cleared once per call, before the first chunk, so
 * moe_read_device_status(ws) reports MOE_ERR_DEVICE_TIMEOUT whichever chunk's
 * wait expired.  y is then incomplete; the CUDA context stays usable.
 */
int moe_forward_hostio_stall_test(moe_shape s, const void* x_host, const void* Wg,
                                  const float* bias, const void* W1, const void* W3,
                                  const void* W2, void* y_host, void* ws, size_t ws_bytes,
                                  int stall_chunk, int stall_after, uint64_t timeout_ns,
                                  void* stream);

/*
 * moe_aux_loss -- load-balancing auxiliary term of the router (Mixtral textbook
 * page, section "Load-balancing loss"):
 *     aux = E * sum_{s<k} sum_{i<E} f_{s,i} * P_i
 * f_{s,i}: fraction of the counted tokens whose top-k slot s holds expert i;
 * P_i: mean over the counted tokens of the softmax over all E router logits.
 * The training loss adds alpha * aux (alpha = router_aux_loss_coef); under
 * uniform load aux = k.  The page gathers the statistic over all MoE layers at
 * once: pass the layers' logits and idx stacked as T = layers * tokens rows.
 *   logits [T,E] float (moe_route's logits), idx [T,k] int32 (in)
 *   mask [T] uint8 or NULL: rows with 0 (padding) are not counted (in)
 *   aux [1] float (out); f [k,E] float, P [E] float: the statistics, or NULL (out)
 * Only s.T, s.E and s.k are used (s.d and s.d_ff are ignored).  Deterministic
 * (fixed reduction order); aux = 0 when no row is counted.
 */
int moe_aux_loss(moe_shape s, const float* logits, const int32_t* idx, const uint8_t* mask,
                 float* aux, float* f, float* P, void* stream);

/*
 * moe_forward_static -- moe_forward for callers that cannot allocate device
 * memory.  No counterpart on the pages: it exists for callers such as code
 * running while a stream is being captured into a CUDA graph (where cudaMalloc
 * is not allowed), plugins that run inside a host framework which owns every
 * allocation and hands out none, and latency-critical serving loops that must
 * not hit cudaMalloc's implicit device synchronisation.  Instead of a
 * caller-provided workspace it uses a fixed scratch array of 8 MiB
 * (MOE_STATIC_SCRATCH_BYTES) in device memory, compiled into the library; every
 * GPU on which the library is loaded reserves it until the process exits.  The
 * caller still passes every input and the output y, all in device memory.
 *  - Limit: shapes with moe_forward_workspace_bytes(s) > 8 MiB are rejected
 *    with MOE_ERR_WORKSPACE before anything is launched (for d = 4096,
 *    d_ff = 14336, k = 2 that allows T <= 78 tokens: decode-sized batches).
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture begins.
 *  - Calls share the one array and it keeps the previous call's contents; the
 *    call clears the part that must start at zero (its status word) itself.
 *    Calls whose work overlaps on the GPU (different streams, or different
 *    host threads, on one device) race on the array: serialise them.
 *  - device_status: nullable device int32; when given, it receives the call's
 *    status word (0, or nonzero after an expired device wait; see
 *    moe_read_device_status) once the call's work has run.  With T == 0 nothing
 *    is launched except the write of 0 to device_status.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
#define MOE_STATIC_SCRATCH_BYTES (8u << 20)
int moe_forward_static(moe_shape s, const void* x, const void* Wg, const float* bias,
                       const void* W1, const void* W3, const void* W2, void* y,
                       int32_t* device_status, void* stream);

/*
 * moe_read_device_status -- SYNCHRONISES `stream`, then reads the status word
 * that moe_expert_swiglu / moe_forward keep at the start of their workspace:
 * MOE_OK, or MOE_ERR_DEVICE_TIMEOUT when a bounded device wait gave up
 * (the kernel then stopped issuing work, drained its copies, freed its tensor
 * memory and returned).  The word is reset by the next call that uses `ws`.
 */
int moe_read_device_status(const void* ws, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
