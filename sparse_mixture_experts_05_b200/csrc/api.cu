// api.cu -- the C ABI declared in include/moe.h: argument checks, workspace
// carving and the launch sequence of the MoE layer.
//
// The launch sequence follows the loop of the Mixtral textbook page, section
// "Алгоритм": route (topk of X W_r, softmax over the k), dispatch (per-expert
// token lists), experts (one grouped pass per GEMM over all expert groups),
// combine (k gate-weighted terms per token).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "aux_loss.cuh"
#include "combine.cuh"
#include "common.cuh"
#include "dispatch.cuh"
#include "expert_gemm.cuh"
#include "router.cuh"

namespace moe {

int device_sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

namespace {

constexpr size_t kAlign = 256;

int check_shape(const moe_shape& s) {
    if (s.T < 0 || s.d <= 0 || s.d_ff <= 0 || s.E <= 0 || s.k <= 0) return MOE_ERR_INVALID_ARG;
    if (s.k > s.E) return MOE_ERR_INVALID_ARG;  // top_k_experts must lie in 1 .. num_experts
    if (s.E > 32 || s.k > 8) return MOE_ERR_UNSUPPORTED;
    if (s.d % 128 != 0 || s.d_ff % 128 != 0) return MOE_ERR_UNSUPPORTED;
    const int64_t R = (int64_t)s.T * s.k;
    if (R * (int64_t)std::max(s.d, s.d_ff) >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
    if ((int64_t)s.E * std::max(s.d, s.d_ff) >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
    if ((int64_t)16 * s.d * ((s.E + 7) / 8) > 163840) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }

// Workspace of moe_forward, in order; every segment starts on a 256-byte boundary.
struct FwdLayout {
    size_t hdr, idx, gate, offsets, perm, inv, x_sorted, h, o, cnt, total;
};

FwdLayout fwd_layout(const moe_shape& s) {
    const size_t T = (size_t)s.T, R = (size_t)s.T * s.k;
    FwdLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes, kAlign);
        return at;
    };
    L.hdr = take(kWsHeaderBytes);
    L.idx = take(T * s.k * 4);
    L.gate = take(T * s.k * 4);
    L.offsets = take((size_t)(s.E + 1) * 4);
    L.perm = take(R * 4);
    L.inv = take(R * 4);
    L.x_sorted = take(R * s.d * 2);
    L.h = take(R * s.d_ff * 2);
    L.o = take(R * s.d * 4);
    // counters of the combine fused into the down projection (when it can be)
    L.cnt = take(combine_fusable(s) ? T * (s.d / 128) * 4 : 0);
    L.total = off;
    return L;
}

template <typename T>
T* at(void* base, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

constexpr int kProfileEvents = 7;

// Biases of the expert Linear layers (each nullable): b1, b3 [E, d_ff], b2 [E, d].
struct ExpertBias {
    const float* b1 = nullptr;
    const float* b3 = nullptr;
    const float* b2 = nullptr;
};

// Variations of one forward pass.
struct FwdOptions {
    const void* residual = nullptr;  // [T, d] bf16 added before the rounding of y (block edge)
    ExpertBias eb;                   // expert Linear biases
    int router_cluster = 0;          // router cluster size, fixing its k split (0: chosen for this T)
    bool clear_status = true;        // the router (first kernel) zeroes the status word first
    int stall_after = -1;            // test hook: expert producer stops after this many stages
    uint64_t timeout_ns = kDefaultWaitTimeoutNs;  // bound on every device wait
    const RouterNorm* norm = nullptr;  // block edge: x is U, the router forms u = RMSNorm_2(U)
    int* status = nullptr;           // status word (nullptr: the workspace header's)
};

// Records events[i] (when given) between the launches: 0 before the router, 1
// after it, 2 after the dispatch index kernel, 3 after the scatter, 4 after
// GEMM1, 5 after GEMM2, 6 after the combine (right after 5 when the combine is
// fused into GEMM2).
int forward_impl(const moe_shape& s, const void* x, const void* Wg, const float* bias,
                 const void* W1, const void* W3, const void* W2, void* y, int32_t* idx_out,
                 float* gate_out, void* ws, cudaStream_t st, void* const* events,
                 const FwdOptions& opt = FwdOptions{}) {
    auto mark = [&](int i) {
        return !events || cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st) == cudaSuccess;
    };
    const FwdLayout L = fwd_layout(s);
    int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, L.idx);
    float* gate = gate_out ? gate_out : at<float>(ws, L.gate);
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* perm = at<int32_t>(ws, L.perm);
    int32_t* inv = at<int32_t>(ws, L.inv);
    void* xs = at<void>(ws, L.x_sorted);
    void* h = at<void>(ws, L.h);
    float* o = at<float>(ws, L.o);
    int* status = opt.status ? opt.status : at<int>(ws, L.hdr);
    if (!mark(0)) return MOE_ERR_CUDA;
    int rc = launch_router(s, x, Wg, bias, idx, gate, nullptr, st, opt.router_cluster, opt.norm,
                           status, opt.clear_status);
    if (rc) return rc;
    if (!mark(1)) return MOE_ERR_CUDA;
    rc = launch_dispatch_index(s, idx, offsets, perm, inv, st);
    if (rc) return rc;
    if (!mark(2)) return MOE_ERR_CUDA;
    // the experts' rows: the layer input, or the router's normalised rows u
    // A routed batch that gives the down projection several rounds of CTA-pair
    // tiles has the combine fused into that GEMM's epilogue (same bits, one
    // launch less).
    const bool fused = combine_fused(s);
    int* cnt = fused ? at<int>(ws, L.cnt) : nullptr;
    rc = launch_dispatch_scatter(s, opt.norm ? opt.norm->u : x, inv, xs, st, cnt);
    if (rc) return rc;
    if (!mark(3)) return MOE_ERR_CUDA;
    FusedCombine fc;
    fc.perm_tok = perm;
    fc.inv = inv;
    fc.gate = gate;
    fc.residual = opt.residual;
    fc.y = y;
    fc.cnt = cnt;
    rc = expert_gemms(s, xs, offsets, W1, W3, W2, h, o, status, opt.timeout_ns, opt.stall_after,
                      st, events ? events[4] : nullptr, opt.eb.b1, opt.eb.b3, opt.eb.b2,
                      fused ? &fc : nullptr);
    if (rc) return rc;
    if (!mark(5)) return MOE_ERR_CUDA;
    if (!fused) {
        rc = launch_combine(s, o, inv, gate, y, st, opt.residual);
        if (rc) return rc;
    }
    return mark(6) ? MOE_OK : MOE_ERR_CUDA;
}

// Scratch of moe_forward_static: a fixed 8 MiB array in device memory that
// every GPU which loads this library holds until the process exits.  Host code
// only ever sees a host-side stand-in for this name; the device address comes
// from cudaGetSymbolAddress, once per device.
constexpr size_t kStaticScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device (looked up on the
// first call per device, with that device current).  nullptr on failure.
void* static_scratch_address() {
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

// moe_forward_hostio splits batches of 2048+ tokens into three token chunks:
// a small first chunk (T/8 rounded down to 64 tokens), the bulk, and a small
// last chunk of the same size.  Copies run ahead of the computation (a token's
// 8 KB cross the host link faster than the layer processes it), so only the
// first chunk's upload and the last chunk's download are exposed; keeping those
// chunks small shortens both, while the bulk keeps the GEMM tiles full.
// (Two equal halves exposed 16 MiB each way at T = 4096; four equal chunks
// measured slower, the down projection's tiles filling fewer rounds.)
constexpr int kMaxHostioChunks = 3;
int hostio_chunks(int T, int (&sizes)[kMaxHostioChunks]) {
    if (T < 2048) {
        sizes[0] = T;
        return 1;
    }
    const int edge = (T / 8) / 64 * 64;
    sizes[0] = edge;
    sizes[1] = T - 2 * edge;
    sizes[2] = edge;
    return 3;
}

// Two copy streams (host->device, device->host) and the events that order them
// against the caller's stream; created once per device and kept for the life
// of the process.  The mutex serialises the enqueueing of one call's pipeline.
struct CopyStreams {
    cudaStream_t up = nullptr, down = nullptr;
    // moe_forward_hostio_batches: the second compute stream (odd batches)
    cudaStream_t comp = nullptr;
    cudaEvent_t ev[2 + 2 * kMaxHostioChunks] = {};
    // moe_forward_hostio_batches: start, x landed in slot 0/1, slot 0/1's layer
    // done, slot 0/1's y left, copies' end, second compute stream's end
    cudaEvent_t evb[9] = {};
    std::mutex mu;
};

CopyStreams* copy_streams() {
    static std::mutex mu;
    static CopyStreams* per_device[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!per_device[dev]) {
        CopyStreams* cs = new CopyStreams();
        bool ok = cudaStreamCreateWithFlags(&cs->up, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&cs->down, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&cs->comp, cudaStreamNonBlocking) == cudaSuccess;
        for (auto& e : cs->ev)
            ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
        for (auto& e : cs->evb)
            ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
        if (!ok) return nullptr;  // (leaks the partial set; only on a failing device)
        per_device[dev] = cs;
    }
    return per_device[dev];
}

// moe_forward_hostio with an optional stall of the expert producer in chunk
// `stall_chunk` (test hook; -1: none).  The status word is cleared once, by the
// first chunk's router kernel: a later chunk must not erase an expired wait that
// an earlier chunk recorded.
int hostio_impl(const moe_shape& s, const void* x_host, const void* Wg, const float* bias,
                const void* W1, const void* W3, const void* W2, void* y_host, void* ws,
                size_t ws_bytes, cudaStream_t st, int stall_chunk, int stall_after,
                uint64_t timeout_ns) {
    int rc = check_shape(s);
    if (rc || s.T == 0) return rc;
    if (!x_host || !y_host || !ok_ptr(Wg) || !ok_opt(bias) || !ok_ptr(W1) || !ok_ptr(W3) ||
        !ok_ptr(W2) || !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_forward_hostio_workspace_bytes(s)) return MOE_ERR_WORKSPACE;
    const size_t fwd = moe_forward_workspace_bytes(s);
    const size_t io_bytes = (size_t)s.T * s.d * 2;
    char* x_dev = static_cast<char*>(ws) + fwd;
    char* y_dev = static_cast<char*>(ws) + fwd + align_up(io_bytes, 256);
    auto chunk_opt = [&](int c) {
        FwdOptions opt;
        opt.clear_status = c == 0;
        if (c == stall_chunk) {
            opt.stall_after = stall_after;
            opt.timeout_ns = timeout_ns;
        }
        return opt;
    };
    int sizes[kMaxHostioChunks];
    const int chunks = hostio_chunks(s.T, sizes);
    if (chunks == 1) {
        if (cudaMemcpyAsync(x_dev, x_host, io_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
            return MOE_ERR_CUDA;
        rc = forward_impl(s, x_dev, Wg, bias, W1, W3, W2, y_dev, nullptr, nullptr, ws, st,
                          nullptr, chunk_opt(0));
        if (rc) return rc;
        if (cudaMemcpyAsync(y_host, y_dev, io_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    // Token chunks in a pipeline: the layer is independent per token, so chunk c
    // computes (on `st`) while chunk c+1's x is still arriving and chunk c-1's y
    // is leaving, on the two copy engines.  The result equals the unchunked
    // layer bit for bit: no row's arithmetic depends on the other rows.
    CopyStreams* cs = copy_streams();
    if (!cs) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(cs->mu);
    int start[kMaxHostioChunks + 1] = {0};
    for (int c = 0; c < chunks; ++c) start[c + 1] = start[c] + sizes[c];
    const int split = router_cluster(s);  // the whole batch's: every chunk rounds alike
    const size_t row_bytes = (size_t)s.d * 2;
    bool ok = cudaEventRecord(cs->ev[0], st) == cudaSuccess &&
              cudaStreamWaitEvent(cs->up, cs->ev[0], 0) == cudaSuccess &&
              cudaStreamWaitEvent(cs->down, cs->ev[0], 0) == cudaSuccess;
    for (int c = 0; ok && c < chunks; ++c) {
        const int t0 = start[c], tn = sizes[c];
        ok = cudaMemcpyAsync(x_dev + t0 * row_bytes, static_cast<const char*>(x_host) + t0 * row_bytes,
                             (size_t)tn * row_bytes, cudaMemcpyHostToDevice, cs->up) == cudaSuccess &&
             cudaEventRecord(cs->ev[1 + c], cs->up) == cudaSuccess;
    }
    for (int c = 0; ok && c < chunks; ++c) {
        const int t0 = start[c], tn = sizes[c];
        moe_shape sc = s;
        sc.T = tn;
        FwdOptions opt = chunk_opt(c);
        opt.router_cluster = split;
        ok = cudaStreamWaitEvent(st, cs->ev[1 + c], 0) == cudaSuccess &&
             forward_impl(sc, x_dev + t0 * row_bytes, Wg, bias, W1, W3, W2, y_dev + t0 * row_bytes,
                          nullptr, nullptr, ws, st, nullptr, opt) == MOE_OK &&
             cudaEventRecord(cs->ev[1 + kMaxHostioChunks + c], st) == cudaSuccess &&
             cudaStreamWaitEvent(cs->down, cs->ev[1 + kMaxHostioChunks + c], 0) == cudaSuccess &&
             cudaMemcpyAsync(static_cast<char*>(y_host) + t0 * row_bytes, y_dev + t0 * row_bytes,
                             (size_t)tn * row_bytes, cudaMemcpyDeviceToHost,
                             cs->down) == cudaSuccess;
    }
    // join: the caller's stream waits for the last copy back
    const int last = 1 + 2 * kMaxHostioChunks;
    ok = ok && cudaEventRecord(cs->ev[last], cs->down) == cudaSuccess &&
         cudaStreamWaitEvent(st, cs->ev[last], 0) == cudaSuccess;
    return ok ? MOE_OK : MOE_ERR_CUDA;
}

// moe_forward_hostio_batches: n independent batches through two staging slots.
// Batch b uses slot b & 1; its upload waits until batch b-2's layer has read
// the slot's x (so it runs while batch b-1 computes), its layer waits for its x
// and for batch b-2's y to have left the slot, and its download runs while
// batch b+1 computes.  Each batch is one whole-batch forward, so the weights
// are streamed once per batch and y_host[b] equals moe_forward on x_host[b].
// Whether moe_forward_hostio_batches runs alternate batches on two compute
// streams: only for batches whose expert GEMMs are small (R d d_ff < 2^34, e.g.
// the decode batch or the quarter-width one).  Measured on a queue of 20
// batches, two streams against one: decode 0.421 vs 0.443 ms a batch, quarter
// width 0.081 vs 0.089, but the Mixtral prefill batch 2.72 vs 2.36 ms -- its
// persistent GEMM grids, dealt their tiles up front, lose SMs to the other
// stream's kernels and wait for them.
bool queue_two_streams(const moe_shape& s) {
    return (int64_t)s.T * s.k * s.d * (int64_t)s.d_ff < (int64_t(1) << 34);
}

int hostio_batches_impl(const moe_shape& s, int nb, const void* const* x_host, const void* Wg,
                        const float* bias, const void* W1, const void* W3, const void* W2,
                        void* const* y_host, void* ws, size_t ws_bytes, cudaStream_t st,
                        int stall_batch = -1, int stall_after = -1,
                        uint64_t timeout_ns = kDefaultWaitTimeoutNs) {
    int rc = check_shape(s);
    if (rc) return rc;
    if (nb < 1 || !x_host || !y_host) return MOE_ERR_INVALID_ARG;
    for (int b = 0; b < nb; ++b)
        if (!x_host[b] || !y_host[b]) return MOE_ERR_INVALID_ARG;
    if (s.T == 0) return MOE_OK;
    if (!ok_ptr(Wg) || !ok_opt(bias) || !ok_ptr(W1) || !ok_ptr(W3) || !ok_ptr(W2) || !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_forward_hostio_batches_workspace_bytes(s)) return MOE_ERR_WORKSPACE;
    const size_t io_bytes = (size_t)s.T * s.d * 2;
    const size_t slot = align_up(io_bytes, 256);
    const size_t fwd = moe_forward_workspace_bytes(s);
    const bool two = queue_two_streams(s);
    char* base = static_cast<char*>(ws) + (two ? 2 : 1) * fwd;
    int* status = at<int>(ws, fwd_layout(s).hdr);  // every layer reports here
    CopyStreams* cs = copy_streams();
    if (!cs) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(cs->mu);
    // Small batches: even batches run on the caller's stream with workspace part
    // 0, odd ones on a second compute stream with part 1, so one batch's short
    // kernels overlap the other's.  Large ones all run on the caller's stream.
    cudaStream_t comp[2] = {st, two ? cs->comp : st};
    // [0] start, [1+i] x in slot i, [3+i] slot i's layer done, [5+i] y out of
    // slot i, [7] copies' end, [8] second compute stream's end
    cudaEvent_t* ev = cs->evb;
    bool ok = cudaMemsetAsync(status, 0, sizeof(int), st) == cudaSuccess &&
              cudaEventRecord(ev[0], st) == cudaSuccess &&
              cudaStreamWaitEvent(cs->up, ev[0], 0) == cudaSuccess &&
              cudaStreamWaitEvent(cs->down, ev[0], 0) == cudaSuccess &&
              cudaStreamWaitEvent(cs->comp, ev[0], 0) == cudaSuccess;
    for (int b = 0; ok && b < nb; ++b) {
        const int i = b & 1;
        cudaStream_t cst = comp[i];
        char* x_dev = base + (size_t)i * slot;
        char* y_dev = base + (size_t)(2 + i) * slot;
        if (b >= 2) ok = cudaStreamWaitEvent(cs->up, ev[3 + i], 0) == cudaSuccess;
        ok = ok &&
             cudaMemcpyAsync(x_dev, x_host[b], io_bytes, cudaMemcpyHostToDevice, cs->up) ==
                 cudaSuccess &&
             cudaEventRecord(ev[1 + i], cs->up) == cudaSuccess &&
             cudaStreamWaitEvent(cst, ev[1 + i], 0) == cudaSuccess;
        if (ok && b >= 2) ok = cudaStreamWaitEvent(cst, ev[5 + i], 0) == cudaSuccess;
        FwdOptions opt;
        opt.clear_status = false;  // cleared once above: an expired wait in any batch stays
        opt.status = status;
        if (b == stall_batch) {
            opt.stall_after = stall_after;
            opt.timeout_ns = timeout_ns;
        }
        ok = ok &&
             forward_impl(s, x_dev, Wg, bias, W1, W3, W2, y_dev, nullptr, nullptr,
                          static_cast<char*>(ws) + (two ? (size_t)i * fwd : 0), cst, nullptr,
                          opt) == MOE_OK &&
             cudaEventRecord(ev[3 + i], cst) == cudaSuccess &&
             cudaStreamWaitEvent(cs->down, ev[3 + i], 0) == cudaSuccess &&
             cudaMemcpyAsync(y_host[b], y_dev, io_bytes, cudaMemcpyDeviceToHost, cs->down) ==
                 cudaSuccess &&
             cudaEventRecord(ev[5 + i], cs->down) == cudaSuccess;
    }
    ok = ok && cudaEventRecord(ev[7], cs->down) == cudaSuccess &&
         cudaEventRecord(ev[8], cs->comp) == cudaSuccess &&
         cudaStreamWaitEvent(st, ev[7], 0) == cudaSuccess &&
         cudaStreamWaitEvent(st, ev[8], 0) == cudaSuccess;
    return ok ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument (null/misaligned pointer, k outside 1..E, negative size)";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape outside the supported limits";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace too small";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or kernel launch failed";
        case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT: a bounded device-side wait expired";
        default: return "unknown moe status";
    }
}

int moe_check_shape(moe_shape s) { return check_shape(s); }

size_t moe_expert_workspace_bytes(moe_shape s) {
    if (check_shape(s)) return 0;
    return kWsHeaderBytes;
}

size_t moe_forward_workspace_bytes(moe_shape s) {
    if (check_shape(s)) return 0;
    return fwd_layout(s).total;
}

int moe_forward_kernel_count(moe_shape s) {
    if (const int rc = check_shape(s)) return -rc;
    if (s.T == 0) return 0;
    return combine_fused(s) ? 5 : 6;
}

size_t moe_block_workspace_bytes(moe_shape s) {
    if (check_shape(s)) return 0;
    return fwd_layout(s).total + align_up((size_t)s.T * s.d * 2, 256);
}

size_t moe_forward_hostio_workspace_bytes(moe_shape s) {
    if (check_shape(s)) return 0;
    const size_t io = align_up((size_t)s.T * s.d * 2, 256);
    return fwd_layout(s).total + 2 * io;
}

size_t moe_forward_hostio_batches_workspace_bytes(moe_shape s) {
    if (check_shape(s)) return 0;
    const size_t io = align_up((size_t)s.T * s.d * 2, 256);
    // a forward workspace per compute stream
    return (queue_two_streams(s) ? 2 : 1) * fwd_layout(s).total + 4 * io;
}

int moe_route(moe_shape s, const void* x, const void* Wg, const float* bias, int32_t* idx,
              float* gate, float* logits, void* stream) {
    int rc = check_shape(s);
    if (rc || s.T == 0) return rc;
    if (!ok_ptr(x) || !ok_ptr(Wg) || !ok_opt(bias) || !ok_ptr(idx) || !ok_ptr(gate) ||
        !ok_opt(logits))
        return MOE_ERR_INVALID_ARG;
    return launch_router(s, x, Wg, bias, idx, gate, logits, static_cast<cudaStream_t>(stream));
}

int moe_dispatch(moe_shape s, const int32_t* idx, const void* x, int32_t* offsets,
                 int32_t* perm_tok, int32_t* inv, void* x_sorted, void* stream) {
    int rc = check_shape(s);
    if (rc) return rc;
    if (!ok_ptr(offsets)) return MOE_ERR_INVALID_ARG;
    if (s.T > 0 && (!ok_ptr(idx) || !ok_ptr(x) || !ok_ptr(perm_tok) || !ok_ptr(inv) ||
                    !ok_ptr(x_sorted)))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = launch_dispatch_index(s, idx, offsets, perm_tok, inv, st);
    if (rc) return rc;
    return launch_dispatch_scatter(s, x, inv, x_sorted, st);
}

int moe_expert_swiglu(moe_shape s, const void* x_sorted, const int32_t* offsets, const void* W1,
                      const void* W3, const void* W2, void* h, float* o, void* ws,
                      size_t ws_bytes, void* stream) {
    int rc = check_shape(s);
    if (rc || s.T == 0) return rc;
    if (!ok_ptr(x_sorted) || !ok_ptr(offsets) || !ok_ptr(W1) || !ok_ptr(W3) || !ok_ptr(W2) ||
        !ok_ptr(h) || !ok_ptr(o) || !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_expert_workspace_bytes(s)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) return MOE_ERR_CUDA;
    return expert_gemms(s, x_sorted, offsets, W1, W3, W2, h, o, static_cast<int*>(ws),
                        kDefaultWaitTimeoutNs, -1, st, nullptr);
}

int moe_expert_swiglu_bias(moe_shape s, const void* x_sorted, const int32_t* offsets,
                           const void* W1, const void* W3, const void* W2, const float* b1,
                           const float* b3, const float* b2, void* h, float* o, void* ws,
                           size_t ws_bytes, void* stream) {
    int rc = check_shape(s);
    if (rc || s.T == 0) return rc;
    if (!ok_ptr(x_sorted) || !ok_ptr(offsets) || !ok_ptr(W1) || !ok_ptr(W3) || !ok_ptr(W2) ||
        !ok_opt(b1) || !ok_opt(b3) || !ok_opt(b2) || !ok_ptr(h) || !ok_ptr(o) || !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_expert_workspace_bytes(s)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) return MOE_ERR_CUDA;
    return expert_gemms(s, x_sorted, offsets, W1, W3, W2, h, o, static_cast<int*>(ws),
                        kDefaultWaitTimeoutNs, -1, st, nullptr, b1, b3, b2);
}

int moe_expert_swiglu_stall_test(moe_shape s, const void* x_sorted, const int32_t* offsets,
                                 const void* W1, const void* W3, const void* W2, void* h, float* o,
                                 void* ws, size_t ws_bytes, int stall_after,
                                 uint64_t timeout_ns, void* stream) {
    int rc = check_shape(s);
    if (rc || s.T == 0) return rc;
    if (!ok_ptr(x_sorted) || !ok_ptr(offsets) || !ok_ptr(W1) || !ok_ptr(W3) || !ok_ptr(W2) ||
        !ok_ptr(h) || !ok_ptr(o) || !ok_ptr(ws) || stall_after < 0)
        return MOE_ERR_INVALID_ARG;
    if (timeout_ns < 1000 || timeout_ns > kDefaultWaitTimeoutNs) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_expert_workspace_bytes(s)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) return MOE_ERR_CUDA;
    return expert_gemms(s, x_sorted, offsets, W1, W3, W2, h, o, static_cast<int*>(ws), timeout_ns,
                        stall_after, st, nullptr);
}

int moe_combine(moe_shape s, const float* o, const int32_t* inv, const float* gate, void* y,
                void* stream) {
    int rc = check_shape(s);
    if (rc || s.T == 0) return rc;
    if (!ok_ptr(o) || !ok_ptr(inv) || !ok_ptr(gate) || !ok_ptr(y)) return MOE_ERR_INVALID_ARG;
    return launch_combine(s, o, inv, gate, y, static_cast<cudaStream_t>(stream));
}

int moe_forward(moe_shape s, const void* x, const void* Wg, const float* bias, const void* W1,
                const void* W3, const void* W2, void* y, int32_t* idx_out, float* gate_out,
                void* ws, size_t ws_bytes, void* stream) {
    int rc = check_shape(s);
    if (rc || s.T == 0) return rc;
    if (!ok_ptr(x) || !ok_ptr(Wg) || !ok_opt(bias) || !ok_ptr(W1) || !ok_ptr(W3) || !ok_ptr(W2) ||
        !ok_ptr(y) || !ok_opt(idx_out) || !ok_opt(gate_out) || !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_forward_workspace_bytes(s)) return MOE_ERR_WORKSPACE;
    return forward_impl(s, x, Wg, bias, W1, W3, W2, y, idx_out, gate_out, ws,
                        static_cast<cudaStream_t>(stream), nullptr);
}

int moe_forward_bias(moe_shape s, const void* x, const void* Wg, const float* bias,
                     const void* W1, const void* W3, const void* W2, const float* b1,
                     const float* b3, const float* b2, void* y, int32_t* idx_out,
                     float* gate_out, void* ws, size_t ws_bytes, void* stream) {
    int rc = check_shape(s);
    if (rc || s.T == 0) return rc;
    if (!ok_ptr(x) || !ok_ptr(Wg) || !ok_opt(bias) || !ok_ptr(W1) || !ok_ptr(W3) || !ok_ptr(W2) ||
        !ok_opt(b1) || !ok_opt(b3) || !ok_opt(b2) || !ok_ptr(y) || !ok_opt(idx_out) ||
        !ok_opt(gate_out) || !ok_ptr(ws))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_forward_workspace_bytes(s)) return MOE_ERR_WORKSPACE;
    FwdOptions opt;
    opt.eb.b1 = b1;
    opt.eb.b3 = b3;
    opt.eb.b2 = b2;
    return forward_impl(s, x, Wg, bias, W1, W3, W2, y, idx_out, gate_out, ws,
                        static_cast<cudaStream_t>(stream), nullptr, opt);
}

int moe_forward_profiled(moe_shape s, const void* x, const void* Wg, const float* bias,
                         const void* W1, const void* W3, const void* W2, void* y, void* ws,
                         size_t ws_bytes, void* const* events, int n_events, void* stream) {
    int rc = check_shape(s);
    if (rc || s.T == 0) return rc;
    if (!ok_ptr(x) || !ok_ptr(Wg) || !ok_opt(bias) || !ok_ptr(W1) || !ok_ptr(W3) || !ok_ptr(W2) ||
        !ok_ptr(y) || !ok_ptr(ws) || !events || n_events != kProfileEvents)
        return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < kProfileEvents; ++i)
        if (!events[i]) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_forward_workspace_bytes(s)) return MOE_ERR_WORKSPACE;
    return forward_impl(s, x, Wg, bias, W1, W3, W2, y, nullptr, nullptr, ws,
                        static_cast<cudaStream_t>(stream), events);
}

int moe_block_forward(moe_shape s, const void* U, const void* gamma, float eps, const void* Wg,
                      const float* bias, const void* W1, const void* W3, const void* W2, void* H,
                      void* ws, size_t ws_bytes, void* stream) {
    int rc = check_shape(s);
    if (rc || s.T == 0) return rc;
    if (!ok_ptr(U) || !ok_ptr(gamma) || !ok_ptr(Wg) || !ok_opt(bias) || !ok_ptr(W1) ||
        !ok_ptr(W3) || !ok_ptr(W2) || !ok_ptr(H) || !ok_ptr(ws) || !(eps >= 0.0f))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_block_workspace_bytes(s)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // RMSNorm_2 runs inside the router (which reads every row of U anyway) and
    // leaves u in the workspace for the scatter; the residual is added in the
    // combine.
    RouterNorm norm;
    norm.gamma = gamma;
    norm.eps = eps;
    norm.u = static_cast<char*>(ws) + moe_forward_workspace_bytes(s);
    FwdOptions opt;
    opt.residual = U;
    opt.norm = &norm;
    return forward_impl(s, U, Wg, bias, W1, W3, W2, H, nullptr, nullptr, ws, st, nullptr, opt);
}

int moe_forward_hostio(moe_shape s, const void* x_host, const void* Wg, const float* bias,
                       const void* W1, const void* W3, const void* W2, void* y_host, void* ws,
                       size_t ws_bytes, void* stream) {
    return hostio_impl(s, x_host, Wg, bias, W1, W3, W2, y_host, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream), -1, -1, kDefaultWaitTimeoutNs);
}

int moe_forward_hostio_batches(moe_shape s, int n_batches, const void* const* x_host,
                               const void* Wg, const float* bias, const void* W1,
                               const void* W3, const void* W2, void* const* y_host, void* ws,
                               size_t ws_bytes, void* stream) {
    return hostio_batches_impl(s, n_batches, x_host, Wg, bias, W1, W3, W2, y_host, ws, ws_bytes,
                               static_cast<cudaStream_t>(stream));
}

int moe_forward_hostio_batches_stall_test(moe_shape s, int n_batches,
                                          const void* const* x_host, const void* Wg,
                                          const float* bias, const void* W1, const void* W3,
                                          const void* W2, void* const* y_host, void* ws,
                                          size_t ws_bytes, int stall_batch, int stall_after,
                                          uint64_t timeout_ns, void* stream) {
    if (stall_batch < 0 || stall_after < 0) return MOE_ERR_INVALID_ARG;
    if (timeout_ns < 1000 || timeout_ns > kDefaultWaitTimeoutNs) return MOE_ERR_INVALID_ARG;
    return hostio_batches_impl(s, n_batches, x_host, Wg, bias, W1, W3, W2, y_host, ws, ws_bytes,
                               static_cast<cudaStream_t>(stream), stall_batch, stall_after,
                               timeout_ns);
}

int moe_forward_hostio_stall_test(moe_shape s, const void* x_host, const void* Wg,
                                  const float* bias, const void* W1, const void* W3,
                                  const void* W2, void* y_host, void* ws, size_t ws_bytes,
                                  int stall_chunk, int stall_after, uint64_t timeout_ns,
                                  void* stream) {
    if (stall_chunk < 0 || stall_after < 0) return MOE_ERR_INVALID_ARG;
    if (timeout_ns < 1000 || timeout_ns > kDefaultWaitTimeoutNs) return MOE_ERR_INVALID_ARG;
    return hostio_impl(s, x_host, Wg, bias, W1, W3, W2, y_host, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream), stall_chunk, stall_after, timeout_ns);
}

int moe_forward_static(moe_shape s, const void* x, const void* Wg, const float* bias,
                       const void* W1, const void* W3, const void* W2, void* y,
                       int32_t* device_status, void* stream) {
    int rc = check_shape(s);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (s.T == 0) {  // nothing to compute; the status word still reports "fine"
        if (!ok_opt(device_status)) return MOE_ERR_INVALID_ARG;
        if (device_status && cudaMemsetAsync(device_status, 0, sizeof(int32_t), st) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!ok_ptr(x) || !ok_ptr(Wg) || !ok_opt(bias) || !ok_ptr(W1) || !ok_ptr(W3) || !ok_ptr(W2) ||
        !ok_ptr(y) || !ok_opt(device_status))
        return MOE_ERR_INVALID_ARG;
    if (moe_forward_workspace_bytes(s) > kStaticScratchBytes) return MOE_ERR_WORKSPACE;
    void* ws = static_scratch_address();
    if (!ws) return MOE_ERR_CUDA;
    // forward_impl zeroes the status word (first word of the scratch) itself and
    // overwrites every other scratch byte it reads, so nothing else needs clearing.
    rc = forward_impl(s, x, Wg, bias, W1, W3, W2, y, nullptr, nullptr, ws, st, nullptr);
    if (rc) return rc;
    if (device_status &&
        cudaMemcpyAsync(device_status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) !=
            cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

int moe_aux_loss(moe_shape s, const float* logits, const int32_t* idx, const uint8_t* mask,
                 float* aux, float* f, float* P, void* stream) {
    // Only T, E and k matter here (T may count the rows of several layers).
    if (s.T < 0 || s.E < 1 || s.k < 1 || s.k > s.E) return MOE_ERR_INVALID_ARG;
    if (s.E > 32 || s.k > 8) return MOE_ERR_UNSUPPORTED;
    if (!ok_ptr(aux) || !ok_opt(f) || !ok_opt(P) || !ok_opt(mask)) return MOE_ERR_INVALID_ARG;
    if (s.T > 0 && (!ok_ptr(logits) || !ok_ptr(idx))) return MOE_ERR_INVALID_ARG;
    return launch_aux_loss(s, logits, idx, mask, aux, f, P, static_cast<cudaStream_t>(stream));
}

int moe_read_device_status(const void* ws, void* stream) {
    if (!ok_ptr(ws)) return MOE_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (word == 0) return MOE_OK;
    if (word & kDeviceTimeoutBase) return MOE_ERR_DEVICE_TIMEOUT;
    return MOE_ERR_CUDA;
}

}  // extern "C"
