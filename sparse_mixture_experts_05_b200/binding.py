"""Thin Python binding of the C ABI in include/moe.h (libmoe.so).

Argument marshalling only: every function here checks tensor devices, dtypes
and shapes, allocates missing outputs with torch, and calls the C entry point of
the same name on the current CUDA stream.  Every step of the layer runs in the
library's CUDA kernels; there is no fallback path.  If libmoe.so is missing the
first call raises ImportError.

Shapes follow the C header: `shape = (T, d, d_ff, E, k)`.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_TIMEOUT = 5

# Entry points declared in include/moe.h.
EXPORTS = (
    "moe_status_string", "moe_check_shape", "moe_expert_workspace_bytes",
    "moe_forward_workspace_bytes", "moe_forward_kernel_count", "moe_forward_hostio_workspace_bytes",
    "moe_route",
    "moe_dispatch", "moe_expert_swiglu", "moe_expert_swiglu_bias", "moe_expert_swiglu_stall_test",
    "moe_combine", "moe_forward", "moe_forward_bias", "moe_forward_profiled", "moe_forward_hostio", "moe_forward_hostio_stall_test",
    "moe_forward_hostio_batches_workspace_bytes", "moe_forward_hostio_batches",
    "moe_forward_hostio_batches_stall_test",
    "moe_forward_static",
    "moe_aux_loss", "moe_block_workspace_bytes", "moe_block_forward", "moe_read_device_status",
)

MOE_STATIC_SCRATCH_BYTES = 8 << 20


class MoeShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32)]


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libmoe.so (raises ImportError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m sparse_mixture_experts_05_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int
        S = MoeShape
        Z = ctypes.c_size_t
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [I]
        L.moe_check_shape.restype = I
        L.moe_check_shape.argtypes = [S]
        for fn in ("moe_expert_workspace_bytes", "moe_forward_workspace_bytes",
                   "moe_forward_hostio_workspace_bytes", "moe_block_workspace_bytes",
                   "moe_forward_hostio_batches_workspace_bytes"):
            getattr(L, fn).restype = Z
            getattr(L, fn).argtypes = [S]
        L.moe_forward_kernel_count.restype = I
        L.moe_forward_kernel_count.argtypes = [S]
        L.moe_route.restype = I
        L.moe_route.argtypes = [S, P, P, P, P, P, P, P]
        L.moe_dispatch.restype = I
        L.moe_dispatch.argtypes = [S, P, P, P, P, P, P, P]
        L.moe_expert_swiglu.restype = I
        L.moe_expert_swiglu.argtypes = [S, P, P, P, P, P, P, P, P, Z, P]
        L.moe_expert_swiglu_stall_test.restype = I
        L.moe_expert_swiglu_stall_test.argtypes = [S, P, P, P, P, P, P, P, P, Z, I,
                                                   ctypes.c_uint64, P]
        L.moe_combine.restype = I
        L.moe_expert_swiglu_bias.restype = I
        L.moe_expert_swiglu_bias.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, Z, P]
        L.moe_forward_bias.restype = I
        L.moe_forward_bias.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, P, Z, P]
        L.moe_combine.argtypes = [S, P, P, P, P, P]
        L.moe_forward.restype = I
        L.moe_forward.argtypes = [S, P, P, P, P, P, P, P, P, P, P, Z, P]
        L.moe_forward_profiled.restype = I
        L.moe_forward_profiled.argtypes = [S, P, P, P, P, P, P, P, P, Z, P, I, P]
        L.moe_forward_hostio.restype = I
        L.moe_forward_hostio.argtypes = [S, P, P, P, P, P, P, P, P, Z, P]
        L.moe_forward_hostio_batches.restype = I
        L.moe_forward_hostio_batches.argtypes = [S, I, P, P, P, P, P, P, P, P, Z, P]
        L.moe_forward_hostio_batches_stall_test.restype = I
        L.moe_forward_hostio_batches_stall_test.argtypes = [S, I, P, P, P, P, P, P, P, P, Z, I,
                                                            I, ctypes.c_uint64, P]
        L.moe_forward_hostio_stall_test.restype = I
        L.moe_forward_hostio_stall_test.argtypes = [S, P, P, P, P, P, P, P, P, Z, I, I,
                                                    ctypes.c_uint64, P]
        L.moe_forward_static.restype = I
        L.moe_forward_static.argtypes = [S, P, P, P, P, P, P, P, P, P]
        L.moe_block_forward.restype = I
        L.moe_block_forward.argtypes = [S, P, P, ctypes.c_float, P, P, P, P, P, P, P, Z, P]
        L.moe_aux_loss.restype = I
        L.moe_aux_loss.argtypes = [S, P, P, P, P, P, P, P]
        L.moe_read_device_status.restype = I
        L.moe_read_device_status.argtypes = [P, P]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def _shape(shape) -> MoeShape:
    T, d, d_ff, E, k = (int(v) for v in shape)
    return MoeShape(T, d, d_ff, E, k)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, rc: int):
    if rc != MOE_OK:
        raise MoeError(fn, rc)


def _dev(t: torch.Tensor, name: str, dtype, shape=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _new(shape, dtype, like):
    return torch.empty(shape, dtype=dtype, device=like.device)


def moe_check_shape(shape) -> int:
    return lib().moe_check_shape(_shape(shape))


def moe_expert_workspace_bytes(shape) -> int:
    return lib().moe_expert_workspace_bytes(_shape(shape))


def moe_forward_workspace_bytes(shape) -> int:
    return lib().moe_forward_workspace_bytes(_shape(shape))


def moe_forward_kernel_count(shape) -> int:
    """Kernels one moe_forward of `shape` launches on the current device (5 or 6; 0 for
    T == 0); MoeError for a shape moe_forward rejects."""
    n = lib().moe_forward_kernel_count(_shape(shape))
    if n < 0:
        _check("moe_forward_kernel_count", -n)
    return n


def moe_forward_hostio_workspace_bytes(shape) -> int:
    return lib().moe_forward_hostio_workspace_bytes(_shape(shape))


def workspace(nbytes: int, device) -> torch.Tensor:
    """Device workspace of `nbytes` bytes (256-byte aligned by the caching allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def moe_route(shape, x, Wg, bias=None, idx=None, gate=None, logits=None, want_logits=False,
              stream=None):
    T, d, d_ff, E, k = shape
    _dev(x, "x", torch.bfloat16, (T, d))
    _dev(Wg, "Wg", torch.bfloat16, (d, E))
    _dev(bias, "bias", torch.float32, (E,))
    idx = _new((T, k), torch.int32, x) if idx is None else idx
    gate = _new((T, k), torch.float32, x) if gate is None else gate
    if logits is None and want_logits:
        logits = _new((T, E), torch.float32, x)
    _dev(idx, "idx", torch.int32, (T, k))
    _dev(gate, "gate", torch.float32, (T, k))
    _dev(logits, "logits", torch.float32, (T, E))
    _check("moe_route", lib().moe_route(_shape(shape), _p(x), _p(Wg), _p(bias), _p(idx), _p(gate),
                                        _p(logits), _stream(stream)))
    return idx, gate, logits


def moe_dispatch(shape, idx, x, offsets=None, perm_tok=None, inv=None, x_sorted=None,
                 stream=None):
    T, d, d_ff, E, k = shape
    _dev(idx, "idx", torch.int32, (T, k))
    _dev(x, "x", torch.bfloat16, (T, d))
    offsets = _new((E + 1,), torch.int32, x) if offsets is None else offsets
    perm_tok = _new((T * k,), torch.int32, x) if perm_tok is None else perm_tok
    inv = _new((T, k), torch.int32, x) if inv is None else inv
    x_sorted = _new((T * k, d), torch.bfloat16, x) if x_sorted is None else x_sorted
    _dev(offsets, "offsets", torch.int32, (E + 1,))
    _dev(perm_tok, "perm_tok", torch.int32, (T * k,))
    _dev(inv, "inv", torch.int32, (T, k))
    _dev(x_sorted, "x_sorted", torch.bfloat16, (T * k, d))
    _check("moe_dispatch", lib().moe_dispatch(_shape(shape), _p(idx), _p(x), _p(offsets),
                                              _p(perm_tok), _p(inv), _p(x_sorted),
                                              _stream(stream)))
    return offsets, perm_tok, inv, x_sorted


def _expert_args(shape, x_sorted, offsets, W1, W3, W2, h, o, ws):
    T, d, d_ff, E, k = shape
    R = T * k
    _dev(x_sorted, "x_sorted", torch.bfloat16, (R, d))
    _dev(offsets, "offsets", torch.int32, (E + 1,))
    _dev(W1, "W1", torch.bfloat16, (E, d, d_ff))
    _dev(W3, "W3", torch.bfloat16, (E, d, d_ff))
    _dev(W2, "W2", torch.bfloat16, (E, d_ff, d))
    h = _new((R, d_ff), torch.bfloat16, x_sorted) if h is None else h
    o = _new((R, d), torch.float32, x_sorted) if o is None else o
    ws = workspace(moe_expert_workspace_bytes(shape), x_sorted.device) if ws is None else ws
    _dev(h, "h", torch.bfloat16, (R, d_ff))
    _dev(o, "o", torch.float32, (R, d))
    _dev(ws, "ws", torch.uint8)
    return h, o, ws


def moe_expert_swiglu(shape, x_sorted, offsets, W1, W3, W2, h=None, o=None, ws=None,
                      stream=None):
    h, o, ws = _expert_args(shape, x_sorted, offsets, W1, W3, W2, h, o, ws)
    _check("moe_expert_swiglu",
           lib().moe_expert_swiglu(_shape(shape), _p(x_sorted), _p(offsets), _p(W1), _p(W3),
                                   _p(W2), _p(h), _p(o), _p(ws), ws.numel(), _stream(stream)))
    return h, o, ws


def _expert_bias_args(shape, expert_bias):
    """(b1, b3, b2) float32 device tensors [E,d_ff], [E,d_ff], [E,d], each may be None."""
    T, d, d_ff, E, k = shape
    if expert_bias is None:
        return None, None, None
    b1, b3, b2 = expert_bias
    _dev(b1, "b1", torch.float32, (E, d_ff))
    _dev(b3, "b3", torch.float32, (E, d_ff))
    _dev(b2, "b2", torch.float32, (E, d))
    return b1, b3, b2


def moe_expert_swiglu_bias(shape, x_sorted, offsets, W1, W3, W2, expert_bias, h=None, o=None,
                           ws=None, stream=None):
    """moe_expert_swiglu with the expert Linear biases expert_bias = (b1, b3, b2)."""
    h, o, ws = _expert_args(shape, x_sorted, offsets, W1, W3, W2, h, o, ws)
    b1, b3, b2 = _expert_bias_args(shape, expert_bias)
    _check("moe_expert_swiglu_bias",
           lib().moe_expert_swiglu_bias(_shape(shape), _p(x_sorted), _p(offsets), _p(W1), _p(W3),
                                        _p(W2), _p(b1), _p(b3), _p(b2), _p(h), _p(o), _p(ws),
                                        ws.numel(), _stream(stream)))
    return h, o, ws


def moe_expert_swiglu_stall_test(shape, x_sorted, offsets, W1, W3, W2, stall_after: int,
                                 timeout_ns: int, h=None, o=None, ws=None, stream=None):
    h, o, ws = _expert_args(shape, x_sorted, offsets, W1, W3, W2, h, o, ws)
    _check("moe_expert_swiglu_stall_test",
           lib().moe_expert_swiglu_stall_test(_shape(shape), _p(x_sorted), _p(offsets), _p(W1),
                                              _p(W3), _p(W2), _p(h), _p(o), _p(ws), ws.numel(),
                                              int(stall_after), int(timeout_ns),
                                              _stream(stream)))
    return h, o, ws


def moe_combine(shape, o, inv, gate, y=None, stream=None):
    T, d, d_ff, E, k = shape
    _dev(o, "o", torch.float32, (T * k, d))
    _dev(inv, "inv", torch.int32, (T, k))
    _dev(gate, "gate", torch.float32, (T, k))
    y = _new((T, d), torch.bfloat16, o) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, d))
    _check("moe_combine", lib().moe_combine(_shape(shape), _p(o), _p(inv), _p(gate), _p(y),
                                            _stream(stream)))
    return y


def moe_forward(shape, x, Wg, bias, W1, W3, W2, y=None, idx_out=None, gate_out=None, ws=None,
                stream=None):
    T, d, d_ff, E, k = shape
    _dev(x, "x", torch.bfloat16, (T, d))
    _dev(Wg, "Wg", torch.bfloat16, (d, E))
    _dev(bias, "bias", torch.float32, (E,))
    _dev(W1, "W1", torch.bfloat16, (E, d, d_ff))
    _dev(W3, "W3", torch.bfloat16, (E, d, d_ff))
    _dev(W2, "W2", torch.bfloat16, (E, d_ff, d))
    y = _new((T, d), torch.bfloat16, x) if y is None else y
    ws = workspace(moe_forward_workspace_bytes(shape), x.device) if ws is None else ws
    _dev(y, "y", torch.bfloat16, (T, d))
    _dev(idx_out, "idx_out", torch.int32, (T, k))
    _dev(gate_out, "gate_out", torch.float32, (T, k))
    _dev(ws, "ws", torch.uint8)
    _check("moe_forward", lib().moe_forward(_shape(shape), _p(x), _p(Wg), _p(bias), _p(W1), _p(W3),
                                            _p(W2), _p(y), _p(idx_out), _p(gate_out), _p(ws),
                                            ws.numel(), _stream(stream)))
    return y


def moe_forward_bias(shape, x, Wg, bias, W1, W3, W2, expert_bias, y=None, idx_out=None,
                     gate_out=None, ws=None, stream=None):
    """moe_forward with the expert Linear biases expert_bias = (b1, b3, b2)."""
    T, d, d_ff, E, k = shape
    _dev(x, "x", torch.bfloat16, (T, d))
    _dev(Wg, "Wg", torch.bfloat16, (d, E))
    _dev(bias, "bias", torch.float32, (E,))
    _dev(W1, "W1", torch.bfloat16, (E, d, d_ff))
    _dev(W3, "W3", torch.bfloat16, (E, d, d_ff))
    _dev(W2, "W2", torch.bfloat16, (E, d_ff, d))
    b1, b3, b2 = _expert_bias_args(shape, expert_bias)
    y = _new((T, d), torch.bfloat16, x) if y is None else y
    ws = workspace(moe_forward_workspace_bytes(shape), x.device) if ws is None else ws
    _dev(y, "y", torch.bfloat16, (T, d))
    _dev(idx_out, "idx_out", torch.int32, (T, k))
    _dev(gate_out, "gate_out", torch.float32, (T, k))
    _dev(ws, "ws", torch.uint8)
    _check("moe_forward_bias",
           lib().moe_forward_bias(_shape(shape), _p(x), _p(Wg), _p(bias), _p(W1), _p(W3), _p(W2),
                                  _p(b1), _p(b3), _p(b2), _p(y), _p(idx_out), _p(gate_out),
                                  _p(ws), ws.numel(), _stream(stream)))
    return y


PROFILE_EVENTS = ("start", "router", "dispatch_index", "dispatch_scatter", "gemm1_swiglu",
                  "gemm2_down", "combine")


def moe_forward_profiled(shape, x, Wg, bias, W1, W3, W2, events, y=None, ws=None, stream=None):
    """moe_forward that records the 7 torch.cuda.Event objects in `events` between its
    launches (see PROFILE_EVENTS); the events must have been recorded once already so
    that their CUDA handles exist."""
    T, d, d_ff, E, k = shape
    _dev(x, "x", torch.bfloat16, (T, d))
    _dev(Wg, "Wg", torch.bfloat16, (d, E))
    _dev(bias, "bias", torch.float32, (E,))
    _dev(W1, "W1", torch.bfloat16, (E, d, d_ff))
    _dev(W3, "W3", torch.bfloat16, (E, d, d_ff))
    _dev(W2, "W2", torch.bfloat16, (E, d_ff, d))
    y = _new((T, d), torch.bfloat16, x) if y is None else y
    ws = workspace(moe_forward_workspace_bytes(shape), x.device) if ws is None else ws
    _dev(y, "y", torch.bfloat16, (T, d))
    _dev(ws, "ws", torch.uint8)
    if len(events) != len(PROFILE_EVENTS):
        raise ValueError(f"need {len(PROFILE_EVENTS)} events")
    handles = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    _check("moe_forward_profiled",
           lib().moe_forward_profiled(_shape(shape), _p(x), _p(Wg), _p(bias), _p(W1), _p(W3),
                                      _p(W2), _p(y), _p(ws), ws.numel(), handles, len(events),
                                      _stream(stream)))
    return y


def moe_forward_hostio(shape, x_host, Wg, bias, W1, W3, W2, y_host, ws, stream=None):
    """x_host / y_host: CPU bf16 tensors (pinned for asynchronous copies)."""
    T, d, d_ff, E, k = shape
    for name, t in (("x_host", x_host), ("y_host", y_host)):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() \
                or tuple(t.shape) != (T, d):
            raise ValueError(f"{name} must be a contiguous CPU bf16 tensor of shape {(T, d)}")
    _dev(Wg, "Wg", torch.bfloat16, (d, E))
    _dev(bias, "bias", torch.float32, (E,))
    _dev(W1, "W1", torch.bfloat16, (E, d, d_ff))
    _dev(W3, "W3", torch.bfloat16, (E, d, d_ff))
    _dev(W2, "W2", torch.bfloat16, (E, d_ff, d))
    _dev(ws, "ws", torch.uint8)
    _check("moe_forward_hostio",
           lib().moe_forward_hostio(_shape(shape), _p(x_host), _p(Wg), _p(bias), _p(W1), _p(W3),
                                    _p(W2), _p(y_host), _p(ws), ws.numel(), _stream(stream)))
    return y_host


def moe_forward_hostio_batches_workspace_bytes(shape) -> int:
    return lib().moe_forward_hostio_batches_workspace_bytes(_shape(shape))


def moe_forward_hostio_batches(shape, xs_host, Wg, bias, W1, W3, W2, ys_host, ws, stream=None):
    """xs_host / ys_host: equal-length sequences of CPU bf16 tensors of shape (T, d)
    (pinned for asynchronous copies); batch b reads xs_host[b] and writes ys_host[b]."""
    T, d, d_ff, E, k = shape
    if len(xs_host) != len(ys_host) or len(xs_host) < 1:
        raise ValueError("xs_host and ys_host must be non-empty and of equal length")
    for name, seq in (("xs_host", xs_host), ("ys_host", ys_host)):
        for t in seq:
            if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() \
                    or tuple(t.shape) != (T, d):
                raise ValueError(f"every {name} entry must be a contiguous CPU bf16 tensor "
                                 f"of shape {(T, d)}")
    _dev(Wg, "Wg", torch.bfloat16, (d, E))
    _dev(bias, "bias", torch.float32, (E,))
    _dev(W1, "W1", torch.bfloat16, (E, d, d_ff))
    _dev(W3, "W3", torch.bfloat16, (E, d, d_ff))
    _dev(W2, "W2", torch.bfloat16, (E, d_ff, d))
    _dev(ws, "ws", torch.uint8)
    n = len(xs_host)
    xp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in xs_host])
    yp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in ys_host])
    _check("moe_forward_hostio_batches",
           lib().moe_forward_hostio_batches(_shape(shape), n, ctypes.cast(xp, ctypes.c_void_p),
                                            _p(Wg), _p(bias), _p(W1), _p(W3), _p(W2),
                                            ctypes.cast(yp, ctypes.c_void_p), _p(ws), ws.numel(),
                                            _stream(stream)))
    return ys_host


def _host_batches(shape, xs_host, ys_host):
    T, d, d_ff, E, k = shape
    if len(xs_host) != len(ys_host) or len(xs_host) < 1:
        raise ValueError("xs_host and ys_host must be non-empty and of equal length")
    for name, seq in (("xs_host", xs_host), ("ys_host", ys_host)):
        for t in seq:
            if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() \
                    or tuple(t.shape) != (T, d):
                raise ValueError(f"every {name} entry must be a contiguous CPU bf16 tensor "
                                 f"of shape {(T, d)}")
    n = len(xs_host)
    xp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in xs_host])
    yp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in ys_host])
    return n, xp, yp


def moe_forward_hostio_batches_stall_test(shape, xs_host, Wg, bias, W1, W3, W2, ys_host, ws,
                                          stall_batch: int, stall_after: int, timeout_ns: int,
                                          stream=None):
    """moe_forward_hostio_batches with the expert producer of batch `stall_batch`
    stopping after `stall_after` stages and that batch's waits bounded by
    `timeout_ns` (test of the error path of the queue)."""
    T, d, d_ff, E, k = shape
    n, xp, yp = _host_batches(shape, xs_host, ys_host)
    _dev(Wg, "Wg", torch.bfloat16, (d, E))
    _dev(bias, "bias", torch.float32, (E,))
    _dev(W1, "W1", torch.bfloat16, (E, d, d_ff))
    _dev(W3, "W3", torch.bfloat16, (E, d, d_ff))
    _dev(W2, "W2", torch.bfloat16, (E, d_ff, d))
    _dev(ws, "ws", torch.uint8)
    _check("moe_forward_hostio_batches_stall_test",
           lib().moe_forward_hostio_batches_stall_test(
               _shape(shape), n, ctypes.cast(xp, ctypes.c_void_p), _p(Wg), _p(bias), _p(W1),
               _p(W3), _p(W2), ctypes.cast(yp, ctypes.c_void_p), _p(ws), ws.numel(),
               int(stall_batch), int(stall_after), int(timeout_ns), _stream(stream)))
    return ys_host


def moe_forward_hostio_stall_test(shape, x_host, Wg, bias, W1, W3, W2, y_host, ws,
                                  stall_chunk: int, stall_after: int, timeout_ns: int,
                                  stream=None):
    """moe_forward_hostio with the expert producer of token chunk `stall_chunk`
    stopping after `stall_after` stages and that chunk's waits bounded by
    `timeout_ns` (test of the error path of the chunked pipeline)."""
    T, d, d_ff, E, k = shape
    for name, t in (("x_host", x_host), ("y_host", y_host)):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() \
                or tuple(t.shape) != (T, d):
            raise ValueError(f"{name} must be a contiguous CPU bf16 tensor of shape {(T, d)}")
    _dev(Wg, "Wg", torch.bfloat16, (d, E))
    _dev(bias, "bias", torch.float32, (E,))
    _dev(W1, "W1", torch.bfloat16, (E, d, d_ff))
    _dev(W3, "W3", torch.bfloat16, (E, d, d_ff))
    _dev(W2, "W2", torch.bfloat16, (E, d_ff, d))
    _dev(ws, "ws", torch.uint8)
    _check("moe_forward_hostio_stall_test",
           lib().moe_forward_hostio_stall_test(_shape(shape), _p(x_host), _p(Wg), _p(bias), _p(W1),
                                               _p(W3), _p(W2), _p(y_host), _p(ws), ws.numel(),
                                               int(stall_chunk), int(stall_after),
                                               int(timeout_ns), _stream(stream)))
    return y_host


def moe_forward_static(shape, x, Wg, bias, W1, W3, W2, y=None, device_status=None, stream=None):
    """moe_forward without a workspace argument: the library's fixed 8 MiB device
    scratch array stands in for it (for callers that cannot allocate device memory).
    `device_status`: optional CUDA int32 tensor of one element that receives the
    call's status word."""
    T, d, d_ff, E, k = shape
    _dev(x, "x", torch.bfloat16, (T, d))
    _dev(Wg, "Wg", torch.bfloat16, (d, E))
    _dev(bias, "bias", torch.float32, (E,))
    _dev(W1, "W1", torch.bfloat16, (E, d, d_ff))
    _dev(W3, "W3", torch.bfloat16, (E, d, d_ff))
    _dev(W2, "W2", torch.bfloat16, (E, d_ff, d))
    y = _new((T, d), torch.bfloat16, x) if y is None else y
    _dev(y, "y", torch.bfloat16, (T, d))
    _dev(device_status, "device_status", torch.int32, (1,))
    _check("moe_forward_static",
           lib().moe_forward_static(_shape(shape), _p(x), _p(Wg), _p(bias), _p(W1), _p(W3),
                                    _p(W2), _p(y), _p(device_status), _stream(stream)))
    return y


def moe_block_workspace_bytes(shape) -> int:
    return lib().moe_block_workspace_bytes(_shape(shape))


def moe_block_forward(shape, U, gamma, Wg, bias, W1, W3, W2, eps=1e-5, H=None, ws=None,
                      stream=None):
    """H = U + MoE(RMSNorm(U)) through moe_block_forward."""
    T, d, d_ff, E, k = shape
    _dev(U, "U", torch.bfloat16, (T, d))
    _dev(gamma, "gamma", torch.bfloat16, (d,))
    _dev(Wg, "Wg", torch.bfloat16, (d, E))
    _dev(bias, "bias", torch.float32, (E,))
    _dev(W1, "W1", torch.bfloat16, (E, d, d_ff))
    _dev(W3, "W3", torch.bfloat16, (E, d, d_ff))
    _dev(W2, "W2", torch.bfloat16, (E, d_ff, d))
    H = _new((T, d), torch.bfloat16, U) if H is None else H
    ws = workspace(moe_block_workspace_bytes(shape), U.device) if ws is None else ws
    _dev(H, "H", torch.bfloat16, (T, d))
    _dev(ws, "ws", torch.uint8)
    _check("moe_block_forward",
           lib().moe_block_forward(_shape(shape), _p(U), _p(gamma), float(eps), _p(Wg), _p(bias),
                                   _p(W1), _p(W3), _p(W2), _p(H), _p(ws), ws.numel(),
                                   _stream(stream)))
    return H


def moe_aux_loss(shape, logits, idx, mask=None, want_stats=False, stream=None):
    """Load-balancing term E * sum_s sum_i f_{s,i} P_i.  Returns (aux [1], f [k,E] or None,
    P [E] or None) as CUDA float32 tensors.  shape's T is the number of rows of logits."""
    T, d, d_ff, E, k = shape
    _dev(logits, "logits", torch.float32, (T, E))
    _dev(idx, "idx", torch.int32, (T, k))
    _dev(mask, "mask", torch.uint8, (T,))
    aux = _new((1,), torch.float32, logits)
    f = _new((k, E), torch.float32, logits) if want_stats else None
    P = _new((E,), torch.float32, logits) if want_stats else None
    _check("moe_aux_loss", lib().moe_aux_loss(_shape(shape), _p(logits), _p(idx), _p(mask), _p(aux),
                                              _p(f), _p(P), _stream(stream)))
    return aux, f, P


def moe_read_device_status(ws, stream=None) -> int:
    """Synchronises the stream and returns the status word of `ws` (MOE_OK or an error code)."""
    return lib().moe_read_device_status(_p(ws), _stream(stream))
