"""CPU oracle for the Mixtral sparse-MoE layer (ctypes wrapper around moe_oracle.c).

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers; the product package never imports this
module and shares no code with it.

Every routine follows the Mixtral textbook page (llm-arch-research), section
"Прямой проход в формулах" (the MoE equation) and section "Алгоритм" (the loop
over experts, gathering each expert's tokens and accumulating the gate-weighted
outputs back per token); the C source cites the passage per routine.

Arrays are numpy: bf16 tensors travel as uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so (plain gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O3", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        lib.orc_bf16_value.restype = ctypes.c_double
        lib.orc_bf16_value.argtypes = [ctypes.c_uint16]
        lib.orc_round_bf16.restype = ctypes.c_double
        lib.orc_round_bf16.argtypes = [ctypes.c_double]
        lib.orc_bf16_bits.restype = ctypes.c_uint16
        lib.orc_bf16_bits.argtypes = [ctypes.c_double]
        lib.orc_round_bf16_array.restype = None
        lib.orc_round_bf16_array.argtypes = [I64, P, P]
        lib.orc_silu.restype = ctypes.c_double
        lib.orc_silu.argtypes = [ctypes.c_double]
        lib.orc_route.restype = I
        lib.orc_route.argtypes = [I, I, I, I, P, P, P, P, P, P]
        lib.orc_dispatch.restype = I
        lib.orc_dispatch.argtypes = [I, I, I, P, P, P, P]
        lib.orc_gather.restype = None
        lib.orc_gather.argtypes = [I, I, P, P, P]
        lib.orc_expert.restype = I
        lib.orc_expert.argtypes = [I, I, I, I, P, P, P, P, P, I, P, P]
        lib.orc_expert_bias.restype = I
        lib.orc_expert_bias.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P, I, P, P]
        lib.orc_combine.restype = None
        lib.orc_combine.argtypes = [I, I, I, P, P, P, P]
        lib.orc_forward.restype = I
        lib.orc_forward.argtypes = [I, I, I, I, I, P, P, P, P, P, P, I, P, P, P]
        lib.orc_forward_tokens.restype = I
        lib.orc_forward_tokens.argtypes = [I, P, I, I, I, I, I, P, P, P, P, P, P, I, P, P, P]
        lib.orc_forward_bias.restype = I
        lib.orc_forward_bias.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P, P, I, P, P, P]
        lib.orc_forward_tokens_bias.restype = I
        lib.orc_forward_tokens_bias.argtypes = [I, P, I, I, I, I, I, P, P, P, P, P, P, P, P, P, I,
                                                P, P, P]
        lib.orc_rmsnorm.restype = None
        lib.orc_rmsnorm.argtypes = [I, I, P, P, ctypes.c_double, P]
        lib.orc_block_forward.restype = I
        lib.orc_block_forward.argtypes = [I, I, I, I, I, P, P, ctypes.c_double, P, P, P, P, P, I,
                                          P, P, P]
        lib.orc_aux_loss.restype = ctypes.c_double
        lib.orc_aux_loss.argtypes = [I, I, I, P, P, P, P, P]
        lib.orc_param_count.restype = None
        lib.orc_param_count.argtypes = [I64] * 9 + [I, P, P]
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _u16(a):
    """bf16 data as a C-contiguous uint16 array (accepts torch bf16 tensors or uint16 arrays)."""
    if hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        a = a.contiguous().view(dtype=__import__("torch").int16).numpy().view(np.uint16)
    return np.ascontiguousarray(a, dtype=np.uint16)


def bf16_to_f64(bits) -> np.ndarray:
    """Values of bf16 bit patterns (uint16) as float64."""
    b = _u16(bits)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(v) -> np.ndarray:
    """Round float64 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().orc_round_bf16_array(v.size, _p(v), _p(out))
    return out


def round_bf16_scalar(v: float) -> float:
    return _load().orc_round_bf16(float(v))


def silu(a: float) -> float:
    return _load().orc_silu(float(a))


def route(x, wg, E: int, k: int, bias=None):
    """Router + top-k + softmax.  Returns (idx int32 [T,k], gate float32 [T,k], logits float32 [T,E])."""
    x = _u16(x)
    wg = _u16(wg)
    T, d = x.shape
    assert wg.shape == (d, E)
    idx = np.empty((T, k), np.int32)
    gate = np.empty((T, k), np.float32)
    logits = np.empty((T, E), np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    rc = _load().orc_route(T, d, E, k, _p(x), _p(wg), _p(b), _p(idx), _p(gate), _p(logits))
    if rc:
        raise ValueError(f"orc_route rejected the arguments (rc={rc})")
    return idx, gate, logits


def dispatch(idx, E: int):
    """Per-expert token lists.  Returns (offsets [E+1], perm_tok [T*k], inv [T,k]), all int32."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty((T, k), np.int32)
    rc = _load().orc_dispatch(T, E, k, _p(idx), _p(offsets), _p(perm), _p(inv))
    if rc:
        raise ValueError(f"orc_dispatch rejected the arguments (rc={rc})")
    return offsets, perm, inv


def gather(x, perm_tok):
    x = _u16(x)
    perm_tok = np.ascontiguousarray(perm_tok, dtype=np.int32)
    R = perm_tok.shape[0]
    d = x.shape[1]
    out = np.empty((R, d), np.uint16)
    _load().orc_gather(R, d, _p(perm_tok), _p(x), _p(out))
    return out


def _expert_bias(expert_bias, E: int, d: int, d_ff: int):
    """(b1 [E,d_ff], b3 [E,d_ff], b2 [E,d]) as float32 arrays, or three Nones."""
    if expert_bias is None:
        return None, None, None
    b1, b3, b2 = (np.ascontiguousarray(b, dtype=np.float32) for b in expert_bias)
    assert b1.shape == (E, d_ff) and b3.shape == (E, d_ff) and b2.shape == (E, d)
    return b1, b3, b2


def expert(x_sorted, offsets, W1, W3, W2, round_h: bool = True, expert_bias=None):
    """SwiGLU experts over sorted rows.  Returns (h [R,d_ff], o [R,d]) as float64 values
    (h rounded to bf16 values when round_h; o never rounded).  expert_bias =
    (b1, b3, b2) adds the biases of the three Linear layers."""
    xs = _u16(x_sorted)
    W1 = _u16(W1)
    W3 = _u16(W3)
    W2 = _u16(W2)
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    R, d = xs.shape
    E, d1, d_ff = W1.shape
    assert d1 == d and W3.shape == W1.shape and W2.shape == (E, d_ff, d)
    b1, b3, b2 = _expert_bias(expert_bias, E, d, d_ff)
    h = np.empty((R, d_ff), np.float64)
    o = np.empty((R, d), np.float64)
    rc = _load().orc_expert_bias(R, d, d_ff, E, _p(offsets), _p(xs), _p(W1), _p(W3), _p(W2),
                                 _p(b1), _p(b3), _p(b2), int(round_h), _p(h), _p(o))
    if rc:
        raise ValueError(f"orc_expert failed (rc={rc})")
    return h, o


def combine(o, inv, gate):
    o = np.ascontiguousarray(o, dtype=np.float64)
    inv = np.ascontiguousarray(inv, dtype=np.int32)
    gate = np.ascontiguousarray(gate, dtype=np.float32)
    T, k = inv.shape
    d = o.shape[1]
    y = np.empty((T, d), np.float64)
    _load().orc_combine(T, d, k, _p(o), _p(inv), _p(gate), _p(y))
    return y


def forward(x, wg, W1, W3, W2, k: int, bias=None, round_h: bool = True, expert_bias=None):
    """Whole layer, expert-major.  Returns (y float64 [T,d] unrounded, idx [T,k], gate [T,k]).
    bias: router bias [E]; expert_bias: (b1, b3, b2) of the expert Linear layers."""
    x = _u16(x)
    wg = _u16(wg)
    W1 = _u16(W1)
    W3 = _u16(W3)
    W2 = _u16(W2)
    T, d = x.shape
    E, _, d_ff = W1.shape
    y = np.empty((T, d), np.float64)
    idx = np.empty((T, k), np.int32)
    gate = np.empty((T, k), np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    b1, b3, b2 = _expert_bias(expert_bias, E, d, d_ff)
    rc = _load().orc_forward_bias(T, d, d_ff, E, k, _p(x), _p(wg), _p(b), _p(W1), _p(W3), _p(W2),
                                  _p(b1), _p(b3), _p(b2), int(round_h), _p(y), _p(idx), _p(gate))
    if rc:
        raise ValueError(f"orc_forward failed (rc={rc})")
    return y, idx, gate


def forward_tokens(tokens, x, wg, W1, W3, W2, k: int, bias=None, round_h: bool = True,
                   expert_bias=None):
    """Naive per-token loop for the listed tokens.  Returns (y [n,d], idx [n,k], gate [n,k])."""
    toks = np.ascontiguousarray(tokens, dtype=np.int32)
    x = _u16(x)
    wg = _u16(wg)
    W1 = _u16(W1)
    W3 = _u16(W3)
    W2 = _u16(W2)
    T, d = x.shape
    E, _, d_ff = W1.shape
    n = toks.shape[0]
    y = np.empty((n, d), np.float64)
    idx = np.empty((n, k), np.int32)
    gate = np.empty((n, k), np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    b1, b3, b2 = _expert_bias(expert_bias, E, d, d_ff)
    rc = _load().orc_forward_tokens_bias(n, _p(toks), T, d, d_ff, E, k, _p(x), _p(wg), _p(b),
                                         _p(W1), _p(W3), _p(W2), _p(b1), _p(b3), _p(b2),
                                         int(round_h), _p(y), _p(idx), _p(gate))
    if rc:
        raise ValueError(f"orc_forward_tokens failed (rc={rc})")
    return y, idx, gate


def rmsnorm(U, gamma, eps: float = 1e-5):
    """bf16(U / sqrt(mean(U^2) + eps) * gamma) row by row; returns uint16 bit patterns."""
    U = _u16(U)
    gamma = _u16(gamma)
    T, d = U.shape
    u = np.empty((T, d), np.uint16)
    _load().orc_rmsnorm(T, d, _p(U), _p(gamma), float(eps), _p(u))
    return u


def block_forward(U, gamma, wg, W1, W3, W2, k: int, eps: float = 1e-5, bias=None,
                  round_h: bool = True):
    """H = U + MoE(RMSNorm(U)) (float64, unrounded).  Returns (H, idx, gate)."""
    U = _u16(U)
    gamma = _u16(gamma)
    wg = _u16(wg)
    W1 = _u16(W1)
    W3 = _u16(W3)
    W2 = _u16(W2)
    T, d = U.shape
    E, _, d_ff = W1.shape
    H = np.empty((T, d), np.float64)
    idx = np.empty((T, k), np.int32)
    gate = np.empty((T, k), np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    rc = _load().orc_block_forward(T, d, d_ff, E, k, _p(U), _p(gamma), float(eps), _p(wg), _p(b),
                                   _p(W1), _p(W3), _p(W2), int(round_h), _p(H), _p(idx), _p(gate))
    if rc:
        raise ValueError(f"orc_block_forward failed (rc={rc})")
    return H, idx, gate


def aux_loss(logits, idx, mask=None):
    """Load-balancing auxiliary term E * sum_s sum_i f_{s,i} P_i.  Returns (aux, f [k,E], P [E])."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, E = logits.shape
    k = idx.shape[1]
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    f = np.empty((k, E), np.float64)
    P = np.empty(E, np.float64)
    aux = _load().orc_aux_loss(T, E, k, _p(logits), _p(idx), _p(m), _p(f), _p(P))
    return aux, f, P


def param_count(V, d, L, H, G, dh, d_ff, E, k, bias=False):
    """(total, active) parameter counts of a Mixtral-style model."""
    tot = ctypes.c_int64()
    act = ctypes.c_int64()
    _load().orc_param_count(V, d, L, H, G, dh, d_ff, E, k, int(bias), ctypes.byref(tot),
                            ctypes.byref(act))
    return tot.value, act.value


def near_tie_flags(logits, k: int, eps: float = 1e-4):
    """Per token: (k-th vs (k+1)-th logit gap < eps, 1st vs 2nd gap < eps).

    Tokens flagged in the first array may be routed either way by a correct
    implementation whose float32 logits differ in the last bits."""
    srt = -np.sort(-np.asarray(logits, dtype=np.float64), axis=1)
    E = srt.shape[1]
    if k < E:
        kth = (srt[:, k - 1] - srt[:, k]) < eps
    else:
        kth = np.zeros(srt.shape[0], bool)
    first = (srt[:, 0] - srt[:, 1]) < eps if E > 1 else np.zeros(srt.shape[0], bool)
    return kth, first
