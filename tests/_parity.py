"""Comparison rules between the CUDA path and the CPU oracle.

Acceptance (the layer's contract):
  * expert indices bit-exact, except tokens whose k-th and (k+1)-th oracle
    logits lie within 1e-4 (either routing is correct; those tokens are
    counted, and the GPU's choice must still be among the experts within 1e-4
    of the oracle's k-th logit);
  * gates within 1e-5 absolute;
  * y: max |y - y_ref| <= 2e-2 * rms(y_ref) over the other tokens, and near-tie
    tokens re-checked with the GPU's routing forced into the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

NEAR_TIE = 1e-4
GATE_TOL = 1e-5
Y_TOL = 2e-2


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_values(t: torch.Tensor) -> np.ndarray:
    return oracle.bf16_to_f64(u16(t))


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |v| (normal range; subnormal spacing below 2^-126)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def to_dev(inp: dict, device="cuda") -> dict:
    out = dict(inp)
    for key in ("x", "Wg", "W1", "W3", "W2", "bias"):
        if inp.get(key) is not None:
            out[key] = inp[key].to(device)
    return out


def check_routing(g_idx, g_gate, o_idx, o_gate, o_logits, k):
    """Returns (mask of tokens held to the bit-exact rule, stats).  Asserts the rules."""
    g_idx = np.asarray(g_idx)
    g_gate = np.asarray(g_gate)
    kth_tie, first_tie = oracle.near_tie_flags(o_logits, k, NEAR_TIE)
    strict = ~kth_tie
    # bit-exact selection and order where no near tie can flip them
    exact_order = strict & ~first_tie
    assert np.array_equal(g_idx[exact_order], o_idx[exact_order]), "expert ids differ"
    # 1st/2nd near tie: same set, order may swap
    if np.any(strict & first_tie):
        a = np.sort(g_idx[strict & first_tie], axis=1)
        b = np.sort(o_idx[strict & first_tie], axis=1)
        assert np.array_equal(a, b), "expert sets differ on a 1st/2nd near tie"
    # near ties of the k-th place: the GPU's choices must be valid
    T = g_idx.shape[0]
    srt = -np.sort(-o_logits.astype(np.float64), axis=1)
    kth_val = srt[:, k - 1]
    for t in np.nonzero(kth_tie)[0]:
        chosen = o_logits[t, g_idx[t]].astype(np.float64)
        assert np.all(chosen >= kth_val[t] - NEAR_TIE), f"token {t}: invalid near-tie routing"
        assert len(set(g_idx[t].tolist())) == k
    # gates: compare per expert id on tokens whose set matches
    same_set = np.array([set(g_idx[t]) == set(o_idx[t]) for t in range(T)])
    gerr = 0.0
    for t in np.nonzero(same_set)[0]:
        og = dict(zip(o_idx[t].tolist(), o_gate[t].tolist()))
        for s in range(k):
            gerr = max(gerr, abs(float(g_gate[t, s]) - og[int(g_idx[t, s])]))
    assert gerr <= GATE_TOL, f"gate error {gerr}"
    return strict, {"near_ties_kth": int(kth_tie.sum()), "near_ties_first": int(first_tie.sum()),
                    "gate_max_abs_err": gerr}


def check_y(y_gpu: torch.Tensor, y_ref: np.ndarray, rows=None, rms_ref=None):
    """max |y - y_ref| <= 2e-2 rms(y_ref) on the given rows; returns (err/rms, ulp stats)."""
    y = bf16_values(y_gpu)
    if rows is not None:
        y = y[rows]
        y_ref = y_ref[rows]
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if rms_ref is None else rms_ref
    err = np.abs(y - y_ref)
    rel = float(err.max() / rms) if err.size else 0.0
    assert rel <= Y_TOL, f"max|y-y_ref| = {rel:.4g} * rms(y_ref) > {Y_TOL}"
    ulps = err / bf16_ulp(y_ref)
    return rel, float(ulps.max()) if ulps.size else 0.0


def _silu_parts(a):
    sig = 1.0 / (1.0 + np.exp(-a))
    return a * sig, sig * (1.0 + a * (1.0 - sig))


def check_expert_rows(hv, ov, xv, row_expert, W1, W3, W2, h_ref, o_ref, expert_bias=None):
    """Expert kernel outputs on the given sorted rows against the oracle, with
    a-priori float32 accumulation bounds.

    hv, ov: GPU h (bf16 values, float64) and o (float64) of the rows; xv: the
    rows' inputs (bf16 values); row_expert: expert of each row; W1/W3/W2:
    torch bf16 weights [E, ...]; h_ref/o_ref: oracle outputs on the same rows.

    A float32 dot product of K terms accumulated in blocks of 16 has
    |error| <= (K/16 + 16) * 2^-24 * sum|terms|.  h = SiLU(a) * b is then within
    one bf16 ulp of the oracle's bf16 h plus the propagated accumulation error;
    o differs from the oracle's o by at most |h - h_ref| . |W2| plus GEMM2's own
    accumulation error.  With expert_bias = (b1, b3, b2) (float32 tensors) each
    bias is one more float32 addition: 2^-24 of the sum's magnitude on a, b and
    o.  Returns (fraction of h elements that differ, max o error / its bound).
    """
    u = 2.0 ** -24
    if expert_bias is not None:
        b1s, b3s, b2s = (b.detach().cpu().numpy().astype(np.float64) for b in expert_bias)
    from_bf16 = bf16_values
    K1 = xv.shape[1]
    K2 = hv.shape[1]
    g1 = (K1 / 16 + 16) * 2.0 ** -24
    g2 = (K2 / 16 + 16) * 2.0 ** -24
    worst = 0.0
    for e in np.unique(row_expert):
        m = row_expert == e
        x = xv[m]
        w1 = from_bf16(W1[int(e)])
        w3 = from_bf16(W3[int(e)])
        w2 = from_bf16(W2[int(e)])
        a = x @ w1
        b = x @ w3
        sa = np.abs(x) @ np.abs(w1)
        sb = np.abs(x) @ np.abs(w3)
        if expert_bias is not None:
            a = a + b1s[int(e)]
            b = b + b3s[int(e)]
            sa = sa + np.abs(a) / g1 * u     # the bias addition's rounding, in units of g1
            sb = sb + np.abs(b) / g1 * u
        silu, dsilu = _silu_parts(a)
        # + float32 evaluation of SiLU(a) * b itself (a few float32 ulps of h)
        tol_h = (bf16_ulp(h_ref[m]) * 1.0001 + g1 * (np.abs(dsilu * b) * sa + np.abs(silu) * sb)
                 + 16 * 2.0 ** -24 * np.abs(h_ref[m]))
        dh = np.abs(hv[m] - h_ref[m])
        assert np.all(dh <= tol_h), float(np.max(dh / tol_h))
        tol_o = dh @ np.abs(w2) + g2 * (np.abs(hv[m]) @ np.abs(w2))
        if expert_bias is not None:
            tol_o = tol_o + u * (np.abs(o_ref[m]) + tol_o)
        do = np.abs(ov[m] - o_ref[m])
        assert np.all(do <= tol_o * 1.0001 + 1e-30), float(np.max(do / (tol_o + 1e-30)))
        worst = max(worst, float(np.max(do / (tol_o + 1e-30))))
    frac = float(np.mean(hv != h_ref))
    assert frac < 0.02, frac
    return frac, worst
