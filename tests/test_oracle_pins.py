"""Pins for the CPU oracle: each check compares it with something other than
itself -- numbers the pages print, closed forms, library routines, brute force or
a special case that reduces to a textbook formula.

Pages: the Mixtral textbook page (llm-arch-research), sections "Прямой проход в
формулах" (the MoE equation), "MoE изнутри" (the softmax over the k selected
logits equals the renormalised full softmax), "Алгоритм" (dispatch/combine loop,
k terms per token, kN routed rows), "Подсчёт параметров" (parameter counts); the
NVIDIA blog page "Applying Mixture of Experts in LLM Architectures" (C(8,2) = 28
expert pairs per layer).
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from sparse_mixture_experts_05_b200.inputs import expert_biases, identical_experts, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _f64(t) -> np.ndarray:
    return oracle.bf16_to_f64(t)


def _dense_swiglu(x, W1, W3, W2):
    """Textbook SwiGLU, (SiLU(x W1) * (x W3)) W2, with numpy float64 matmuls."""
    a = x @ W1
    b = x @ W3
    return ((a * expit(a)) * b) @ W2


# ---------------------------------------------------------------- bf16 rounding
def test_bf16_round_matches_torch_on_float32_values():
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32),
        (rng.standard_normal(50_000) * 1e-38).astype(np.float32),   # subnormal range
        (rng.standard_normal(50_000) * 3e38).astype(np.float32),    # near overflow
        np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38, 3.4e38, np.inf, -np.inf], np.float32),
    ])
    # exact ties: bf16 value + half an ulp (low 16 bits = 0x8000)
    ties = (rng.integers(0, 0x7F00, 20_000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    v = np.concatenate([v, ties, -ties])
    ref = _bits(torch.from_numpy(v).to(torch.bfloat16))
    got = oracle.round_bf16(v.astype(np.float64))
    assert np.array_equal(got, ref)


def _all_finite_bf16():
    bits = np.arange(0, 0x7F80, dtype=np.uint32)  # +0 .. largest finite
    return (bits << 16).view(np.float32).astype(np.float64)


def test_bf16_round_doubles_by_nearest_neighbour_search():
    """Doubles that are not float32 values: round by searching the sorted list of
    every finite bf16 value for the two neighbours (exact rationals), nearest
    wins, ties go to the even bit pattern."""
    vals = _all_finite_bf16()
    rng = np.random.default_rng(1)
    xs = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-40, 38, 3000))
    # exact midpoints between neighbours, then nudged by one double ulp each way
    for i in rng.integers(1, len(vals) - 2, 300):
        mid = (vals[i] + vals[i + 1]) / 2
        xs += [mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf)]
    for x in xs:
        ax = abs(x)
        j = int(np.searchsorted(vals, ax))
        if j == 0:
            want = 0.0
        elif j >= len(vals):
            top = Fraction(vals[-1])
            half_ulp = (Fraction(2) ** 128 - top) / 2
            want = math.inf if Fraction(ax) >= top + half_ulp else vals[-1]
        else:
            lo, hi = vals[j - 1], vals[j]
            if ax == hi:
                want = hi
            else:
                dlo = Fraction(ax) - Fraction(lo)
                dhi = Fraction(hi) - Fraction(ax)
                if dlo < dhi:
                    want = lo
                elif dhi < dlo:
                    want = hi
                else:
                    want = lo if (j - 1) % 2 == 0 else hi
        want = math.copysign(want, x)
        assert oracle.round_bf16_scalar(x) == want, x


# ---------------------------------------------------------------- SiLU
def test_silu_against_library_and_identities():
    a = np.linspace(-30, 30, 2001)
    got = np.array([oracle.silu(v) for v in a])
    assert np.allclose(got, a * expit(a), rtol=1e-14, atol=1e-300)
    assert oracle.silu(0.0) == 0.0
    # sigmoid(-a) = 1 - sigmoid(a)  =>  silu(a) - silu(-a) = a
    assert np.allclose(got - got[::-1], a, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- parameter counts
def _golden_counts():
    rows = []
    with open(os.path.join(GOLDEN, "param_counts.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            p = line.split()
            rows.append((p[0], [int(v) for v in p[1:11]], int(p[11]), int(p[12])))
    return rows


@pytest.mark.parametrize("row", _golden_counts(), ids=lambda r: r[0])
def test_param_counts_match_pages(row):
    name, (V, d, L, H, G, dh, d_ff, E, k, bias), total, active = row
    assert oracle.param_count(V, d, L, H, G, dh, d_ff, E, k, bias=bool(bias)) == (total, active)


def test_expert_share_of_mixtral():
    # Experts hold 45 097 156 608 parameters, 96.6% of the total (same section).
    tot, act = oracle.param_count(32000, 4096, 32, 32, 8, 128, 14336, 8, 2)
    tot0, _ = oracle.param_count(32000, 4096, 32, 32, 8, 128, 14336, 0, 0)
    experts = tot - tot0 - 32 * 4096 * 8
    assert experts == 45_097_156_608
    assert round(experts / tot, 3) == 0.966


# ---------------------------------------------------------------- router
def _case(T=96, d=128, d_ff=192, E=8, k=2, seed=11, bias=False):
    return make_inputs(T, d, d_ff, E, k, seed, bias=bias)


def _logits_numpy(inp):
    x = _f64(inp["x"])
    wg = _f64(inp["Wg"])
    g = x @ wg
    if inp["bias"] is not None:
        g = g + inp["bias"].numpy().astype(np.float64)
    return g


def test_router_logits_equal_float32_of_library_matmul():
    inp = _case(bias=True)
    _, _, logits = oracle.route(inp["x"], inp["Wg"], 8, 2, bias=inp["bias"])
    ref = _logits_numpy(inp).astype(np.float32)
    ulp = np.abs(np.spacing(ref))
    assert np.all(np.abs(logits - ref) <= ulp)


def test_top2_equals_brute_force_over_all_28_pairs():
    inp = _case(T=256)
    idx, _, logits = oracle.route(inp["x"], inp["Wg"], 8, 2)
    pairs = list(itertools.combinations(range(8), 2))
    assert len(pairs) == 28  # C(8,2), the NVIDIA blog's count of expert pairs per layer
    g = logits.astype(np.float64)
    for t in range(g.shape[0]):
        best = max(pairs, key=lambda p: (g[t, p[0]] + g[t, p[1]], -p[0], -p[1]))
        assert set(idx[t]) == set(best)
        assert g[t, idx[t, 0]] >= g[t, idx[t, 1]]


def test_topk_ties_go_to_lower_expert_index():
    inp = _case(T=32, E=8)
    wg = inp["Wg"].clone()
    wg[:, 5] = wg[:, 2]          # experts 2 and 5 produce identical logits
    inp["x"][:, 0] = torch.tensor(1.0, dtype=torch.bfloat16)
    wg[0, 2] = wg[0, 5] = torch.tensor(50.0, dtype=torch.bfloat16)
    idx, gate, logits = oracle.route(inp["x"], wg, 8, 2)
    assert np.all(logits[:, 2] == logits[:, 5])
    assert np.all(idx[:, 0] == 2) and np.all(idx[:, 1] == 5)
    assert np.all(gate == np.float32(0.5))


def test_gates_equal_renormalised_full_softmax():
    """Section "MoE изнутри": softmax over the top-k equals softmax over all E,
    restricted to the top-k and renormalised (the common denominator cancels)."""
    for k in (1, 2, 3, 8):
        inp = _case(T=200, seed=20 + k)
        idx, gate, logits = oracle.route(inp["x"], inp["Wg"], 8, k)
        g = logits.astype(np.float64)
        p = np.exp(g - g.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        sel = np.take_along_axis(p, idx.astype(np.int64), 1)
        hf = sel / sel.sum(1, keepdims=True)
        assert np.max(np.abs(gate - hf)) < 2e-7
        assert np.allclose(gate.sum(1), 1.0, atol=1e-6)
        if k == 1:
            assert np.all(gate == 1.0)
        if k == 8:
            assert np.max(np.abs(gate - np.take_along_axis(p, idx.astype(np.int64), 1))) < 2e-7


def test_bias_is_added_to_logits():
    inp = _case(T=64, bias=True)
    bias = torch.zeros(8)
    bias[6] = 100.0
    idx, _, _ = oracle.route(inp["x"], inp["Wg"], 8, 2, bias=bias)
    assert np.all(idx[:, 0] == 6)


def test_route_rejects_bad_k():
    inp = _case(T=4)
    for k in (0, 9):
        with pytest.raises(ValueError):
            oracle.route(inp["x"], inp["Wg"], 8, k)


# ---------------------------------------------------------------- dispatch
def test_dispatch_matches_numpy_where_and_invariants():
    inp = _case(T=333, seed=5)
    idx, _, _ = oracle.route(inp["x"], inp["Wg"], 8, 2)
    offsets, perm, inv = oracle.dispatch(idx, 8)
    T, k = idx.shape
    # numpy's nonzero on (idx == e) lists (token, slot) pairs in row-major order
    for e in range(8):
        tok, slot = np.nonzero(idx == e)
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.array_equal(seg, tok)
        assert np.array_equal(inv[tok, slot], np.arange(offsets[e], offsets[e + 1]))
    assert offsets[0] == 0 and offsets[-1] == T * k          # kN routed rows
    assert np.all(np.diff(offsets) >= 0)
    assert np.array_equal(np.bincount(perm, minlength=T), np.full(T, k))  # k terms per token
    assert np.array_equal(np.sort(inv.ravel()), np.arange(T * k))


def test_dispatch_empty_experts_and_empty_batch():
    idx = np.array([[3, 1], [1, 3], [3, 1]], np.int32)
    offsets, perm, inv = oracle.dispatch(idx, 8)
    assert offsets.tolist() == [0, 0, 3, 3, 6, 6, 6, 6, 6]
    assert perm.tolist() == [0, 1, 2, 0, 1, 2]
    assert inv.tolist() == [[3, 0], [1, 4], [5, 2]]
    offsets, perm, inv = oracle.dispatch(np.zeros((0, 2), np.int32), 8)
    assert offsets.tolist() == [0] * 9 and perm.size == 0


# ---------------------------------------------------------------- expert + combine
def test_E1_k1_reduces_to_dense_swiglu():
    inp = make_inputs(40, 64, 96, 1, 1, seed=3)
    y, idx, gate = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], 1,
                                  round_h=False)
    assert np.all(idx == 0) and np.all(gate == 1.0)
    ref = _dense_swiglu(_f64(inp["x"]), _f64(inp["W1"][0]), _f64(inp["W3"][0]), _f64(inp["W2"][0]))
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_identical_experts_give_swiglu_because_gates_sum_to_one():
    inp = identical_experts(make_inputs(50, 64, 128, 8, 2, seed=4))
    y, _, _ = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], 2,
                             round_h=False)
    ref = _dense_swiglu(_f64(inp["x"]), _f64(inp["W1"][0]), _f64(inp["W3"][0]), _f64(inp["W2"][0]))
    assert np.max(np.abs(y - ref)) <= 1e-6 * np.max(np.abs(ref))   # float32 gates sum to 1 +- 1e-7


def _dense_masked(inp, k):
    """All experts on all tokens, weighted by a dense [T,E] gate matrix that is
    zero off the top-k (renormalised full softmax of the float32 logits)."""
    x = _f64(inp["x"])
    g = _logits_numpy(inp).astype(np.float32).astype(np.float64)
    T, E = g.shape
    order = np.lexsort((np.tile(np.arange(E), (T, 1)), -g), axis=1)[:, :k]
    p = np.exp(g - g.max(1, keepdims=True))
    G = np.zeros_like(p)
    np.put_along_axis(G, order, np.take_along_axis(p, order, 1), 1)
    G /= G.sum(1, keepdims=True)
    y = np.zeros_like(x)
    for e in range(E):
        y += G[:, e:e + 1] * _dense_swiglu(x, _f64(inp["W1"][e]), _f64(inp["W3"][e]), _f64(inp["W2"][e]))
    return y


@pytest.mark.parametrize("k", [1, 2, 4])
def test_layer_equals_dense_all_experts_masked(k):
    inp = make_inputs(70, 64, 96, 8, k, seed=30 + k, bias=(k == 2))
    y, _, _ = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], k,
                             bias=inp["bias"], round_h=False)
    ref = _dense_masked(inp, k)
    assert np.max(np.abs(y - ref)) <= 2e-6 * np.max(np.abs(ref))


def test_per_token_loop_equals_expert_major_loop():
    inp = make_inputs(90, 64, 160, 8, 2, seed=6, bias=True)
    y, idx, gate = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], 2,
                                  bias=inp["bias"])
    toks = np.arange(90)[::-1].copy()
    y2, idx2, gate2 = oracle.forward_tokens(toks, inp["x"], inp["Wg"], inp["W1"], inp["W3"],
                                            inp["W2"], 2, bias=inp["bias"])
    assert np.array_equal(y[toks], y2)
    assert np.array_equal(idx[toks], idx2) and np.array_equal(gate[toks], gate2)


def test_bf16_storage_of_h_stays_within_rounding_budget():
    """Rounding h to bf16 (the down projection's input) moves y by far less than
    the 2e-2 rms parity bound; y itself comes back unrounded."""
    inp = make_inputs(128, 128, 256, 8, 2, seed=7)
    yr, _, _ = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], 2)
    ye, _, _ = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], 2,
                              round_h=False)
    rms = np.sqrt(np.mean(ye ** 2))
    assert 0 < np.max(np.abs(yr - ye)) < 1e-2 * rms


def test_combine_slot_order_equals_expert_order():
    """Accumulating over experts (section "Алгоритм") adds a token's terms in expert
    order; slot order gives the same value because both products are formed
    before a single addition of two terms (k = 2)."""
    rng = np.random.default_rng(8)
    T, d, k = 50, 32, 2
    o = rng.standard_normal((T * k, d))
    inv = rng.permutation(T * k).reshape(T, k).astype(np.int32)
    gate = rng.random((T, k)).astype(np.float32)
    y = oracle.combine(o, inv, gate)
    idx = rng.integers(0, 8, (T, k))
    y2 = np.zeros((T, d))
    for e in range(8):     # expert order, any fixed choice of experts per slot
        for t, s in zip(*np.nonzero(idx == e)):
            y2[t] += np.float64(gate[t, s]) * o[inv[t, s]]
    # a + b == b + a exactly in binary floating point
    assert np.array_equal(y, y2)


def test_planted_mistakes_fail_the_pins():
    """Swapping the gate and up projections, or feeding a transposed down
    projection, must break the dense-SwiGLU pin (shapes d != d_ff)."""
    inp = make_inputs(24, 64, 96, 1, 1, seed=9)
    ref = _dense_swiglu(_f64(inp["x"]), _f64(inp["W1"][0]), _f64(inp["W3"][0]), _f64(inp["W2"][0]))
    y_swapped, _, _ = oracle.forward(inp["x"], inp["Wg"], inp["W3"], inp["W1"], inp["W2"], 1,
                                     round_h=False)
    assert np.max(np.abs(y_swapped - ref)) > 1e-3 * np.max(np.abs(ref))
    sq = make_inputs(24, 64, 64, 1, 1, seed=9)
    ref_sq = _dense_swiglu(_f64(sq["x"]), _f64(sq["W1"][0]), _f64(sq["W3"][0]), _f64(sq["W2"][0]))
    W2t = sq["W2"].transpose(1, 2).contiguous()
    y_t, _, _ = oracle.forward(sq["x"], sq["Wg"], sq["W1"], sq["W3"], W2t, 1, round_h=False)
    assert np.max(np.abs(y_t - ref_sq)) > 1e-3 * np.max(np.abs(ref_sq))


# ---------------------------------------------------------------- expert Linear biases
# The teaching configuration of the Mixtral page (section "Подсчёт параметров",
# bias on every Linear) gives each expert's three projections a bias:
# SwiGLU(u) = (SiLU(u W1 + b1) * (u W3 + b3)) W2 + b2.

def _dense_swiglu_bias(x, W1, W3, W2, b1, b3, b2):
    a = x @ W1 + b1
    b = x @ W3 + b3
    return ((a * expit(a)) * b) @ W2 + b2


def _np_bias(bs):
    return tuple(b.numpy().astype(np.float64) for b in bs)


def test_expert_bias_E1_k1_reduces_to_dense_linear_layers_with_bias():
    inp = make_inputs(40, 64, 96, 1, 1, seed=13)
    eb = expert_biases(1, 64, 96, seed=113)
    y, _, _ = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], 1,
                             round_h=False, expert_bias=eb)
    b1, b3, b2 = _np_bias(eb)
    ref = _dense_swiglu_bias(_f64(inp["x"]), _f64(inp["W1"][0]), _f64(inp["W3"][0]),
                             _f64(inp["W2"][0]), b1[0], b3[0], b2[0])
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))
    # and the biases matter: without them the result is far off
    y0, _, _ = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], 1,
                              round_h=False)
    assert np.max(np.abs(y0 - ref)) > 1e-3 * np.max(np.abs(ref))


def test_expert_bias_closed_forms_with_zero_weights():
    """W2 = 0: every expert returns b2[e], so y_t = sum_s gate_ts b2[idx_ts].
    W1 = W3 = 0: h = SiLU(b1[e]) * b3[e] for every row of expert e."""
    T, d, d_ff, E, k = 30, 64, 96, 8, 2
    inp = make_inputs(T, d, d_ff, E, k, seed=14)
    eb = expert_biases(E, d, d_ff, seed=114)
    b1, b3, b2 = _np_bias(eb)
    zW2 = torch.zeros_like(inp["W2"])
    y, idx, gate = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], zW2, k,
                                  round_h=False, expert_bias=eb)
    ref = np.einsum("ts,tsc->tc", gate.astype(np.float64), b2[idx])
    assert np.max(np.abs(y - ref)) <= 1e-15 * np.max(np.abs(ref))
    zW = torch.zeros_like(inp["W1"])
    offsets = np.array([0, 3, 3, 7, 8, 8, 8, 12, 15], np.int32)
    xs = inp["x"][:15]
    h, o = oracle.expert(xs, offsets, zW, zW, inp["W2"], round_h=False, expert_bias=eb)
    row_e = np.repeat(np.arange(E), np.diff(offsets))
    h_ref = (b1 * expit(b1) * b3)[row_e]
    assert np.max(np.abs(h - h_ref)) <= 1e-15 * np.max(np.abs(h_ref))
    o_ref = np.stack([h_ref[r] @ _f64(inp["W2"][row_e[r]]) + b2[row_e[r]] for r in range(15)])
    assert np.max(np.abs(o - o_ref)) <= 1e-12 * np.max(np.abs(o_ref))


def test_expert_bias_layer_equals_dense_all_experts_masked():
    T, d, d_ff, E, k = 60, 64, 96, 8, 2
    inp = make_inputs(T, d, d_ff, E, k, seed=15, bias=True)
    eb = expert_biases(E, d, d_ff, seed=115)
    b1, b3, b2 = _np_bias(eb)
    y, _, _ = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], k,
                             bias=inp["bias"], round_h=False, expert_bias=eb)
    x = _f64(inp["x"])
    g = _logits_numpy(inp).astype(np.float32).astype(np.float64)
    order = np.lexsort((np.tile(np.arange(E), (T, 1)), -g), axis=1)[:, :k]
    p = np.exp(g - g.max(1, keepdims=True))
    G = np.zeros_like(p)
    np.put_along_axis(G, order, np.take_along_axis(p, order, 1), 1)
    G /= G.sum(1, keepdims=True)
    ref = np.zeros_like(x)
    for e in range(E):
        ref += G[:, e:e + 1] * _dense_swiglu_bias(x, _f64(inp["W1"][e]), _f64(inp["W3"][e]),
                                                  _f64(inp["W2"][e]), b1[e], b3[e], b2[e])
    assert np.max(np.abs(y - ref)) <= 2e-6 * np.max(np.abs(ref))
    # swapping the gate and up biases must break the pin
    ys, _, _ = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], k,
                              bias=inp["bias"], round_h=False, expert_bias=(eb[1], eb[0], eb[2]))
    assert np.max(np.abs(ys - ref)) > 1e-3 * np.max(np.abs(ref))


def test_expert_bias_per_token_loop_equals_expert_major_loop():
    inp = make_inputs(50, 64, 160, 8, 2, seed=16)
    eb = expert_biases(8, 64, 160, seed=116)
    y, idx, gate = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], 2,
                                  expert_bias=eb)
    toks = np.arange(50)[::-1].copy()
    y2, idx2, _ = oracle.forward_tokens(toks, inp["x"], inp["Wg"], inp["W1"], inp["W3"],
                                        inp["W2"], 2, expert_bias=eb)
    assert np.array_equal(y[toks], y2) and np.array_equal(idx[toks], idx2)


# ---------------------------------------------------------------- load-balancing loss
def test_aux_loss_is_k_under_uniform_load():
    """Section "Load-balancing loss": under uniform load the auxiliary term equals k."""
    E, T = 8, 64
    for k in (1, 2, 3):
        logits = np.zeros((T, E), np.float32)                 # P_i = 1/E
        idx = np.array([[(t + s) % E for s in range(k)] for t in range(T)], np.int32)  # f = 1/E
        aux, f, P = oracle.aux_loss(logits, idx)
        assert aux == pytest.approx(k, abs=1e-12)
        assert np.allclose(f, 1 / E) and np.allclose(P, 1 / E)


def test_aux_loss_closed_form_for_collapsed_routing_and_masking():
    E, T = 8, 40
    logits = np.full((T, E), -1e30, np.float32)
    logits[:, :2] = 0.0                                      # P = (1/2, 1/2, 0, ...)
    idx = np.tile(np.array([[0, 1]], np.int32), (T, 1))      # f_{0,0} = f_{1,1} = 1
    aux, _, P = oracle.aux_loss(logits, idx)
    assert aux == pytest.approx(E, abs=1e-12)                # E * (1 * 1/2 + 1 * 1/2)
    # padding tokens are not counted: append garbage rows with mask 0
    rng = np.random.default_rng(0)
    lg2 = np.concatenate([logits, rng.standard_normal((10, E)).astype(np.float32)])
    id2 = np.concatenate([idx, rng.integers(0, E, (10, 2)).astype(np.int32)])
    mask = np.concatenate([np.ones(T, np.uint8), np.zeros(10, np.uint8)])
    aux2, _, _ = oracle.aux_loss(lg2, id2, mask)
    assert aux2 == pytest.approx(E, abs=1e-12)


def test_aux_loss_matches_brute_force_definition():
    rng = np.random.default_rng(1)
    T, E, k = 37, 8, 2
    logits = rng.standard_normal((T, E)).astype(np.float32)
    idx, _, _ = oracle.route(make_inputs(T, 64, 128, E, k, seed=2)["x"],
                             make_inputs(T, 64, 128, E, k, seed=2)["Wg"], E, k)
    aux, f, P = oracle.aux_loss(logits, idx)
    # explicit double sums over (token, slot, expert) with scipy's softmax
    from scipy.special import softmax
    p = softmax(logits.astype(np.float64), axis=1)
    want = 0.0
    for s in range(k):
        for i in range(E):
            want += np.mean(idx[:, s] == i) * np.mean(p[:, i])
    assert aux == pytest.approx(E * want, rel=1e-12)


# ---------------------------------------------------------------- block edges (RMSNorm, residual)
def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def test_rmsnorm_closed_forms():
    d = 256
    # constant row c, gamma = 1: c / sqrt(c^2 + eps)
    for c in (0.5, -3.0, 1e-3):
        U = _bf16(np.full((1, d), c))
        u = oracle.bf16_to_f64(oracle.rmsnorm(U, _bf16(np.ones(d)), eps=1e-5))
        cv = float(_bf16([c])[0])
        want = oracle.bf16_to_f64(oracle.round_bf16(np.array([cv / math.sqrt(cv * cv + 1e-5)])))[0]
        assert np.all(u == want)
    # with eps = 0 the output is scale-free and has unit mean square before rounding
    rng = np.random.default_rng(3)
    z = rng.standard_normal((4, d))
    u1 = oracle.bf16_to_f64(oracle.rmsnorm(_bf16(z), _bf16(np.ones(d)), eps=0.0))
    u2 = oracle.bf16_to_f64(oracle.rmsnorm(_bf16(4 * z), _bf16(np.ones(d)), eps=0.0))  # 4x: exact in bf16
    assert np.array_equal(u1, u2)
    assert np.allclose(np.mean(u1 ** 2, axis=1), 1.0, atol=1e-2)
    # gamma scales column j; gamma = 0 gives zeros
    g = np.linspace(-2, 2, d)
    ug = oracle.bf16_to_f64(oracle.rmsnorm(_bf16(z), _bf16(g), eps=0.0))
    assert np.max(np.abs(ug - u1 * oracle.bf16_to_f64(oracle.round_bf16(g)))) <= 0.02 * np.max(np.abs(ug))
    assert np.all(oracle.bf16_to_f64(oracle.rmsnorm(_bf16(z), _bf16(np.zeros(d)))) == 0)


def test_block_residual_passes_through_when_the_layer_is_zero():
    inp = make_inputs(30, 128, 256, 8, 2, seed=50)
    gamma = _bf16(np.ones(128))
    zero_W2 = torch.zeros_like(inp["W2"])
    H, _, _ = oracle.block_forward(inp["x"], gamma, inp["Wg"], inp["W1"], inp["W3"], zero_W2, 2)
    assert np.array_equal(H, _f64(inp["x"]))
    H0, idx0, _ = oracle.block_forward(inp["x"], _bf16(np.zeros(128)), inp["Wg"], inp["W1"],
                                       inp["W3"], inp["W2"], 2)
    assert np.array_equal(H0, _f64(inp["x"]))          # u = 0 -> h = SiLU(0) * 0 = 0
    assert np.all(idx0 == np.array([0, 1]))            # all logits 0: ties go to the lower index


def test_block_equals_residual_plus_layer_of_the_normalised_rows():
    inp = make_inputs(40, 128, 256, 8, 2, seed=51, bias=True)
    rng = np.random.default_rng(4)
    gamma = _bf16(1 + 0.1 * rng.standard_normal(128))
    u = oracle.rmsnorm(inp["x"], gamma)
    y, idx, _ = oracle.forward(u, inp["Wg"], inp["W1"], inp["W3"], inp["W2"], 2, bias=inp["bias"])
    H, idx2, _ = oracle.block_forward(inp["x"], gamma, inp["Wg"], inp["W1"], inp["W3"], inp["W2"],
                                      2, bias=inp["bias"])
    assert np.array_equal(idx, idx2)
    assert np.array_equal(H, _f64(inp["x"]) + y)
