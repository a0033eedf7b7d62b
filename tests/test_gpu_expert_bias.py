"""Expert Linear biases on the GPU against the oracle.

The teaching configuration of the Mixtral textbook page (section "Подсчёт
параметров": bias on every Linear; d = 256, d_ff = 1024, E = 8, k = 2) gives each
expert SwiGLU(u) = (SiLU(u W1 + b1) * (u W3 + b3)) W2 + b2.  The kernels add the
biases to the float32 accumulators in their epilogues.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_05_b200 as moe
from sparse_mixture_experts_05_b200.inputs import expert_biases, make_inputs, workload_inputs

from _parity import bf16_values, check_expert_rows, check_routing, check_y, to_dev

pytestmark = pytest.mark.gpu

CASES = {
    # name: (T, d, d_ff, E, k, seed, router bias)
    "teaching": (300, 256, 1024, 8, 2, 21, True),   # R = 600: down projection on CTA pairs
    "tiny": (64, 128, 256, 8, 2, 22, False),        # single CTAs, ragged expert tails
    "E5k3": (45, 128, 384, 5, 3, 23, False),
}


def _inputs(name):
    if name == "quarter":
        inp = workload_inputs("quarter")
        T, d, d_ff, E, k = inp["shape"]
        return inp, expert_biases(E, d, d_ff, seed=101)
    T, d, d_ff, E, k, seed, bias = CASES[name]
    return (make_inputs(T, d, d_ff, E, k, seed, bias=bias),
            expert_biases(E, d, d_ff, seed=100 + seed))


ALL = list(CASES) + ["quarter"]


@pytest.mark.parametrize("name", ALL)
def test_expert_swiglu_bias(name):
    inp, eb = _inputs(name)
    T, d, d_ff, E, k = inp["shape"]
    o_idx, _, _ = oracle.route(inp["x"], inp["Wg"], E, k, bias=inp["bias"])
    r_off, r_perm, _ = oracle.dispatch(o_idx, E)
    xs = oracle.gather(inp["x"], r_perm)
    h_ref, o_ref = oracle.expert(xs, r_off, inp["W1"], inp["W3"], inp["W2"], expert_bias=eb)
    dev = to_dev(inp)
    xs_t = torch.from_numpy(xs.view(np.int16)).view(torch.bfloat16).cuda()
    h, o, ws = moe.moe_expert_swiglu_bias(inp["shape"], xs_t, torch.from_numpy(r_off).cuda(),
                                          dev["W1"], dev["W3"], dev["W2"],
                                          tuple(b.cuda() for b in eb))
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    row_expert = np.searchsorted(r_off, np.arange(T * k), side="right") - 1
    check_expert_rows(bf16_values(h), o.cpu().numpy().astype(np.float64), oracle.bf16_to_f64(xs),
                      row_expert, inp["W1"], inp["W3"], inp["W2"], h_ref, o_ref, expert_bias=eb)


@pytest.mark.parametrize("name", ALL)
def test_forward_bias(name):
    inp, eb = _inputs(name)
    T, d, d_ff, E, k = inp["shape"]
    dev = to_dev(inp)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    y = moe.moe_forward_bias(inp["shape"], dev["x"], dev["Wg"], dev["bias"], dev["W1"], dev["W3"],
                             dev["W2"], tuple(b.cuda() for b in eb), idx_out=idx, gate_out=gate)
    torch.cuda.synchronize()
    o_idx, o_gate, o_logits = oracle.route(inp["x"], inp["Wg"], E, k, bias=inp["bias"])
    strict, _ = check_routing(idx.cpu().numpy(), gate.cpu().numpy(), o_idx, o_gate, o_logits, k)
    y_ref, _, _ = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], k,
                                 bias=inp["bias"], expert_bias=eb)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    check_y(y, y_ref, rows=strict, rms_ref=rms)
    if not np.all(strict):
        g_idx = idx.cpu().numpy()
        f_off, f_perm, f_inv = oracle.dispatch(g_idx, E)
        _, f_o = oracle.expert(oracle.gather(inp["x"], f_perm), f_off, inp["W1"], inp["W3"],
                               inp["W2"], expert_bias=eb)
        check_y(y, oracle.combine(f_o, f_inv, gate.cpu().numpy()), rows=~strict, rms_ref=rms)


def test_null_biases_equal_the_unbiased_layer():
    """All three biases NULL is bit-for-bit moe_forward; zero biases too."""
    inp, eb = _inputs("tiny")
    T, d, d_ff, E, k = inp["shape"]
    dev = to_dev(inp)
    y0 = moe.moe_forward(inp["shape"], dev["x"], dev["Wg"], None, dev["W1"], dev["W3"], dev["W2"])
    y1 = moe.moe_forward_bias(inp["shape"], dev["x"], dev["Wg"], None, dev["W1"], dev["W3"],
                              dev["W2"], None)
    z = tuple(torch.zeros_like(b).cuda() for b in eb)
    y2 = moe.moe_forward_bias(inp["shape"], dev["x"], dev["Wg"], None, dev["W1"], dev["W3"],
                              dev["W2"], z)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1) and torch.equal(y0, y2)
