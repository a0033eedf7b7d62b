"""The block edges around the layer (Mixtral page, "Прямой проход в формулах"):
H = U + MoE(RMSNorm_2(U)) through moe_block_forward against the oracle.

Bound on H: its one bf16 rounding (half an ulp of H) plus the layer's own
2e-2 * rms(MoE) parity bound; tokens whose routing is a near tie are excluded
(counted) as for the layer itself."""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_05_b200 as moe
from sparse_mixture_experts_05_b200.inputs import make_inputs, workload_inputs

from _parity import Y_TOL, bf16_ulp, bf16_values, to_dev

pytestmark = pytest.mark.gpu


def _gamma(d, seed):
    rng = np.random.default_rng(seed)
    return torch.from_numpy((1 + 0.2 * rng.standard_normal(d)).astype(np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("name", ["tiny", "ragged", "quarter"])
def test_block_forward_matches_oracle(name):
    inp = workload_inputs("quarter") if name == "quarter" else (
        workload_inputs("tiny") if name == "tiny" else make_inputs(77, 256, 384, 8, 2, 5, bias=True))
    T, d, d_ff, E, k = inp["shape"]
    gamma = _gamma(d, 7)
    dev = to_dev(inp)
    H = moe.moe_block_forward(inp["shape"], dev["x"], gamma.cuda(), dev["Wg"], dev["bias"],
                              dev["W1"], dev["W3"], dev["W2"], eps=1e-5)
    torch.cuda.synchronize()
    H_ref, _, _ = oracle.block_forward(inp["x"], gamma, inp["Wg"], inp["W1"], inp["W3"], inp["W2"],
                                       k, eps=1e-5, bias=inp["bias"])
    u_ref = oracle.rmsnorm(inp["x"], gamma, 1e-5)
    _, _, logits = oracle.route(u_ref, inp["Wg"], E, k, bias=inp["bias"])
    kth_tie, _ = oracle.near_tie_flags(logits, k)
    U = bf16_values(inp["x"])
    moe_part = H_ref - U
    rms = float(np.sqrt(np.mean(moe_part ** 2)))
    err = np.abs(bf16_values(H) - H_ref)[~kth_tie]
    bound = (0.5 * bf16_ulp(H_ref) + Y_TOL * rms)[~kth_tie]
    assert np.all(err <= bound), float(np.max(err / bound))


def test_block_zero_down_projection_returns_the_residual_exactly():
    inp = workload_inputs("tiny")
    dev = to_dev(inp)
    zero = torch.zeros_like(dev["W2"])
    H = moe.moe_block_forward(inp["shape"], dev["x"], _gamma(128, 8).cuda(), dev["Wg"], None,
                              dev["W1"], dev["W3"], zero)
    assert torch.equal(H, dev["x"])
