"""Load-balancing auxiliary term (Mixtral page, section "Load-balancing loss"):
the CUDA kernel against the oracle on the router's own logits and choices,
with padding masks, and the uniform-load closed form (aux = k)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_05_b200 as moe
from sparse_mixture_experts_05_b200.inputs import make_inputs, workload_inputs

from _parity import to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", ["tiny", "quarter", "layers", "k4"])
def test_aux_loss_matches_oracle(case):
    if case == "layers":   # three layers' rows stacked, as the page gathers them
        inps = [make_inputs(300, 256, 256, 8, 2, seed=60 + i, bias=(i == 1)) for i in range(3)]
    elif case == "k4":
        inps = [make_inputs(500, 256, 256, 16, 4, seed=64)]
    else:
        inps = [workload_inputs(case)]
    logits, idx = [], []
    for inp in inps:
        dev = to_dev(inp)
        i_, g_, l_ = moe.moe_route(inp["shape"], dev["x"], dev["Wg"], dev["bias"], want_logits=True)
        logits.append(l_)
        idx.append(i_)
    logits = torch.cat(logits)
    idx = torch.cat(idx)
    T, E = logits.shape
    k = idx.shape[1]
    rng = np.random.default_rng(5)
    for mask in (None, torch.from_numpy((rng.random(T) > 0.3).astype(np.uint8)).cuda()):
        aux, f, P = moe.moe_aux_loss((T, 128, 128, E, k), logits, idx, mask=mask, want_stats=True)
        ref, f_ref, P_ref = oracle.aux_loss(logits.cpu().numpy(), idx.cpu().numpy(),
                                            None if mask is None else mask.cpu().numpy())
        assert abs(float(aux.item()) - ref) <= 1e-5 * ref
        assert np.max(np.abs(f.cpu().numpy() - f_ref)) <= 1e-7
        assert np.max(np.abs(P.cpu().numpy() - P_ref)) <= 2e-6


def test_aux_loss_uniform_load_equals_k():
    E, T, k = 8, 4096, 2
    logits = torch.zeros(T, E, dtype=torch.float32, device="cuda")
    idx = torch.tensor([[(t + s) % E for s in range(k)] for t in range(T)], dtype=torch.int32,
                       device="cuda")
    aux, _, _ = moe.moe_aux_loss((T, 128, 128, E, k), logits, idx)
    assert float(aux.item()) == pytest.approx(k, rel=1e-6)


def test_aux_loss_deterministic():
    inp = to_dev(workload_inputs("quarter"))
    idx, _, logits = moe.moe_route(inp["shape"], inp["x"], inp["Wg"], want_logits=True)
    shape = (1024, 128, 128, 8, 2)
    a = [moe.moe_aux_loss(shape, logits, idx)[0].item() for _ in range(3)]
    assert a[0] == a[1] == a[2]
