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


BLOCK_CASES = {
    # the router normalises the rows itself; its cluster size (CTAs sharing a
    # token tile's contraction) depends on T and d: 1 for tiny and ragged, 4 for
    # the quarter-width batch, 8 for the decode-sized batch at d = 4096
    "ragged": (77, 256, 384, 8, 2, 5, True),
    "decode-d4096": (16, 4096, 256, 8, 2, 6, False),
    "mid-d2048": (300, 2048, 256, 8, 2, 7, True),
    # at least one 16-token tile per SM (148 SMs): the streaming router, which
    # normalises the tile it holds in shared memory
    "stream-d1024": (3000, 1024, 512, 8, 2, 11, True),
    "stream-d4096": (2400, 4096, 256, 8, 2, 12, False),
}


@pytest.mark.parametrize("name", ["tiny", "ragged", "quarter", "decode-d4096", "mid-d2048",
                                  "stream-d1024", "stream-d4096"])
def test_block_forward_matches_oracle(name):
    if name in BLOCK_CASES:
        T, d, d_ff, E, k, seed, bias = BLOCK_CASES[name]
        inp = make_inputs(T, d, d_ff, E, k, seed, bias=bias)
    else:
        inp = workload_inputs(name)
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


@pytest.mark.parametrize("name", ["quarter", "decode-d4096", "stream-d1024", "stream-d4096"])
def test_router_normalised_rows_match_oracle_rmsnorm(name):
    """The router writes u = bf16((U * inv) * gamma) into the block workspace (right
    after moe_forward's part) for the scatter; u equals the oracle's RMSNorm to
    within one bf16 ulp (the float32 sum of squares is added in another order
    than the oracle's double sum), and nearly always exactly."""
    if name in BLOCK_CASES:
        T, d, d_ff, E, k, seed, bias = BLOCK_CASES[name]
        inp = make_inputs(T, d, d_ff, E, k, seed, bias=bias)
    else:
        inp = workload_inputs(name)
    T, d, d_ff, E, k = inp["shape"]
    gamma = _gamma(d, 9)
    dev = to_dev(inp)
    ws = moe.workspace(moe.moe_block_workspace_bytes(inp["shape"]), "cuda")
    moe.moe_block_forward(inp["shape"], dev["x"], gamma.cuda(), dev["Wg"], dev["bias"], dev["W1"],
                          dev["W3"], dev["W2"], eps=1e-5, ws=ws)
    torch.cuda.synchronize()
    off = moe.moe_forward_workspace_bytes(inp["shape"])
    u = ws[off:off + T * d * 2].view(torch.bfloat16).view(T, d)
    u_ref = oracle.bf16_to_f64(oracle.rmsnorm(inp["x"], gamma, 1e-5))
    uv = bf16_values(u)
    diff = np.abs(uv - u_ref)
    assert np.all(diff <= bf16_ulp(u_ref) * 1.0001 + 1e-30)
    assert np.mean(diff > 0) < 1e-3



def test_block_forward_prefill_size_sampled_tokens():
    """The block edges at the Mixtral 8x7B prefill size (T = 4096, d = 4096,
    d_ff = 14336), where the streaming router normalises the rows it holds in
    shared memory: u on every row against the oracle's RMSNorm (within one
    bf16 ulp), and H on at least 256 sampled tokens -- the first and last row of
    every expert group, the near ties, random ones -- against U plus the
    oracle's layer on the GPU's u (so both sides route the same rows; near ties
    of the k-th place are counted and left out, as for the layer's own parity)."""
    inp = workload_inputs("prefill")
    T, d, d_ff, E, k = inp["shape"]
    gamma = _gamma(d, 15)
    dev = to_dev(inp)
    ws = moe.workspace(moe.moe_block_workspace_bytes(inp["shape"]), "cuda")
    H = moe.moe_block_forward(inp["shape"], dev["x"], gamma.cuda(), dev["Wg"], None, dev["W1"],
                              dev["W3"], dev["W2"], eps=1e-5, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    off = moe.moe_forward_workspace_bytes(inp["shape"])
    u = ws[off:off + T * d * 2].view(torch.bfloat16).view(T, d).cpu()
    u_ref = oracle.bf16_to_f64(oracle.rmsnorm(inp["x"], gamma, 1e-5))
    diff = np.abs(bf16_values(u) - u_ref)
    assert np.all(diff <= bf16_ulp(u_ref) * 1.0001 + 1e-30)
    assert np.mean(diff > 0) < 1e-3

    o_idx, _, o_logits = oracle.route(u, inp["Wg"], E, k)
    kth_tie, _ = oracle.near_tie_flags(o_logits, k)
    off_e, perm, _ = oracle.dispatch(o_idx, E)
    picks = {0, T - 1}
    for e in range(E):
        if off_e[e + 1] > off_e[e]:
            picks.update([int(perm[off_e[e]]), int(perm[off_e[e + 1] - 1])])
    picks.update(np.nonzero(kth_tie)[0].tolist())
    rng = np.random.default_rng(29)
    rest = np.setdiff1d(np.arange(T), np.fromiter(picks, int))
    picks.update(rng.choice(rest, max(0, 256 - len(picks)), replace=False).tolist())
    toks = np.array(sorted(picks))
    y_ref, _, _ = oracle.forward_tokens(toks, u, inp["Wg"], inp["W1"], inp["W3"], inp["W2"], k)
    keep = ~kth_tie[toks]
    U = bf16_values(inp["x"][torch.from_numpy(toks).long()])
    H_ref = U + y_ref
    Hv = bf16_values(H[torch.from_numpy(toks).long().cuda()])
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    err = np.abs(Hv - H_ref)[keep]
    bound = (0.5 * bf16_ulp(H_ref) + Y_TOL * rms)[keep]
    assert np.all(err <= bound), float(np.max(err / bound))
    print("tokens", len(toks), "near ties left out", int((~keep).sum()),
          "max err / bound", float(np.max(err / bound)))
