"""Mixtral 8x7B shapes at full size (d = 4096, d_ff = 14336, E = 8, k = 2):
prefill T = 4096, decode T = 16, skewed prefill T = 16384 with router bias, and
a T = 65536 batch near the largest the library accepts.

  * routing is checked on every token;
  * dispatch (offsets, the permutation, the inverse map and x_sorted) is
    compared bit for bit with the oracle's on every row, from the GPU's routing
    (the dispatch of section "Алгоритм" is integer bookkeeping: one correct
    answer);
  * the fused forward is checked on at least 256 sampled tokens per workload
    (every token for decode): the tokens of the first and last row of every
    expert group, every near-tie token, and random ones; tokens whose routing
    is a near tie are re-checked with the GPU's routing forced through the
    oracle's dispatch, experts and combine;
  * the expert kernel on sampled sorted rows, including the last row of every
    expert group, where tiles are ragged.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_05_b200 as moe
from sparse_mixture_experts_05_b200.inputs import workload_inputs

from _parity import bf16_values, check_expert_rows, check_routing, check_y, to_dev, u16

pytestmark = pytest.mark.gpu

SAMPLE_TOKENS = 256


@pytest.fixture(scope="module", params=["decode", "prefill", "skew", "max"])
def case(request):
    # "max": the prefill recipe at T = 65536, close to the largest batch the
    # library accepts at these widths (T * k * d_ff < 2^31)
    inp = (workload_inputs("prefill", T=65536) if request.param == "max"
           else workload_inputs(request.param))
    dev = to_dev(inp)
    T, d, d_ff, E, k = inp["shape"]
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    ws = moe.workspace(moe.moe_forward_workspace_bytes(inp["shape"]), "cuda")
    y = moe.moe_forward(inp["shape"], dev["x"], dev["Wg"], dev["bias"], dev["W1"], dev["W3"],
                        dev["W2"], idx_out=idx, gate_out=gate, ws=ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    yield request.param, inp, dev, idx.cpu().numpy(), gate.cpu().numpy(), y
    del dev, ws, y
    torch.cuda.empty_cache()


def test_routing_all_tokens(case):
    name, inp, dev, g_idx, g_gate, y = case
    T, d, d_ff, E, k = inp["shape"]
    o_idx, o_gate, o_logits = oracle.route(inp["x"], inp["Wg"], E, k, bias=inp["bias"])
    _, stats = check_routing(g_idx, g_gate, o_idx, o_gate, o_logits, k)
    print(name, stats)


def test_dispatch_bit_exact_all_rows(case):
    """Every sorted row: offsets, perm_tok, inv and x_sorted equal the oracle's
    dispatch of the same routing.  At T = 16384 and 65536 the index kernel's
    per-warp runs span many 256-slot batches, so this covers its carried
    positions across batches."""
    name, inp, dev, g_idx, g_gate, y = case
    T, d, d_ff, E, k = inp["shape"]
    offsets, perm, inv, xs = moe.moe_dispatch(inp["shape"], torch.from_numpy(g_idx).cuda(),
                                              dev["x"])
    r_off, r_perm, r_inv = oracle.dispatch(g_idx, E)
    assert np.array_equal(offsets.cpu().numpy(), r_off)
    assert np.array_equal(perm.cpu().numpy(), r_perm)
    assert np.array_equal(inv.cpu().numpy(), r_inv)
    R = T * k
    step = 8192  # rows per comparison: bounds the host memory at T = 65536
    for r0 in range(0, R, step):
        r1 = min(R, r0 + step)
        assert np.array_equal(u16(xs[r0:r1]), oracle.gather(inp["x"], r_perm[r0:r1])), (r0, r1)
    del offsets, perm, inv, xs


def _sample_tokens(T, g_idx, E, kth_tie, rng):
    """Tokens of the first and last sorted row of every expert group, every
    near-tie token, then random tokens up to SAMPLE_TOKENS (all tokens when T is
    no larger)."""
    if T <= SAMPLE_TOKENS:
        return np.arange(T)
    off, perm, _ = oracle.dispatch(g_idx, E)
    picks = {0, T - 1}
    for e in range(E):
        if off[e + 1] > off[e]:
            picks.update([int(perm[off[e]]), int(perm[off[e + 1] - 1])])
    picks.update(np.nonzero(kth_tie)[0].tolist())
    rest = np.setdiff1d(np.arange(T), np.fromiter(picks, int))
    need = max(0, SAMPLE_TOKENS - len(picks))
    picks.update(rng.choice(rest, need, replace=False).tolist())
    return np.array(sorted(picks))


def test_forward_sampled_tokens(case):
    name, inp, dev, g_idx, g_gate, y = case
    T, d, d_ff, E, k = inp["shape"]
    _, _, all_logits = oracle.route(inp["x"], inp["Wg"], E, k, bias=inp["bias"])
    all_kth_tie, _ = oracle.near_tie_flags(all_logits, k)
    toks = _sample_tokens(T, g_idx, E, all_kth_tie, np.random.default_rng(17))
    assert len(toks) >= min(T, SAMPLE_TOKENS)
    y_ref, r_idx, _ = oracle.forward_tokens(toks, inp["x"], inp["Wg"], inp["W1"], inp["W3"],
                                            inp["W2"], k, bias=inp["bias"])
    kth_tie = all_kth_tie[toks]
    same = np.array([set(g_idx[t]) == set(r_idx[i]) for i, t in enumerate(toks)])
    assert np.all(same | kth_tie)
    yv = y[torch.from_numpy(toks).long().cuda()]
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    rel, ulps = check_y(yv, y_ref, rows=same, rms_ref=rms)
    # near ties routed differently from the oracle: the GPU's own routing forced
    # through the oracle's dispatch, experts and combine
    diff = np.nonzero(~same)[0]
    if diff.size:
        tt = toks[diff]
        f_off, f_perm, f_inv = oracle.dispatch(g_idx[tt], E)
        x_sub = inp["x"][torch.from_numpy(tt).long()]
        _, f_o = oracle.expert(oracle.gather(x_sub, f_perm), f_off, inp["W1"], inp["W3"],
                               inp["W2"])
        y_forced = oracle.combine(f_o, f_inv, g_gate[tt])
        check_y(yv[torch.from_numpy(diff).long().cuda()], y_forced, rms_ref=rms)
    print(name, len(toks), "tokens; max|y-y_ref|/rms", rel, "max ulps", ulps,
          "near-tie tokens rerouted", int(diff.size))


def test_expert_sampled_rows(case):
    name, inp, dev, g_idx, g_gate, y = case
    T, d, d_ff, E, k = inp["shape"]
    shape = inp["shape"]
    offsets, perm, inv, xs = moe.moe_dispatch(shape, torch.from_numpy(g_idx).cuda(), dev["x"])
    h, o, ws = moe.moe_expert_swiglu(shape, xs, offsets, dev["W1"], dev["W3"], dev["W2"])
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    off = offsets.cpu().numpy()
    rng = np.random.default_rng(23)
    rows = set()
    for e in range(E):
        if off[e + 1] > off[e]:
            rows.update([int(off[e]), int(off[e + 1] - 1)])
            rows.update(rng.integers(off[e], off[e + 1], 2).tolist())
    rows = np.array(sorted(rows))
    row_expert = np.searchsorted(off, rows, side="right") - 1
    sub_off = np.concatenate([[0], np.cumsum(np.bincount(row_expert, minlength=E))]).astype(np.int32)
    xs_sub = xs[torch.from_numpy(rows).long().cuda()].cpu()
    h_ref, o_ref = oracle.expert(xs_sub, sub_off, inp["W1"], inp["W3"], inp["W2"])
    sel = torch.from_numpy(rows).long().cuda()
    frac, worst = check_expert_rows(bf16_values(h[sel]), o[sel].cpu().numpy().astype(np.float64),
                                    bf16_values(xs_sub), row_expert, inp["W1"], inp["W3"],
                                    inp["W2"], h_ref, o_ref)
    print(name, "h elements differing from the oracle", frac, "o error / bound", worst)


def test_hostio_batches_prefill_size_bit_exact():
    """The queue of host batches at the Mixtral prefill size (the bench's
    end-to-end path): three batches of 4096 tokens, two of them with the same
    host buffers (pinned) and one pageable, each equal to moe_forward on its x
    bit for bit."""
    inp = workload_inputs("prefill")
    dev = to_dev(inp)
    T, d, d_ff, E, k = inp["shape"]
    args = (dev["Wg"], dev["bias"], dev["W1"], dev["W3"], dev["W2"])
    g = torch.Generator().manual_seed(81)
    x1 = inp["x"].clone()
    x2 = (inp["x"].float() + 0.5 * torch.randn(T, d, generator=g)).to(torch.bfloat16)
    refs = [moe.moe_forward(inp["shape"], x.cuda(), *args).cpu() for x in (x1, x2)]
    xs = [x1.pin_memory(), x2.pin_memory(), x1.clone()]          # the last one pageable
    ys = [torch.empty(T, d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    ys.append(torch.empty(T, d, dtype=torch.bfloat16))
    ws = moe.workspace(moe.moe_forward_hostio_batches_workspace_bytes(inp["shape"]), "cuda")
    moe.moe_forward_hostio_batches(inp["shape"], xs, *args, ys, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    assert torch.equal(ys[0], refs[0])
    assert torch.equal(ys[1], refs[1])
    assert torch.equal(ys[2], refs[0])
