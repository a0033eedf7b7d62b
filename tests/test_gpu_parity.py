"""CUDA path vs CPU oracle, element by element, through the C ABI.

Every kernel is checked on its own (same inputs on both sides) and the fused
forward is checked end to end, on the tiny and quarter-width workloads, on
ragged and degenerate shapes, and -- in test_gpu_fullsize.py -- on the
Mixtral 8x7B workloads at full size.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_05_b200 as moe
from sparse_mixture_experts_05_b200.inputs import identical_experts, make_inputs, workload_inputs

from _parity import (bf16_ulp, bf16_values, check_expert_rows, check_routing, check_y, to_dev,
                     u16)

pytestmark = pytest.mark.gpu

CASES = {
    # name: (T, d, d_ff, E, k, seed, bias)
    "tiny": (64, 128, 256, 8, 2, 0, False),
    "ragged": (77, 256, 384, 8, 2, 5, False),
    "tail": (300, 128, 256, 8, 2, 6, True),
    "k1": (50, 128, 256, 8, 1, 7, False),
    "E1k1": (40, 128, 128, 1, 1, 8, False),
    "E16k4": (96, 256, 256, 16, 4, 9, False),
    "E5k3": (33, 128, 256, 5, 3, 10, False),
    "E32k8": (64, 128, 256, 32, 8, 18, False),    # the largest E and k the library takes
    "single": (1, 128, 256, 8, 2, 11, False),
    "batch16": (16, 256, 384, 8, 2, 16, True),    # decode-sized: R = 32 rows over 8 experts
    "batch30": (30, 128, 512, 8, 2, 17, False),
    # GEMM1 on CTA pairs with its half tiles in place (R = 9600 rows: about 16
    # rounds of pair tiles), GEMM2 on pairs with its half tiles last
    "pairs-inline": (4800, 256, 4096, 8, 2, 19, True),
    # one expert: four full pair tiles and a 76-row half tile
    "E1-pairs": (1100, 256, 512, 1, 1, 21, False),
}


def _inputs(name):
    if name == "quarter":
        return workload_inputs("quarter")
    T, d, d_ff, E, k, seed, bias = CASES[name]
    return make_inputs(T, d, d_ff, E, k, seed, bias=bias)


ALL = list(CASES) + ["quarter"]


@pytest.mark.parametrize("name", ALL)
def test_route(name):
    inp = _inputs(name)
    T, d, d_ff, E, k = inp["shape"]
    dev = to_dev(inp)
    idx, gate, logits = moe.moe_route(inp["shape"], dev["x"], dev["Wg"], dev["bias"],
                                      want_logits=True)
    torch.cuda.synchronize()
    o_idx, o_gate, o_logits = oracle.route(inp["x"], inp["Wg"], E, k, bias=inp["bias"])
    lerr = np.max(np.abs(logits.cpu().numpy() - o_logits))
    assert lerr < 1e-4, lerr
    check_routing(idx.cpu().numpy(), gate.cpu().numpy(), o_idx, o_gate, o_logits, k)


@pytest.mark.parametrize("T,d,E,k", [(40, 10240, 8, 2), (40, 8192, 8, 2), (40, 2560, 32, 8)],
                         ids=["d10240", "d8192", "E32-d2560"])
def test_route_wide_rows(T, d, E, k):
    # W_r staged in shared memory near the largest size the library takes (160 KB)
    inp = make_inputs(T, d, 128, E, k, seed=20 + E, bias=True)
    dev = to_dev(inp)
    idx, gate, logits = moe.moe_route(inp["shape"], dev["x"], dev["Wg"], dev["bias"],
                                      want_logits=True)
    torch.cuda.synchronize()
    o_idx, o_gate, o_logits = oracle.route(inp["x"], inp["Wg"], E, k, bias=inp["bias"])
    lerr = np.max(np.abs(logits.cpu().numpy() - o_logits))
    assert lerr < 1e-4, lerr
    check_routing(idx.cpu().numpy(), gate.cpu().numpy(), o_idx, o_gate, o_logits, k)


# Batches with at least one 16-token tile per SM run the streaming router (one
# CTA per SM, a TMA ring per consumer warp, an epilogue warp); these shapes
# cover its variants on 148 SMs: the threshold batch (148 tiles of 16 rows),
# ragged last tiles, E not a multiple of 8 (W_r staged with plain stores), two
# and four 8-expert planes, rings 1 to 4 slots deep holding 2 to 8 chunks of 64
# columns, with the router bias and the logits output.
STREAM_ROUTE = {
    "threshold-d4096": (2368, 4096, 8, 2),
    "ragged-E5k3-d1024": (3001, 1024, 5, 3),
    "E32k8-d1024": (4097, 1024, 32, 8),
    "E16k4-d2048": (5000, 2048, 16, 4),
    "d1536": (2500, 1536, 8, 2),
    # rings 4 slots deep refilled: 5-6 tiles of 14 rows per CTA at d = 1024
    "depth4-reuse-d1024": (12000, 1024, 8, 2),
}


@pytest.mark.parametrize("name", list(STREAM_ROUTE))
def test_route_streaming_kernel_shapes(name):
    T, d, E, k = STREAM_ROUTE[name]
    inp = make_inputs(T, d, 128, E, k, seed=30 + E + k, bias=True)
    dev = to_dev(inp)
    idx, gate, logits = moe.moe_route(inp["shape"], dev["x"], dev["Wg"], dev["bias"],
                                      want_logits=True)
    torch.cuda.synchronize()
    o_idx, o_gate, o_logits = oracle.route(inp["x"], inp["Wg"], E, k, bias=inp["bias"])
    lerr = np.max(np.abs(logits.cpu().numpy() - o_logits))
    assert lerr < 1e-4, lerr
    check_routing(idx.cpu().numpy(), gate.cpu().numpy(), o_idx, o_gate, o_logits, k)


def test_route_ties_to_lower_index():
    inp = make_inputs(48, 128, 256, 8, 2, seed=12)
    inp["Wg"][:, 6] = inp["Wg"][:, 3]
    inp["x"][:, 0] = 1.0
    inp["Wg"][0, 3] = inp["Wg"][0, 6] = 40.0
    dev = to_dev(inp)
    idx, gate, logits = moe.moe_route(inp["shape"], dev["x"], dev["Wg"], want_logits=True)
    idx = idx.cpu().numpy()
    lg = logits.cpu().numpy()
    assert np.all(lg[:, 3] == lg[:, 6])
    assert np.all(idx[:, 0] == 3) and np.all(idx[:, 1] == 6)
    assert np.all(gate.cpu().numpy() == 0.5)


@pytest.mark.parametrize("name", ALL)
def test_dispatch_bit_exact(name):
    inp = _inputs(name)
    T, d, d_ff, E, k = inp["shape"]
    o_idx, _, _ = oracle.route(inp["x"], inp["Wg"], E, k, bias=inp["bias"])
    dev = to_dev(inp)
    offsets, perm, inv, xs = moe.moe_dispatch(inp["shape"], torch.from_numpy(o_idx).cuda(),
                                              dev["x"])
    r_off, r_perm, r_inv = oracle.dispatch(o_idx, E)
    assert np.array_equal(offsets.cpu().numpy(), r_off)
    assert np.array_equal(perm.cpu().numpy(), r_perm)
    assert np.array_equal(inv.cpu().numpy(), r_inv)
    assert np.array_equal(u16(xs), oracle.gather(inp["x"], r_perm))


def test_dispatch_skips_out_of_range_ids():
    T, d, E, k = 40, 128, 8, 2
    x = torch.randn(T, d).to(torch.bfloat16).cuda()
    idx = torch.randint(0, E, (T, k), dtype=torch.int32)
    idx[:, 1] = (idx[:, 0] + 1) % E
    idx[5, 1] = -1
    idx[9, 0] = E
    offsets, perm, inv, xs = moe.moe_dispatch((T, d, 256, E, k), idx.cuda(), x)
    inv = inv.cpu().numpy()
    assert inv[5, 1] == -1 and inv[9, 0] == -1
    assert offsets.cpu().numpy()[-1] == T * k - 2
    valid = idx.numpy()
    keep = (valid >= 0) & (valid < E)
    assert np.all(inv[keep] >= 0)
    assert np.array_equal(np.sort(inv[keep]), np.arange(T * k - 2))


@pytest.mark.parametrize("name", ALL)
def test_expert_swiglu(name):
    inp = _inputs(name)
    T, d, d_ff, E, k = inp["shape"]
    o_idx, _, _ = oracle.route(inp["x"], inp["Wg"], E, k, bias=inp["bias"])
    r_off, r_perm, _ = oracle.dispatch(o_idx, E)
    xs = oracle.gather(inp["x"], r_perm)
    h_ref, o_ref = oracle.expert(xs, r_off, inp["W1"], inp["W3"], inp["W2"])
    dev = to_dev(inp)
    xs_t = torch.from_numpy(xs.view(np.int16)).view(torch.bfloat16).cuda()
    h, o, ws = moe.moe_expert_swiglu(inp["shape"], xs_t, torch.from_numpy(r_off).cuda(),
                                     dev["W1"], dev["W3"], dev["W2"])
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    row_expert = np.searchsorted(r_off, np.arange(T * k), side="right") - 1
    check_expert_rows(bf16_values(h), o.cpu().numpy().astype(np.float64), oracle.bf16_to_f64(xs),
                      row_expert, inp["W1"], inp["W3"], inp["W2"], h_ref, o_ref)


def test_expert_swiglu_extreme_gate_inputs():
    """SiLU's tails: W1 scaled by 32 and W3 by 4 (powers of two, so the bf16
    weights stay exact) make a = x W1 span about +-100 and b = x W3 about +-12,
    including many a < -87.3, where 1 + e^-a exceeds 2^126.  h must still meet
    the one-bf16-ulp-plus-accumulation bound against the oracle there."""
    inp = make_inputs(512, 256, 512, 8, 2, seed=47)
    inp["W1"] = (inp["W1"].float() * 32).to(torch.bfloat16)
    inp["W3"] = (inp["W3"].float() * 4).to(torch.bfloat16)
    T, d, d_ff, E, k = inp["shape"]
    o_idx, _, _ = oracle.route(inp["x"], inp["Wg"], E, k)
    r_off, r_perm, _ = oracle.dispatch(o_idx, E)
    xs = oracle.gather(inp["x"], r_perm)
    h_ref, o_ref = oracle.expert(xs, r_off, inp["W1"], inp["W3"], inp["W2"])
    row_expert = np.searchsorted(r_off, np.arange(T * k), side="right") - 1
    xv = oracle.bf16_to_f64(xs)
    a = np.concatenate([xv[row_expert == e] @ bf16_values(inp["W1"][e]) for e in range(E)])
    assert a.min() < -100 and a.max() > 100
    assert np.sum((a < -87.3) & (a > -104)) > 100   # the region the plain form gets wrong
    dev = to_dev(inp)
    xs_t = torch.from_numpy(xs.view(np.int16)).view(torch.bfloat16).cuda()
    h, o, ws = moe.moe_expert_swiglu(inp["shape"], xs_t, torch.from_numpy(r_off).cuda(),
                                     dev["W1"], dev["W3"], dev["W2"])
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    check_expert_rows(bf16_values(h), o.cpu().numpy().astype(np.float64), xv, row_expert,
                      inp["W1"], inp["W3"], inp["W2"], h_ref, o_ref)


@pytest.mark.parametrize("name", ALL)
def test_combine(name):
    inp = _inputs(name)
    T, d, d_ff, E, k = inp["shape"]
    rng = np.random.default_rng(3)
    o32 = rng.standard_normal((T * k, d)).astype(np.float32)
    inv = rng.permutation(T * k).reshape(T, k).astype(np.int32)
    gate = rng.random((T, k)).astype(np.float32)
    gate /= gate.sum(1, keepdims=True)
    y = moe.moe_combine(inp["shape"], torch.from_numpy(o32).cuda(), torch.from_numpy(inv).cuda(),
                        torch.from_numpy(gate).cuda())
    y_ref = oracle.combine(o32.astype(np.float64), inv, gate)
    err = np.abs(bf16_values(y) - y_ref)
    # float32 products and their sum each round once (relative 2^-24 of their own
    # magnitude), then y rounds once to bf16: |err| <= ulp/2 + 2^-23 * sum_s |g_s o_s|
    mag = oracle.combine(np.abs(o32.astype(np.float64)), inv, gate)
    assert np.all(err <= 0.5 * bf16_ulp(y_ref) + 2.0 ** -23 * mag + 1e-30)
    assert np.mean(err > 0.5 * bf16_ulp(y_ref)) < 1e-3


def _forward_and_check(inp, ws=None):
    T, d, d_ff, E, k = inp["shape"]
    dev = to_dev(inp)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    y = moe.moe_forward(inp["shape"], dev["x"], dev["Wg"], dev["bias"], dev["W1"], dev["W3"],
                        dev["W2"], idx_out=idx, gate_out=gate, ws=ws)
    torch.cuda.synchronize()
    o_idx, o_gate, o_logits = oracle.route(inp["x"], inp["Wg"], E, k, bias=inp["bias"])
    g_idx = idx.cpu().numpy()
    g_gate = gate.cpu().numpy()
    strict, stats = check_routing(g_idx, g_gate, o_idx, o_gate, o_logits, k)
    y_ref, _, _ = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], k,
                                 bias=inp["bias"])
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    rel, ulps = check_y(y, y_ref, rows=strict, rms_ref=rms)
    # forced routing: the GPU's idx/gate through the oracle's dispatch, experts and combine
    if not np.all(strict):
        f_off, f_perm, f_inv = oracle.dispatch(g_idx, E)
        _, f_o = oracle.expert(oracle.gather(inp["x"], f_perm), f_off, inp["W1"], inp["W3"],
                               inp["W2"])
        y_forced = oracle.combine(f_o, f_inv, g_gate)
        check_y(y, y_forced, rows=~strict, rms_ref=rms)
    return y, stats, rel


@pytest.mark.parametrize("name", ALL)
def test_forward(name):
    _forward_and_check(_inputs(name))


def test_forward_identical_experts_equal_swiglu():
    inp = identical_experts(make_inputs(64, 128, 256, 8, 2, seed=13))
    y, _, _ = _forward_and_check(inp)
    x = bf16_values(inp["x"])
    W1 = bf16_values(inp["W1"][0])
    W3 = bf16_values(inp["W3"][0])
    W2 = bf16_values(inp["W2"][0])
    a = x @ W1
    ref = ((a / (1 + np.exp(-a))) * (x @ W3)) @ W2
    assert np.max(np.abs(bf16_values(y) - ref)) <= 2e-2 * np.sqrt(np.mean(ref ** 2))


def test_forward_all_tokens_one_expert():
    inp = make_inputs(200, 128, 256, 8, 2, seed=14)
    inp["bias"] = torch.tensor([0, 0, 0, 50.0, 0, 0, 0, 0], dtype=torch.float32)
    y, _, _ = _forward_and_check(inp)


def test_forward_empty_batch_is_noop():
    inp = make_inputs(0, 128, 256, 8, 2, seed=15)
    dev = to_dev(inp)
    y = torch.full((0, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(inp["shape"], dev["x"], dev["Wg"], None, dev["W1"], dev["W3"], dev["W2"], y=y,
                    ws=moe.workspace(4096, "cuda"))
    torch.cuda.synchronize()


def test_forward_deterministic_and_hostio_matches():
    inp = workload_inputs("tiny")
    T, d, d_ff, E, k = inp["shape"]
    dev = to_dev(inp)
    ws = moe.workspace(moe.moe_forward_hostio_workspace_bytes(inp["shape"]), "cuda")
    y1 = moe.moe_forward(inp["shape"], dev["x"], dev["Wg"], None, dev["W1"], dev["W3"], dev["W2"],
                         ws=ws)
    y2 = moe.moe_forward(inp["shape"], dev["x"], dev["Wg"], None, dev["W1"], dev["W3"], dev["W2"],
                         ws=ws)
    x_host = inp["x"].clone().pin_memory()
    y_host = torch.empty(T, d, dtype=torch.bfloat16).pin_memory()
    moe.moe_forward_hostio(inp["shape"], x_host, dev["Wg"], None, dev["W1"], dev["W3"], dev["W2"],
                           y_host, ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert torch.equal(y1.cpu(), y_host)


@pytest.mark.parametrize("T", [2048, 4097], ids=["2048-tokens", "4097-tokens"])
def test_hostio_token_chunks_equal_the_whole_batch(T):
    """Large host-I/O batches run as a pipeline of token chunks; every row's
    arithmetic (including the router's summation split) is that of the whole
    batch, so y matches moe_forward bit for bit."""
    inp = make_inputs(T, 1024, 512, 8, 2, seed=19, bias=True)
    dev = to_dev(inp)
    args = (dev["Wg"], dev["bias"], dev["W1"], dev["W3"], dev["W2"])
    y_dev = moe.moe_forward(inp["shape"], dev["x"], *args)
    x_host = inp["x"].clone().pin_memory()
    y_host = torch.full((T, 1024), 3.0, dtype=torch.bfloat16).pin_memory()
    ws = moe.workspace(moe.moe_forward_hostio_workspace_bytes(inp["shape"]), "cuda")
    for _ in range(2):  # twice on the same buffers: the pipeline orders itself after earlier work
        moe.moe_forward_hostio(inp["shape"], x_host, *args, y_host, ws)
    torch.cuda.synchronize()
    assert torch.equal(y_dev.cpu(), y_host)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK


@pytest.mark.parametrize("T,E,k", [(3200, 5, 3), (4097, 32, 8), (3500, 16, 4), (12000, 8, 2)],
                         ids=["E5k3", "E32k8", "E16k4", "E8k2-deep-rings"])
def test_hostio_chunks_route_alike_in_both_router_kernels(T, E, k):
    """The host-I/O pipeline routes its small edge chunks through the cluster
    router (C = 1, the whole batch's split) and its large middle chunk through
    the streaming router; the whole batch, through moe_forward, takes the
    streaming router for every token.  Equal y bit for bit means both kernels
    gave every token the same expert ids and the same gate bits."""
    inp = make_inputs(T, 1024, 256, E, k, seed=40 + E, bias=True)
    dev = to_dev(inp)
    args = (dev["Wg"], dev["bias"], dev["W1"], dev["W3"], dev["W2"])
    y_dev = moe.moe_forward(inp["shape"], dev["x"], *args)
    x_host = inp["x"].clone().pin_memory()
    y_host = torch.full((T, 1024), 3.0, dtype=torch.bfloat16).pin_memory()
    ws = moe.workspace(moe.moe_forward_hostio_workspace_bytes(inp["shape"]), "cuda")
    moe.moe_forward_hostio(inp["shape"], x_host, *args, y_host, ws)
    torch.cuda.synchronize()
    assert torch.equal(y_dev.cpu(), y_host)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK


@pytest.mark.parametrize("T,n", [(700, 5), (64, 1), (2048, 3)],
                         ids=["five-batches", "one-batch", "three-large-batches"])
def test_hostio_batches_equal_per_batch_forwards(T, n):
    """A queue of batches through two staging slots: batch b+1's upload and
    batch b-1's download overlap batch b's layer.  Every batch must equal
    moe_forward on its own x bit for bit (a slot reused before its previous
    batch's download or layer finished would show here), and the call twice on
    the same workspace must order itself after the first."""
    d = 1024
    inp = make_inputs(T, d, 512, 8, 2, seed=61, bias=True)
    dev = to_dev(inp)
    shape = inp["shape"]
    args = (dev["Wg"], dev["bias"], dev["W1"], dev["W3"], dev["W2"])
    g = torch.Generator().manual_seed(62)
    xs = [(inp["x"].float() * (1.0 + 0.25 * b) +
           0.1 * torch.randn(T, d, generator=g)).to(torch.bfloat16) for b in range(n)]
    refs = [moe.moe_forward(shape, x.cuda(), *args).cpu() for x in xs]
    xs_host = [x.pin_memory() for x in xs]
    ys_host = [torch.full((T, d), 5.0, dtype=torch.bfloat16).pin_memory() for _ in range(n)]
    ws = moe.workspace(moe.moe_forward_hostio_batches_workspace_bytes(shape), "cuda")
    for _ in range(2):
        moe.moe_forward_hostio_batches(shape, xs_host, *args, ys_host, ws)
    torch.cuda.synchronize()
    for b in range(n):
        assert torch.equal(ys_host[b], refs[b]), f"batch {b}"
    assert moe.moe_read_device_status(ws) == moe.MOE_OK


@pytest.mark.parametrize("stall_batch", [0, 1, 2], ids=["first", "middle", "last"])
def test_hostio_batches_report_a_timeout_in_any_batch(stall_batch):
    """A queue of three batches on one workspace; the status word is cleared
    once, before the first, so an expired wait in any batch must still read
    MOE_ERR_DEVICE_TIMEOUT after the call, the other batches must be right, and a
    normal call afterwards on the same workspace must report MOE_OK."""
    T, d = 600, 256
    inp = make_inputs(T, d, 256, 8, 2, seed=47, bias=True)
    dev = to_dev(inp)
    shape = inp["shape"]
    args = (dev["Wg"], dev["bias"], dev["W1"], dev["W3"], dev["W2"])
    g = torch.Generator().manual_seed(48)
    xs = [(inp["x"].float() + 0.3 * b * torch.randn(T, d, generator=g)).to(torch.bfloat16)
          for b in range(3)]
    refs = [moe.moe_forward(shape, x.cuda(), *args).cpu() for x in xs]
    xs_host = [x.pin_memory() for x in xs]
    ys_host = [torch.zeros(T, d, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    ws = moe.workspace(moe.moe_forward_hostio_batches_workspace_bytes(shape), "cuda")
    moe.moe_forward_hostio_batches_stall_test(shape, xs_host, *args, ys_host, ws,
                                              stall_batch=stall_batch, stall_after=1,
                                              timeout_ns=2_000_000)
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    for b in range(3):
        if b != stall_batch:
            assert torch.equal(ys_host[b], refs[b]), f"batch {b}"
    moe.moe_forward_hostio_batches(shape, xs_host, *args, ys_host, ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    for b in range(3):
        assert torch.equal(ys_host[b], refs[b]), f"batch {b} after the normal call"


@pytest.mark.parametrize("T,stall_chunk", [(2048, 0), (2048, 1), (2048, 2), (300, 0)],
                         ids=["first-of-three-chunks", "middle-chunk", "last-chunk", "one-chunk"])
def test_hostio_reports_a_timeout_in_any_chunk(T, stall_chunk):
    """The host-I/O pipeline runs large batches as token chunks on one
    workspace; a wait that expires in an earlier chunk must not be cleared by a
    later one.  The stalled chunk's producer stops after one stage (2 ms bound):
    the status must read MOE_ERR_DEVICE_TIMEOUT, and a normal call afterwards on
    the same workspace must be correct and report MOE_OK."""
    inp = make_inputs(T, 256, 256, 8, 2, seed=45, bias=True)
    dev = to_dev(inp)
    shape = inp["shape"]
    args = (dev["Wg"], dev["bias"], dev["W1"], dev["W3"], dev["W2"])
    x_host = inp["x"].clone().pin_memory()
    y_host = torch.zeros(T, 256, dtype=torch.bfloat16).pin_memory()
    ws = moe.workspace(moe.moe_forward_hostio_workspace_bytes(shape), "cuda")
    moe.moe_forward_hostio_stall_test(shape, x_host, *args, y_host, ws, stall_chunk=stall_chunk,
                                      stall_after=1, timeout_ns=2_000_000)
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    moe.moe_forward_hostio(shape, x_host, *args, y_host, ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    y_dev = moe.moe_forward(shape, dev["x"], *args)
    torch.cuda.synchronize()
    assert torch.equal(y_dev.cpu(), y_host)


@pytest.mark.parametrize("T", [8, 64, 300], ids=["tiny-batch", "single-cta", "cta-pair"])
def test_bounded_wait_reports_timeout_and_context_survives(T):
    inp = make_inputs(T, 128, 256, 8, 2, seed=44)
    T, d, d_ff, E, k = inp["shape"]
    o_idx, _, _ = oracle.route(inp["x"], inp["Wg"], E, k)
    r_off, r_perm, _ = oracle.dispatch(o_idx, E)
    xs = torch.from_numpy(oracle.gather(inp["x"], r_perm).view(np.int16)).view(torch.bfloat16).cuda()
    dev = to_dev(inp)
    off = torch.from_numpy(r_off).cuda()
    _, _, ws = moe.moe_expert_swiglu_stall_test(inp["shape"], xs, off, dev["W1"], dev["W3"],
                                                dev["W2"], stall_after=1, timeout_ns=2_000_000)
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    # the context is still usable and the next call clears the status word
    h, o, ws = moe.moe_expert_swiglu(inp["shape"], xs, off, dev["W1"], dev["W3"], dev["W2"], ws=ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    xs_np = oracle.gather(inp["x"], r_perm)
    h_ref, o_ref = oracle.expert(xs_np, r_off, inp["W1"], inp["W3"], inp["W2"])
    row_expert = np.searchsorted(r_off, np.arange(T * k), side="right") - 1
    check_expert_rows(bf16_values(h), o.cpu().numpy().astype(np.float64), oracle.bf16_to_f64(xs_np),
                      row_expert, inp["W1"], inp["W3"], inp["W2"], h_ref, o_ref)


def test_host_checks_launch_nothing():
    inp = workload_inputs("tiny")
    dev = to_dev(inp)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_route((64, 128, 256, 8, 9), dev["x"], torch.empty(128, 8, dtype=torch.bfloat16,
                                                                  device="cuda"))
    assert e.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError) as e:
        moe.moe_forward(inp["shape"], dev["x"], dev["Wg"], None, dev["W1"], dev["W3"], dev["W2"],
                        ws=moe.workspace(1024, "cuda"))
    assert e.value.status == moe.MOE_ERR_WORKSPACE
