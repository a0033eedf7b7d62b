"""The combine fused into the down projection's epilogue, bit for bit.

When a routed batch gives the down projection (on CTA pairs, 256-row and
256-column tiles, d a multiple of 256) at least 4 rounds of pair tiles on the
device's SMs, that GEMM forms y itself: the last of a token's k row tiles to
store its o rows adds the token's gate-weighted rows up.  That y must have
exactly the bits of the separate path (dispatch, experts, combine through
their own entry points), and of a float32 model of the combine's arithmetic
written here in numpy: products rounded to float32, summed in slot order, the
block's residual added last, one rounding to bf16 (nearest even).  The cases
below have 1184 or more pair tiles (16 rounds of 74 pairs on 148 SMs, well past
the 4 from which the down projection forms y) unless
marked otherwise.
"""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_05_b200 as moe
from sparse_mixture_experts_05_b200.inputs import make_inputs

from _parity import to_dev, u16

pytestmark = pytest.mark.gpu

CASES = {
    # name: (T, d, d_ff, E, k, seed, bias)
    "k1": (19200, 4096, 256, 8, 1, 31, False),
    "k2": (9600, 4096, 256, 8, 2, 32, True),
    "k2-d768": (50600, 768, 256, 8, 2, 33, False),     # 3 column tiles of 256
    "k2-d2048": (19000, 2048, 256, 8, 2, 34, False),
    "E5k3": (6400, 4096, 256, 5, 3, 35, False),
    "E16k4": (4800, 4096, 256, 16, 4, 36, False),
    "E32k8": (4800, 2048, 256, 32, 8, 37, False),      # the largest E and k (and d for E = 32)
    "E1k1": (19044, 4096, 256, 1, 1, 38, False),       # 74 full pair tiles and a half tile
    # not fused: d not a multiple of 256, fewer than 512 rows, under 4 rounds
    "d384": (1400, 384, 256, 8, 2, 39, False),
    "small": (200, 256, 256, 8, 2, 40, False),
    "rounds": (1024, 1024, 256, 8, 2, 41, False),      # the quarter-width batch: 32 tiles
}


def _round_bf16(a32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits, round to nearest even (finite inputs)."""
    u = a32.astype(np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def _combine_model(o32, inv, gate, residual_bits=None):
    acc = None
    for s in range(inv.shape[1]):
        p = gate[:, s:s + 1].astype(np.float32) * o32[inv[:, s]]
        acc = p if acc is None else acc + p
    if residual_bits is not None:
        res = (residual_bits.astype(np.uint32) << 16).view(np.float32)
        acc = res + acc
    return _round_bf16(acc)


def _split_path(shape, x, idx, gate, dev):
    """dispatch -> experts -> combine, each through its own entry point."""
    offsets, perm, inv, xs = moe.moe_dispatch(shape, idx, x)
    _, o, _ = moe.moe_expert_swiglu(shape, xs, offsets, dev["W1"], dev["W3"], dev["W2"])
    y = moe.moe_combine(shape, o, inv, gate)
    return y, o, inv


@pytest.mark.parametrize("name", list(CASES))
def test_fused_combine_equals_the_separate_path(name):
    T, d, d_ff, E, k, seed, bias = CASES[name]
    inp = make_inputs(T, d, d_ff, E, k, seed, bias=bias)
    shape = inp["shape"]
    dev = to_dev(inp)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    ws = moe.workspace(moe.moe_forward_workspace_bytes(shape), "cuda")
    # twice on one workspace: the counters are zeroed again for the second call
    for _ in range(2):
        y = moe.moe_forward(shape, dev["x"], dev["Wg"], dev["bias"], dev["W1"], dev["W3"],
                            dev["W2"], idx_out=idx, gate_out=gate, ws=ws)
        torch.cuda.synchronize()
        assert moe.moe_read_device_status(ws) == moe.MOE_OK
        y_split, o, inv = _split_path(shape, dev["x"], idx, gate, dev)
        torch.cuda.synchronize()
        assert torch.equal(y, y_split)
    model = _combine_model(o.cpu().numpy(), inv.cpu().numpy(), gate.cpu().numpy())
    assert np.array_equal(u16(y), model)


@pytest.mark.parametrize("name", ["k2", "E16k4", "d384"])
def test_fused_combine_adds_the_block_residual(name):
    """H = U + MoE(u) with u = RMSNorm(U): H against the float32 model on the
    separate path's rows, routed from the u the block left in its workspace."""
    T, d, d_ff, E, k, seed, bias = CASES[name]
    inp = make_inputs(T, d, d_ff, E, k, seed, bias=bias)
    shape = inp["shape"]
    dev = to_dev(inp)
    rng = np.random.default_rng(seed)
    gamma = torch.from_numpy((1 + 0.2 * rng.standard_normal(d)).astype(np.float32))
    gamma = gamma.to(torch.bfloat16).cuda()
    ws = moe.workspace(moe.moe_block_workspace_bytes(shape), "cuda")
    H = moe.moe_block_forward(shape, dev["x"], gamma, dev["Wg"], dev["bias"], dev["W1"],
                              dev["W3"], dev["W2"], eps=1e-5, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    off = moe.moe_forward_workspace_bytes(shape)
    u = ws[off:off + T * d * 2].view(torch.bfloat16).view(T, d).clone()
    idx, gate = moe.moe_route(shape, u, dev["Wg"], dev["bias"])[:2]
    _, o, inv = _split_path(shape, u, idx, gate, dev)
    torch.cuda.synchronize()
    model = _combine_model(o.cpu().numpy(), inv.cpu().numpy(), gate.cpu().numpy(),
                           residual_bits=u16(inp["x"]))
    assert np.array_equal(u16(H), model)


def _our_kernels(fn):
    """Names of this library's kernels (namespace moe) that `fn` launches, from the
    profiler's CUDA activity."""
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    names = [e.name for e in prof.events()]
    if not names:
        pytest.skip("the profiler recorded no CUDA activity")
    return [n for n in names if "moe::" in n]


@pytest.mark.parametrize("name", ["k2", "rounds", "small"])
def test_forward_kernel_count_matches_the_launches(name):
    """moe_forward_kernel_count: 5 kernels where the down projection forms y
    itself, 6 elsewhere, and no combine kernel among the 5."""
    T, d, d_ff, E, k, seed, bias = CASES[name]
    inp = make_inputs(T, d, d_ff, E, k, seed, bias=bias)
    shape = inp["shape"]
    dev = to_dev(inp)
    ws = moe.workspace(moe.moe_forward_workspace_bytes(shape), "cuda")
    run = lambda: moe.moe_forward(shape, dev["x"], dev["Wg"], dev["bias"], dev["W1"],  # noqa: E731
                                  dev["W3"], dev["W2"], ws=ws)
    run()
    kernels = _our_kernels(run)
    n = moe.moe_forward_kernel_count(shape)
    assert len(kernels) == n, kernels
    assert (n == 5) == (name == "k2")
    assert any("combine_kernel" in s for s in kernels) == (n == 6)


@pytest.mark.parametrize("stall_after", [0, 40], ids=["at-once", "after-some-tiles"])
def test_fused_combine_timeout_in_a_queue_of_batches(stall_after):
    """The error path with the combine inside GEMM2: in the middle batch of a
    queue the expert producers stop (at once, or after 40 stages: GEMM1 stalls in
    its first tiles, GEMM2 after about ten, some tokens' counters already
    counted).  The call must report MOE_ERR_DEVICE_TIMEOUT, the other batches'
    y must be exact, and a normal call on the same workspace afterwards (which
    zeroes the counters again) must be exact and report MOE_OK."""
    T, d, d_ff, E, k, seed, bias = CASES["k2"]
    inp = make_inputs(T, d, d_ff, E, k, seed, bias=bias)
    shape = inp["shape"]
    assert moe.moe_forward_kernel_count(shape) == 5
    dev = to_dev(inp)
    args = (dev["Wg"], dev["bias"], dev["W1"], dev["W3"], dev["W2"])
    g = torch.Generator().manual_seed(57)
    xs = [(inp["x"].float() + 0.3 * b * torch.randn(T, d, generator=g)).to(torch.bfloat16)
          for b in range(3)]
    refs = [moe.moe_forward(shape, x.cuda(), *args).cpu() for x in xs]
    xs_host = [x.pin_memory() for x in xs]
    ys_host = [torch.zeros(T, d, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    ws = moe.workspace(moe.moe_forward_hostio_batches_workspace_bytes(shape), "cuda")
    moe.moe_forward_hostio_batches_stall_test(shape, xs_host, *args, ys_host, ws, stall_batch=1,
                                              stall_after=stall_after, timeout_ns=2_000_000)
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    for b in (0, 2):
        assert torch.equal(ys_host[b], refs[b]), f"batch {b}"
    moe.moe_forward_hostio_batches(shape, xs_host, *args, ys_host, ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    for b in range(3):
        assert torch.equal(ys_host[b], refs[b]), f"batch {b} after the normal call"


def test_fused_combine_with_expert_biases():
    """The layer with expert Linear biases (b2 added to o in GEMM2's epilogue
    before the fused combine reads it): y equals the separate path with the
    same biases, and the float32 model, bit for bit."""
    from sparse_mixture_experts_05_b200.inputs import expert_biases
    T, d, d_ff, E, k, seed, bias = CASES["k2"]
    inp = make_inputs(T, d, d_ff, E, k, seed, bias=bias)
    shape = inp["shape"]
    assert moe.moe_forward_kernel_count(shape) == 5
    dev = to_dev(inp)
    eb = tuple(b.cuda() for b in expert_biases(E, d, d_ff, seed=77))
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    y = moe.moe_forward_bias(shape, dev["x"], dev["Wg"], dev["bias"], dev["W1"], dev["W3"],
                             dev["W2"], eb, idx_out=idx, gate_out=gate)
    offsets, perm, inv, xs = moe.moe_dispatch(shape, idx, dev["x"])
    _, o, _ = moe.moe_expert_swiglu_bias(shape, xs, offsets, dev["W1"], dev["W3"], dev["W2"], eb)
    y_split = moe.moe_combine(shape, o, inv, gate)
    torch.cuda.synchronize()
    assert torch.equal(y, y_split)
    model = _combine_model(o.cpu().numpy(), inv.cpu().numpy(), gate.cpu().numpy())
    assert np.array_equal(u16(y), model)


def test_fused_combine_in_token_chunks_equals_the_whole_batch():
    """moe_forward_hostio cuts a batch of 18000 tokens into chunks of 2240, 13520
    and 2240 tokens: the middle chunk (1680 pair tiles) forms y inside GEMM2, the
    edge chunks (272 pair tiles each, under 4 rounds) run the combine kernel, and
    the whole batch (2240 tiles) is fused too; y must be the same bits either way."""
    T, d, d_ff, E, k = 18000, 4096, 256, 8, 2
    inp = make_inputs(T, d, d_ff, E, k, 42, bias=True)
    shape = inp["shape"]
    assert moe.moe_forward_kernel_count(shape) == 5
    assert moe.moe_forward_kernel_count((13520, d, d_ff, E, k)) == 5
    assert moe.moe_forward_kernel_count((2240, d, d_ff, E, k)) == 6
    dev = to_dev(inp)
    y = moe.moe_forward(shape, dev["x"], dev["Wg"], dev["bias"], dev["W1"], dev["W3"], dev["W2"])
    x_host = inp["x"].clone().pin_memory()
    y_host = torch.empty(T, d, dtype=torch.bfloat16).pin_memory()
    ws = moe.workspace(moe.moe_forward_hostio_workspace_bytes(shape), "cuda")
    moe.moe_forward_hostio(shape, x_host, dev["Wg"], dev["bias"], dev["W1"], dev["W3"], dev["W2"],
                           y_host, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    assert torch.equal(y.cpu(), y_host)
