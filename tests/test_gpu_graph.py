"""The layer inside a captured CUDA graph.

The entry points launch only kernels, memsets and device-to-device copies on the
caller's stream and allocate nothing, so a forward can be captured once and
replayed: each replay must equal an eager call on the same inputs, bit for bit.
"""
import pytest
import torch

import sparse_mixture_experts_05_b200 as moe
from sparse_mixture_experts_05_b200.inputs import make_inputs

from _parity import to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,d,d_ff", [(64, 128, 256), (700, 256, 512), (2600, 1024, 256)],
                         ids=["single-cta", "cta-pair", "streaming-router"])
def test_forward_replays_in_a_cuda_graph(T, d, d_ff):
    inp = make_inputs(T, d, d_ff, 8, 2, seed=70, bias=True)
    shape = inp["shape"]
    dev = to_dev(inp)
    ws = moe.workspace(moe.moe_forward_workspace_bytes(shape), "cuda")
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    x_static = dev["x"].clone()
    args = (dev["Wg"], dev["bias"], dev["W1"], dev["W3"], dev["W2"])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up: one-time attribute and address set-up
        moe.moe_forward(shape, x_static, *args, y=y, ws=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        moe.moe_forward(shape, x_static, *args, y=y, ws=ws)

    for seed in (71, 72):
        x_new = make_inputs(T, d, d_ff, 8, 2, seed=seed)["x"].cuda()
        x_static.copy_(x_new)
        graph.replay()
        torch.cuda.synchronize()
        y_eager = moe.moe_forward(shape, x_new, *args)
        torch.cuda.synchronize()
        assert torch.equal(y, y_eager)
        assert moe.moe_read_device_status(ws) == moe.MOE_OK


def test_static_scratch_forward_replays_in_a_cuda_graph():
    T, d, d_ff = 16, 256, 512
    inp = make_inputs(T, d, d_ff, 8, 2, seed=73)
    shape = inp["shape"]
    dev = to_dev(inp)
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    x_static = dev["x"].clone()
    args = (dev["Wg"], None, dev["W1"], dev["W3"], dev["W2"])
    moe.moe_forward_static(shape, x_static, *args, y=y)  # first call: scratch address lookup
    torch.cuda.synchronize()

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        moe.moe_forward_static(shape, x_static, *args, y=y)

    x_new = make_inputs(T, d, d_ff, 8, 2, seed=74)["x"].cuda()
    x_static.copy_(x_new)
    graph.replay()
    torch.cuda.synchronize()
    y_eager = moe.moe_forward(shape, x_new, *args)
    torch.cuda.synchronize()
    assert torch.equal(y, y_eager)
