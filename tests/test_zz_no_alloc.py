"""moe_forward_static: the layer for callers that cannot allocate device memory
(code running while a stream is captured into a CUDA graph, plugins whose host
framework owns every allocation, serving loops that must avoid cudaMalloc's
implicit synchronisation).  It runs on the library's fixed 8 MiB scratch array
instead of a caller workspace.

Checked through the C ABI against moe_forward (the entry point that takes a
workspace) on two calls in a row, so the second call runs on the scratch the
first one left behind.  Both entry points launch the same kernels with the same
shapes and splits, so y must agree bit for bit; the distance in units of the
parity tolerance (2e-2 * rms) is only reported in the failure message.  This
file is collected last on purpose; it must pass both on its own in a fresh
process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import sparse_mixture_experts_05_b200 as moe
from sparse_mixture_experts_05_b200.inputs import make_inputs

from _parity import Y_TOL, bf16_values, to_dev

pytestmark = pytest.mark.gpu

# (T, d, d_ff, E, k, seed, router bias): a decode-sized batch at quarter width, the
# tiny case, and the largest batch the scratch holds at the Mixtral 8x7B widths
SHAPES = [(16, 1024, 3584, 8, 2, 41, False), (64, 128, 256, 8, 2, 42, True),
          (78, 4096, 14336, 8, 2, 46, False)]


@pytest.mark.parametrize("case", SHAPES, ids=["decode-quarter", "tiny-bias", "mixtral-T78"])
def test_static_scratch_forward_matches_moe_forward(case):
    T, d, d_ff, E, k, seed, bias = case
    # both sides read the same device tensors, so they are drawn on the device
    inp = make_inputs(T, d, d_ff, E, k, seed, bias=bias, device="cuda")
    shape = inp["shape"]
    assert moe.moe_forward_workspace_bytes(shape) <= moe.binding.MOE_STATIC_SCRATCH_BYTES
    args = (shape, inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
    y_ref = moe.moe_forward(*args)
    ref = bf16_values(y_ref)
    rms = np.sqrt(np.mean(ref ** 2))
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        y = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        moe.moe_forward_static(*args, y=y, device_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        err = np.max(np.abs(bf16_values(y) - ref))
        assert torch.equal(y, y_ref), f"max|y - y_ref| = {err / rms / Y_TOL:.3g} x the parity bound"


def test_static_scratch_rejects_shapes_beyond_its_size():
    T, d, d_ff, E, k = 1024, 1024, 3584, 8, 2
    shape = (T, d, d_ff, E, k)
    assert moe.moe_forward_workspace_bytes(shape) > moe.binding.MOE_STATIC_SCRATCH_BYTES
    inp = to_dev(make_inputs(T, d, d_ff, E, k, 43))
    with pytest.raises(moe.MoeError) as e:
        moe.moe_forward_static(shape, inp["x"], inp["Wg"], None, inp["W1"], inp["W3"], inp["W2"])
    assert e.value.status == moe.MOE_ERR_WORKSPACE
