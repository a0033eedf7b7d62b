"""The expert-parallel forward on the GPU with the library's kernels and NCCL,
at world size 1 (every expert local; the exchanges are copies through NCCL):
it must reproduce moe_forward bit for bit.  Multi-rank exchanges are covered
by the gloo tests in test_multirank_expert_parallel.py."""
import socket

import pytest
import torch
import torch.distributed as dist

import sparse_mixture_experts_05_b200 as moe
from sparse_mixture_experts_05_b200.expert_parallel import ep_forward
from sparse_mixture_experts_05_b200.inputs import make_inputs, workload_inputs

from _parity import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda:0"))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("name", ["tiny", "quarter", "bias"])
def test_ep_forward_world1_equals_moe_forward(nccl_group, name):
    inp = make_inputs(300, 256, 384, 8, 2, seed=70, bias=True) if name == "bias" else workload_inputs(name)
    dev = to_dev(inp)
    args = (dev["x"], dev["Wg"], dev["bias"], dev["W1"], dev["W3"], dev["W2"])
    y_ref = moe.moe_forward(inp["shape"], *args)
    y = ep_forward(inp["shape"], *args)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
