"""Expert parallelism (NVIDIA blog page, "Applying Mixture of Experts in LLM
Architectures": experts spread over GPUs with all-to-all exchanges): two and
four gloo ranks on CPU, each holding E/G experts and its own tokens, must give
exactly the single-process layer with all experts.  The per-rank compute is
the oracle (tests/_ep_ops.py), so what is checked is the exchange: counts,
split sizes, row order out and back."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(rank, T, seed):
    from sparse_mixture_experts_05_b200.inputs import make_inputs
    weights = make_inputs(8, 64, 128, 8, 2, seed=100, bias=True)        # same model on every rank
    tokens = make_inputs(T, 64, 128, 8, 2, seed=seed + rank)           # each rank its own batch
    return weights, tokens


def _rank_main(rank, world, port, T, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import torch.distributed as dist

    import oracle
    from sparse_mixture_experts_05_b200.expert_parallel import ep_forward
    from _ep_ops import OracleOps
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, t = _case(rank, T, 7)
        E = 8
        El = E // world
        sl = slice(rank * El, (rank + 1) * El)
        y = ep_forward((T, 64, 128, E, 2), t["x"], w["Wg"], w["bias"], w["W1"][sl].contiguous(),
                       w["W3"][sl].contiguous(), w["W2"][sl].contiguous(), ops=OracleOps())
        y_ref, _, _ = oracle.forward(t["x"], w["Wg"], w["W1"], w["W3"], w["W2"], 2, bias=w["bias"])
        out[rank] = bool(np.array_equal(y.numpy(), y_ref))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world,T", [(2, 37), (4, 50), (2, 1)])
def test_expert_parallel_equals_single_process_layer(world, T):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, T, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(150)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        assert dict(out) == {r: True for r in range(world)}
