"""The expert-parallel forward (NVIDIA blog page "Applying Mixture of Experts in
LLM Architectures": experts spread over GPUs, all-to-all exchanges) on the
library's CUDA kernels.

  * G = 2 and 4 ranks emulated in one process on one GPU: each virtual rank
    routes and dispatches its own tokens and runs its E/G local experts over the
    per-source blocks of rows it receives, through the package's phase
    functions and the C ABI; the exchanges are device copies done by the test,
    in the order the all-to-all would deliver them.  No kernel waits on
    another, so nothing here needs more than one GPU.  Each rank's y is checked
    against the oracle's single-process layer over that rank's tokens (the
    layer's parity rules), and bitwise against moe_forward over the same tokens
    (the grouped kernels give every row the same bits however the rows are
    grouped).
  * world size 1 through NCCL (every expert local, the exchanges are copies):
    against the oracle, and bitwise against moe_forward.
Multi-rank exchanges with real process groups are covered on CPU by
test_multirank_expert_parallel.py."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import sparse_mixture_experts_05_b200 as moe
from sparse_mixture_experts_05_b200.expert_parallel import (LibraryOps, ep_forward,
                                                            local_experts, route_and_dispatch)
from sparse_mixture_experts_05_b200.inputs import make_inputs, workload_inputs

from _parity import check_routing, check_y, to_dev

pytestmark = pytest.mark.gpu


def _check_against_oracle(y, x, w, k):
    """The layer's parity rules for y [T, d] (device) against the oracle's layer."""
    T = x.shape[0]
    E = w["W1"].shape[0]
    y_ref, o_idx, o_gate = oracle.forward(x, w["Wg"], w["W1"], w["W3"], w["W2"], k, bias=w["bias"])
    _, _, o_logits = oracle.route(x, w["Wg"], E, k, bias=w["bias"])
    kth_tie, _ = oracle.near_tie_flags(o_logits, k)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    return check_y(y, y_ref, rows=~kth_tie, rms_ref=rms)


def _emulated_ep(shapes, xs, w, G, ops):
    """Runs the expert-parallel phases of G ranks in lockstep in this process.
    shapes[r], xs[r]: rank r's shape and tokens; w: the full model (device)."""
    E = w["W1"].shape[0]
    E_l = E // G
    local_w = [tuple(w[n][r * E_l:(r + 1) * E_l].contiguous() for n in ("W1", "W3", "W2"))
               for r in range(G)]
    routed = [route_and_dispatch(shapes[r], xs[r], w["Wg"], w["bias"], G, ops) for r in range(G)]
    send_rows = [rt.send_counts.sum(1).tolist() for rt in routed]        # [src][dst]
    starts = [np.concatenate([[0], np.cumsum(s)]).astype(int) for s in send_rows]
    outs_in = []
    for r in range(G):  # rank r receives from every source q, in source order
        recv_counts = torch.stack([routed[q].send_counts[r] for q in range(G)])
        rows_in = torch.cat([routed[q].x_sorted[starts[q][r]:starts[q][r + 1]] for q in range(G)])
        outs_in.append((local_experts(rows_in, recv_counts, *local_w[r], ops),
                        [send_rows[q][r] for q in range(G)]))
    ys = []
    for q in range(G):  # source q gets its rows back from every owner r, owner order
        pieces = []
        for r in range(G):
            o_in, counts = outs_in[r]
            a = int(sum(counts[:q]))
            pieces.append(o_in[a:a + counts[q]])
        o = torch.cat(pieces)
        ys.append(ops.combine(shapes[q], o, routed[q].inv, routed[q].gate))
    return ys


@pytest.mark.parametrize("G,T,d,d_ff,E", [(2, 300, 256, 384, 8), (4, 257, 128, 256, 8),
                                          (4, 700, 256, 512, 16), (2, 1024, 1024, 3584, 8)],
                         ids=["G2", "G4", "G4-E16", "G2-quarter-width"])
def test_emulated_expert_parallel_matches_oracle_and_moe_forward(G, T, d, d_ff, E):
    k = 2
    w = make_inputs(8, d, d_ff, E, k, seed=90, bias=True)     # the same model on every rank
    toks = [make_inputs(T + 13 * r, d, d_ff, E, k, seed=91 + r)["x"] for r in range(G)]
    wd = to_dev(w)
    shapes = [(t.shape[0], d, d_ff, E, k) for t in toks]
    ys = _emulated_ep(shapes, [t.cuda() for t in toks], wd, G, LibraryOps())
    torch.cuda.synchronize()
    for r in range(G):
        rel, _ = _check_against_oracle(ys[r], toks[r], w, k)
        y_ref = moe.moe_forward(shapes[r], toks[r].cuda(), wd["Wg"], wd["bias"], wd["W1"],
                                wd["W3"], wd["W2"])
        torch.cuda.synchronize()
        assert torch.equal(ys[r], y_ref), f"rank {r}"
        print(f"rank {r}: max|y-y_ref|/rms {rel:.3g}")


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
def test_ep_forward_world1_matches_oracle_and_moe_forward(nccl_group, name):
    inp = make_inputs(300, 256, 384, 8, 2, seed=70, bias=True) if name == "bias" else workload_inputs(name)
    dev = to_dev(inp)
    args = (dev["x"], dev["Wg"], dev["bias"], dev["W1"], dev["W3"], dev["W2"])
    y = ep_forward(inp["shape"], *args)
    torch.cuda.synchronize()
    _check_against_oracle(y, inp["x"], inp, inp["shape"][4])
    y_ref = moe.moe_forward(inp["shape"], *args)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
