"""Expert-parallel MoE layer across ranks.

The NVIDIA blog page "Applying Mixture of Experts in LLM Architectures" names
expert parallelism with all-to-all exchanges as the way MoE layers are spread
over GPUs.  Here each of G ranks holds E/G consecutive experts (rank r owns
experts [r*E/G, (r+1)*E/G)) and its own batch of T tokens; the router weights
are replicated.  One forward runs in phases:

 1. route_and_dispatch: route the local tokens (top-k over all E experts,
    softmax over the k) and sort the local rows by expert, which also makes
    them contiguous per owning rank;
 2. exchange of the per-(rank, local expert) row counts, then of the rows;
 3. local_experts: every rank runs its own experts over the rows it received
    (one grouped call per source rank, the rows of each source already grouped
    by expert);
 4. exchange of the expert outputs back to the ranks that own the tokens,
    which receive them in their own sorted order;
 5. combine locally with the gates, exactly as the single-GPU layer does.

The exchanges go through an `exchange` object with one method,
all_to_all(out, inp, out_splits, in_splits), plus `world_size`;
DistExchange wraps torch.distributed all_to_all_single (NCCL over NVLink /
NVSwitch on GPUs).  The compute goes through an `ops` object: LibraryOps calls
the library's CUDA kernels through the C ABI; tests substitute a CPU
implementation to check the exchange on gloo ranks, or drive the phases of
several ranks from one process.  Split sizes travel to the host (NCCL needs them
there): one small device-to-host copy of the E+1 offsets per forward.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import binding


class LibraryOps:
    """Steps of the layer on the GPU through the C ABI (libmoe.so)."""

    o_dtype = torch.float32

    def route(self, shape, x, Wg, bias):
        idx, gate, _ = binding.moe_route(shape, x, Wg, bias)
        return idx, gate

    def dispatch(self, shape, idx, x):
        offsets, _, inv, x_sorted = binding.moe_dispatch(shape, idx, x)
        return offsets, inv, x_sorted

    def expert(self, rows, offsets, W1, W3, W2, out):
        """SwiGLU experts over `rows` [R, d] grouped by the local experts' offsets
        [E_l+1]; writes `out` [R, d]."""
        R, d = rows.shape
        E_l, _, d_ff = W1.shape
        shape = (R, d, d_ff, E_l, 1)  # R rows = R "tokens" with one slot each
        binding.moe_expert_swiglu(shape, rows.contiguous(), offsets, W1, W3, W2, o=out)

    def combine(self, shape, o, inv, gate):
        return binding.moe_combine(shape, o, inv, gate)


class DistExchange:
    """All-to-all over a torch.distributed process group."""

    def __init__(self, group=None):
        self.group = group
        self.world_size = dist.get_world_size(group)

    def all_to_all(self, out, inp, out_splits, in_splits):
        dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)
        return out


@dataclass
class Routed:
    """A rank's routing and sorted rows (phase 1)."""
    idx: torch.Tensor          # [T, k] expert ids
    gate: torch.Tensor         # [T, k] gates
    inv: torch.Tensor          # [T, k] sorted row of each (token, slot)
    x_sorted: torch.Tensor     # [T*k, d] rows sorted by expert
    send_counts: torch.Tensor  # [G, E_l] int64 (host): rows for each (owner rank, its local expert)


def route_and_dispatch(shape, x, Wg, bias, G, ops) -> Routed:
    """Phase 1: routing over all E experts and the expert-sorted local rows."""
    T, d, d_ff, E, k = shape
    if E % G:
        raise ValueError(f"E={E} experts do not split evenly over {G} ranks")
    idx, gate = ops.route(shape, x, Wg, bias)
    offsets, inv, x_sorted = ops.dispatch(shape, idx, x)
    off = offsets.to("cpu", torch.int64)
    send_counts = (off[1:] - off[:-1]).view(G, E // G)
    return Routed(idx, gate, inv, x_sorted, send_counts)


def local_experts(rows_in, recv_counts, W1_local, W3_local, W2_local, ops):
    """Phase 3: this rank's E_l experts over the rows received from each source
    rank (recv_counts [G, E_l], host), one grouped call per source block.
    Returns the outputs [rows, d] in the order the rows arrived."""
    E_l = W1_local.shape[0]
    d = rows_in.shape[1]
    o_in = torch.empty(rows_in.shape[0], d, dtype=ops.o_dtype, device=rows_in.device)
    start = 0
    for q in range(recv_counts.shape[0]):
        n = int(recv_counts[q].sum())
        if n:
            loc = torch.zeros(E_l + 1, dtype=torch.int32)
            loc[1:] = torch.cumsum(recv_counts[q], 0).to(torch.int32)
            ops.expert(rows_in[start:start + n], loc.to(rows_in.device), W1_local, W3_local,
                       W2_local, out=o_in[start:start + n])
        start += n
    return o_in


def ep_forward(shape, x, Wg, bias, W1_local, W3_local, W2_local, ops=None, group=None,
               exchange=None):
    """Expert-parallel forward of the local batch.

    shape = (T, d, d_ff, E, k) with E the global expert count; W1_local,
    W3_local [E/G, d, d_ff] and W2_local [E/G, d_ff, d] are this rank's experts.
    `exchange` defaults to DistExchange(group).  Returns y [T, d] for the local
    tokens.
    """
    ops = ops or LibraryOps()
    exchange = exchange or DistExchange(group)
    T, d, d_ff, E, k = shape
    G = exchange.world_size
    E_l = E // G if E % G == 0 else 0
    if W1_local.shape[0] != E_l or W2_local.shape[0] != E_l:
        raise ValueError(f"each of {G} ranks holds E/G experts of E={E}")

    rt = route_and_dispatch(shape, x, Wg, bias, G, ops)

    # counts of rows per (destination rank, its local expert), then the rows
    cdev = x.device if x.is_cuda else torch.device("cpu")
    rc = exchange.all_to_all(torch.empty(G * E_l, dtype=torch.int64, device=cdev),
                             rt.send_counts.reshape(-1).to(cdev), [E_l] * G, [E_l] * G)
    recv_counts = rc.view(G, E_l).to("cpu")
    send_rows = rt.send_counts.sum(1).tolist()
    recv_rows = recv_counts.sum(1).tolist()
    rows_in = torch.empty(sum(recv_rows), d, dtype=rt.x_sorted.dtype, device=rt.x_sorted.device)
    exchange.all_to_all(rows_in, rt.x_sorted.contiguous(), recv_rows, send_rows)

    o_in = local_experts(rows_in, recv_counts, W1_local, W3_local, W2_local, ops)

    # outputs back to the token owners, in their sorted order
    o = torch.empty(rt.x_sorted.shape[0], d, dtype=ops.o_dtype, device=rt.x_sorted.device)
    exchange.all_to_all(o, o_in, send_rows, recv_rows)
    return ops.combine(shape, o, rt.inv, rt.gate)
