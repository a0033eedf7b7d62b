"""Expert-parallel MoE layer across ranks.

The NVIDIA blog page "Applying Mixture of Experts in LLM Architectures" names
expert parallelism with all-to-all exchanges as the way MoE layers are spread
over GPUs.  Here each of G ranks holds E/G consecutive experts (rank r owns
experts [r*E/G, (r+1)*E/G)) and its own batch of T tokens; the router weights
are replicated.  One forward:

 1. route the local tokens (top-k over all E experts, softmax over the k);
 2. dispatch: local rows sorted by expert, hence contiguous per owning rank;
 3. all-to-all of the per-expert row counts, then of the rows themselves;
 4. every rank runs its own experts over the rows it received (one grouped
    call per source rank, the rows of each source already grouped by expert);
 5. all-to-all of the expert outputs back to the ranks that own the tokens,
    which receive them in their own sorted order;
 6. combine locally with the gates, exactly as the single-GPU layer does.

Communication uses torch.distributed all_to_all_single (NCCL over NVLink /
NVSwitch on GPUs).  The compute of steps 1, 2, 4 and 6 goes through an `ops`
object: LibraryOps calls the library's CUDA kernels; tests substitute a CPU
implementation to check the exchange on gloo ranks.  Split sizes travel to the
host (NCCL needs them there): one small device-to-host copy of the E+1 offsets
per forward.
"""
from __future__ import annotations

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


def _a2a(out, inp, out_splits, in_splits, group):
    dist.all_to_all_single(out, inp, out_splits, in_splits, group=group)
    return out


def ep_forward(shape, x, Wg, bias, W1_local, W3_local, W2_local, ops=None, group=None):
    """Expert-parallel forward of the local batch.

    shape = (T, d, d_ff, E, k) with E the global expert count; W1_local,
    W3_local [E/G, d, d_ff] and W2_local [E/G, d_ff, d] are this rank's experts.
    Returns y [T, d] for the local tokens.
    """
    ops = ops or LibraryOps()
    T, d, d_ff, E, k = shape
    G = dist.get_world_size(group)
    if E % G:
        raise ValueError(f"E={E} experts do not split evenly over {G} ranks")
    E_l = E // G
    if W1_local.shape[0] != E_l or W2_local.shape[0] != E_l:
        raise ValueError(f"each rank holds {E_l} experts")

    idx, gate = ops.route(shape, x, Wg, bias)
    offsets, inv, x_sorted = ops.dispatch(shape, idx, x)

    # counts of rows per (destination rank, its local expert), then their exchange
    off = offsets.to("cpu", torch.int64)
    send_counts = (off[1:] - off[:-1]).view(G, E_l)
    cdev = x.device if x.is_cuda else torch.device("cpu")
    rc = _a2a(torch.empty(G * E_l, dtype=torch.int64, device=cdev),
              send_counts.reshape(-1).to(cdev), [E_l] * G, [E_l] * G, group)
    recv_counts = rc.view(G, E_l).to("cpu")
    send_rows = send_counts.sum(1).tolist()
    recv_rows = recv_counts.sum(1).tolist()

    rows_in = torch.empty(sum(recv_rows), d, dtype=x_sorted.dtype, device=x_sorted.device)
    _a2a(rows_in, x_sorted.contiguous(), recv_rows, send_rows, group)

    # local experts over each source's rows (already grouped by expert)
    o_in = torch.empty(sum(recv_rows), d, dtype=ops.o_dtype, device=x_sorted.device)
    start = 0
    for q in range(G):
        n = recv_rows[q]
        if n:
            loc = torch.zeros(E_l + 1, dtype=torch.int32)
            loc[1:] = torch.cumsum(recv_counts[q], 0).to(torch.int32)
            ops.expert(rows_in[start:start + n], loc.to(x_sorted.device), W1_local, W3_local,
                       W2_local, out=o_in[start:start + n])
        start += n

    # outputs back to the token owners, in their sorted order
    o = torch.empty(x_sorted.shape[0], d, dtype=ops.o_dtype, device=x_sorted.device)
    _a2a(o, o_in, send_rows, recv_rows, group)
    return ops.combine(shape, o, inv, gate)
