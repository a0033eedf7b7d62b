"""CPU stand-in for the per-rank compute of the expert-parallel layer: the
oracle's route / dispatch / expert / combine on torch CPU tensors, so that the
all-to-all bookkeeping can run on gloo ranks without a GPU."""
import numpy as np
import torch

import oracle


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class OracleOps:
    o_dtype = torch.float64

    def route(self, shape, x, Wg, bias):
        T, d, d_ff, E, k = shape
        idx, gate, _ = oracle.route(_u16(x), _u16(Wg), E, k, bias=bias)
        return torch.from_numpy(idx), torch.from_numpy(gate)

    def dispatch(self, shape, idx, x):
        T, d, d_ff, E, k = shape
        off, perm, inv = oracle.dispatch(idx.numpy(), E)
        xs = oracle.gather(_u16(x), perm)
        return (torch.from_numpy(off), torch.from_numpy(inv),
                torch.from_numpy(xs.view(np.int16)).view(torch.bfloat16))

    def expert(self, rows, offsets, W1, W3, W2, out):
        _, o = oracle.expert(_u16(rows), offsets.numpy(), _u16(W1), _u16(W3), _u16(W2))
        out.copy_(torch.from_numpy(o))

    def combine(self, shape, o, inv, gate):
        return torch.from_numpy(oracle.combine(o.numpy(), inv.numpy(), gate.numpy()))
