"""Seeded synthetic inputs for the MoE layer.

This module only draws random numbers and rounds them to bf16; it holds none of
the layer's arithmetic.  It is the one module shared by the CUDA path's tests and
benchmark and by the oracle's tests.

Recipe (one per workload, Mixtral 8x7B shapes from the Mixtral textbook page,
section "Научный вклад": d = 4096, d_ff = 14336, E = 8, k = 2):
  x  [T, d]        ~ N(0, 1)
  Wg [d, E]        ~ N(0, 1/d)
  W1, W3 [E, d, d_ff] ~ N(0, 1/d)     (gate and up projections)
  W2 [E, d_ff, d]  ~ N(0, 1/d_ff)     (down projection)
all rounded to bf16 (round to nearest even), drawn in that order from
torch.Generator("cpu").manual_seed(seed) -- or, for the benchmark's device-side
generation, from a CUDA generator with the same seed (same distribution, other
stream of numbers).  The "skew" workload adds a fixed router bias
b_e = 1.5 (E-1-e)/(E-1) (float32) so that low-numbered experts receive more
tokens, mimicking the uneven expert load the NVIDIA blog page reports in
"Experimenting with the Mixtral model / Load balancing".
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    d_ff: int
    E: int
    k: int
    seed: int
    skew_bias: bool = False

    @property
    def R(self) -> int:
        return self.T * self.k


WORKLOADS = {
    "tiny": Workload("tiny", T=64, d=128, d_ff=256, E=8, k=2, seed=0),
    "quarter": Workload("quarter", T=1024, d=1024, d_ff=3584, E=8, k=2, seed=1),
    "prefill": Workload("prefill", T=4096, d=4096, d_ff=14336, E=8, k=2, seed=2),
    "decode": Workload("decode", T=16, d=4096, d_ff=14336, E=8, k=2, seed=3),
    "skew": Workload("skew", T=16384, d=4096, d_ff=14336, E=8, k=2, seed=4, skew_bias=True),
}


def skew_bias(E: int) -> torch.Tensor:
    """b_e = 1.5 (E-1-e)/(E-1), float32 (all zero when E == 1)."""
    if E == 1:
        return torch.zeros(1, dtype=torch.float32)
    return torch.tensor([1.5 * (E - 1 - e) / (E - 1) for e in range(E)], dtype=torch.float32)


def _randn(shape, std, gen, device):
    t = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def make_inputs(T: int, d: int, d_ff: int, E: int, k: int, seed: int, bias: bool = False,
                device: str = "cpu") -> dict:
    """Draw x, Wg, W1, W3, W2 (bf16) and the optional router bias (float32).

    `k` is not used for drawing; it is carried along so a dict fully describes a
    case.  Returns tensors on `device`.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = {
        "x": _randn((T, d), 1.0, gen, device),
        "Wg": _randn((d, E), 1.0 / math.sqrt(d), gen, device),
        "W1": _randn((E, d, d_ff), 1.0 / math.sqrt(d), gen, device),
        "W3": _randn((E, d, d_ff), 1.0 / math.sqrt(d), gen, device),
        "W2": _randn((E, d_ff, d), 1.0 / math.sqrt(d_ff), gen, device),
        "bias": skew_bias(E).to(device) if bias else None,
        "shape": (T, d, d_ff, E, k),
    }
    return out


def expert_biases(E: int, d: int, d_ff: int, seed: int, device: str = "cpu"):
    """Biases of the three expert Linear layers for the layer built with bias
    (the teaching configuration of the Mixtral page's section "Подсчёт
    параметров"): b1, b3 [E, d_ff] ~ U(-1/sqrt(d), 1/sqrt(d)) and b2 [E, d] ~
    U(-1/sqrt(d_ff), 1/sqrt(d_ff)) (the usual Linear initialisation), rounded to
    bf16 values and held as float32.  Drawn from their own generator, seeded
    with `seed`, in the order b1, b3, b2."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)

    def uni(shape, bound):
        t = torch.rand(*shape, generator=gen, device=device, dtype=torch.float32)
        return (t * (2 * bound) - bound).to(torch.bfloat16).to(torch.float32)

    return (uni((E, d_ff), 1.0 / math.sqrt(d)), uni((E, d_ff), 1.0 / math.sqrt(d)),
            uni((E, d), 1.0 / math.sqrt(d_ff)))


def workload_inputs(name: str, device: str = "cpu", T: int | None = None) -> dict:
    """Inputs of a named workload; `T` overrides the token count (same seed)."""
    w = WORKLOADS[name]
    return make_inputs(T if T is not None else w.T, w.d, w.d_ff, w.E, w.k, w.seed,
                       bias=w.skew_bias, device=device)


def identical_experts(inp: dict) -> dict:
    """Copy of `inp` whose E experts all carry expert 0's weights."""
    out = dict(inp)
    for key in ("W1", "W3", "W2"):
        w = inp[key]
        out[key] = w[:1].expand_as(w).contiguous()
    return out
