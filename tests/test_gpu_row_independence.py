"""An expert's rows computed alone give the same bits as inside the whole batch.

The grouped GEMMs accumulate every row in one fixed order whatever else is in
the batch: the tile a row lands in, the CTA pair that runs it and the number of
tiles do not change the result.  The whole batch below spreads over several
hundred down-projection tiles on every CTA pair; each expert alone runs a few
tiles.  The comparison is bitwise, expert by expert, plus the oracle on sampled
rows of every expert.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_05_b200 as moe
from sparse_mixture_experts_05_b200.inputs import make_inputs

from _parity import bf16_values, check_expert_rows

pytestmark = pytest.mark.gpu

# every expert >= 512 rows, so each expert alone also runs on CTA pairs (256-row tiles)
COUNTS = [700, 520, 1000, 513, 760, 530, 900, 600]


@pytest.mark.parametrize("d_ff", [256, 1024])
def test_expert_rows_alone_match_the_batch(d_ff):
    d, E = 2048, len(COUNTS)
    R = sum(COUNTS)
    inp = make_inputs(R, d, d_ff, E, 1, seed=80 + d_ff)
    xs = inp["x"].cuda()  # used directly as the expert-sorted rows
    W1, W3, W2 = (inp[key].cuda() for key in ("W1", "W3", "W2"))
    off = np.concatenate([[0], np.cumsum(COUNTS)]).astype(np.int32)

    h, o, ws = moe.moe_expert_swiglu((R, d, d_ff, E, 1), xs, torch.from_numpy(off).cuda(),
                                     W1, W3, W2)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK

    for e, c in enumerate(COUNTS):
        off_e = np.array([0] * (e + 1) + [c] * (E - e), dtype=np.int32)
        h_e, o_e, ws_e = moe.moe_expert_swiglu((c, d, d_ff, E, 1), xs[off[e]:off[e + 1]].clone(),
                                               torch.from_numpy(off_e).cuda(), W1, W3, W2)
        assert moe.moe_read_device_status(ws_e) == moe.MOE_OK
        assert torch.equal(h[off[e]:off[e + 1]], h_e), e
        assert torch.equal(o[off[e]:off[e + 1]], o_e), e

    # sampled rows of every expert against the oracle
    rng = np.random.default_rng(3)
    rows = np.concatenate([np.unique(np.r_[off[e], off[e + 1] - 1,
                                          rng.integers(off[e], off[e + 1], 3)])
                           for e in range(E)])
    row_expert = np.searchsorted(off, rows, side="right") - 1
    sub_off = np.searchsorted(row_expert, np.arange(E + 1), side="left").astype(np.int32)
    xs_rows = inp["x"][torch.from_numpy(rows)]
    h_ref, o_ref = oracle.expert(xs_rows, sub_off, inp["W1"], inp["W3"], inp["W2"])
    check_expert_rows(bf16_values(h[torch.from_numpy(rows).cuda()]),
                      o[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64),
                      oracle.bf16_to_f64(xs_rows), row_expert, inp["W1"], inp["W3"], inp["W2"],
                      h_ref, o_ref)


def test_rows_on_single_cta_tiles_match_the_cta_pair_batch():
    """Experts of fewer than 512 rows alone run the down projection on single-CTA
    128-row tiles; inside a batch of more than 512 rows they run on CTA pairs.
    The bits must not change with the kernel that runs them."""
    counts = [300, 130, 45, 400, 200, 1, 260, 90]
    d, d_ff, E = 1024, 512, len(counts)
    R = sum(counts)
    assert R >= 512 and max(counts) < 512
    inp = make_inputs(R, d, d_ff, E, 1, seed=85)
    xs = inp["x"].cuda()
    W1, W3, W2 = (inp[key].cuda() for key in ("W1", "W3", "W2"))
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    h, o, ws = moe.moe_expert_swiglu((R, d, d_ff, E, 1), xs, torch.from_numpy(off).cuda(),
                                     W1, W3, W2)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    for e, c in enumerate(counts):
        off_e = np.array([0] * (e + 1) + [c] * (E - e), dtype=np.int32)
        h_e, o_e, ws_e = moe.moe_expert_swiglu((c, d, d_ff, E, 1), xs[off[e]:off[e + 1]].clone(),
                                               torch.from_numpy(off_e).cuda(), W1, W3, W2)
        assert moe.moe_read_device_status(ws_e) == moe.MOE_OK
        assert torch.equal(h[off[e]:off[e + 1]], h_e), e
        assert torch.equal(o[off[e]:off[e + 1]], o_e), e
