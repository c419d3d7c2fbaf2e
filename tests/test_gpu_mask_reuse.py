"""Reusing a class map on new inputs (MC-Sparse page, key facts: query groups
and key/value indices are computed once and reused across denoising steps).

The mask is an explicit input of sla_forward / sla_backward: classify on one
set of inputs, then run the forward and backward on different inputs with that
mask, and compare element by element with the oracle given the same (stale)
class map."""

import numpy as np
import pytest

import oracle
import sla_inputs
from sla_harness import Run, assert_close, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,grid,H,k_h,k_l,n_tokens", [
    ("wan_slice", (21, 30, 52), 12, 0.05, 0.10, 2048),
    ("r37", (2, 37, 32), 2, 0.10, 0.20, None),
])
def test_mask_from_other_inputs(name, grid, H, k_h, k_l, n_tokens):
    import torch
    a = sla_inputs.make_grid(grid, H=H, k_h=k_h, k_l=k_l, name=name, n_tokens=n_tokens, seed=0)
    b = sla_inputs.make_grid(grid, H=H, k_h=k_h, k_l=k_l, name=name, n_tokens=n_tokens, seed=1,
                             with_grad=True)
    run = Run(a)
    run.classify()
    cls_a = run.cls()
    # inputs B through the same buffers, mask A kept
    run.q, run.k, run.v = (to_dev(x, torch.bfloat16) for x in (b.q, b.k, b.v))
    run.w = to_dev(b.w_proj, torch.bfloat16)
    run.forward()
    run.backward(b.d_o)
    # the mask really is stale: B's own classification differs
    lg_b = oracle.pooled_logits(b.q, b.k, b.block, b.scale)
    n_h, n_l = oracle.block_counts(b.T, b.k_h, b.k_l)
    assert not np.array_equal(oracle.classify(lg_b, n_h, n_l), cls_a)
    fwd = oracle.forward(b.q, b.k, b.v, b.w_proj, cls_a, b.block, b.scale)
    g = oracle.backward(b.q, b.k, b.v, b.w_proj, cls_a, b.d_o, b.block, b.scale, fwd=fwd)
    assert_close(run.np(run.o), fwd["o"], "o")
    for nm, t in (("dq", run.dq), ("dk", run.dk), ("dv", run.dv), ("dw", run.dw)):
        assert_close(run.np(t), g[nm], nm)
