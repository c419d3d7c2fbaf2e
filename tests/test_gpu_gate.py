"""GPU parity of the gated linear branch (sla_forward_gated / sla_backward_gated)
against the fp64 oracle with the same gate, through the C ABI."""

import math

import numpy as np
import pytest

import oracle
import sla_inputs
from sla_harness import Run, assert_close, to_dev

pytestmark = pytest.mark.gpu


def _grid(name, grid, H, k_h, k_l, n_tokens=None):
    return sla_inputs.make_grid(grid, H=H, k_h=k_h, k_l=k_l, name=name, n_tokens=n_tokens,
                                with_grad=True)


WORKLOADS = {
    "tiny": lambda: sla_inputs.make("tiny", with_grad=True),
    "mid": lambda: sla_inputs.make("mid", with_grad=True),
    "wan_slice_2048": lambda: _grid("wan_slice", (21, 30, 52), 12, 0.05, 0.10, n_tokens=2048),
    "odd_T_7": lambda: _grid("odd", (3, 7, 21), 3, 0.25, 0.25),
}


def run_gated(wl, logit, skip_below):
    import torch
    run = Run(wl)
    slab = run.slab
    gate = slab.Gate(logit, skip_below)
    run.classify()
    slab.sla_forward_gated(run.shape, run.q, run.k, run.v, run.w, run.buf.mask, gate, run.o,
                           run.buf.saved, run.buf.workspace)
    run.check()
    do = to_dev(wl.d_o, torch.bfloat16)
    grads = {n: torch.empty(run.q.shape, dtype=torch.float32, device="cuda")
             for n in ("dq", "dk", "dv")}
    grads["dw"] = torch.empty(run.w.shape, dtype=torch.float32, device="cuda")
    d_logit = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    slab.sla_backward_gated(run.shape, run.q, run.k, run.v, run.w, run.buf.mask, gate,
                            run.buf.saved, do, grads["dq"], grads["dk"], grads["dv"],
                            grads["dw"], d_logit, run.buf.workspace)
    run.check()
    return run, grads, float(d_logit.item())


def oracle_gated(wl, cls, gate):
    fwd = oracle.forward(wl.q, wl.k, wl.v, wl.w_proj, cls, wl.block, wl.scale, gate=gate)
    g = oracle.backward(wl.q, wl.k, wl.v, wl.w_proj, cls, wl.d_o, wl.block, wl.scale, fwd=fwd,
                        gate=gate)
    return fwd, g


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_gated_parity(name):
    wl = WORKLOADS[name]()
    gate = (0.4, 0.05)
    run, grads, d_logit = run_gated(wl, *gate)
    fwd, g = oracle_gated(wl, run.cls(), gate)
    assert_close(run.np(run.o), fwd["o"], "o")
    for n in ("dq", "dk", "dv", "dw"):
        assert_close(run.np(grads[n]), g[n], n)
    # d logit: a sum over every token and feature; judged against the size of
    # its terms, g (1 - g) * sum |(O_l W) * dO|
    gf = fwd["g"]
    terms = np.abs(np.einsum("bhta,ac->bhtc", fwd["o_l"], wl.w_proj) * wl.d_o).sum()
    assert abs(d_logit - g["d_gamma"]) <= 3e-3 * gf * (1 - gf) * terms, (d_logit, g["d_gamma"])


def test_dropped_gate_is_sparse_only():
    wl = WORKLOADS["mid"]()
    gate = (-4.0, 0.1)  # g = 0.018 < 0.1
    run, grads, d_logit = run_gated(wl, *gate)
    fwd, g = oracle_gated(wl, run.cls(), gate)
    np.testing.assert_array_equal(fwd["o"], fwd["o_s"])
    assert_close(run.np(run.o), fwd["o"], "o")
    for n in ("dq", "dk", "dv"):
        assert_close(run.np(grads[n]), g[n], n)
    assert np.all(run.np(grads["dw"]) == 0.0)
    assert d_logit == 0.0


def test_open_gate_equals_ungated():
    wl = WORKLOADS["tiny"]()
    run, grads, d_logit = run_gated(wl, math.inf, 0.5)  # g = 1 exactly
    ref = Run(wl)
    ref.classify()
    ref.forward()
    ref.backward(wl.d_o)
    np.testing.assert_array_equal(run.np(run.o), ref.np(ref.o))
    for n, t in (("dq", ref.dq), ("dk", ref.dk), ("dv", ref.dv), ("dw", ref.dw)):
        got, want = run.np(grads[n]), ref.np(t)
        # the same kernels and inputs; only the order of fp32 reductions may differ
        assert np.abs(got - want).max() <= 1e-5 * np.abs(want).max(), n
    assert d_logit == 0.0
