"""GPU parity of the hierarchical selection (sla_classify_hierarchical*)
against the fp64 oracle, through the C ABI.  The class map is compared
exactly on identical fp32 scores; the scores themselves within fp32 rounding."""

import numpy as np
import pytest

import oracle
import sla_inputs
from sla_harness import Run, assert_close, check_mask_outputs, to_dev

pytestmark = pytest.mark.gpu


def _scores_workload(B, H, T, fr, d=64):
    z = np.zeros((B, H, T * 64, d), np.float32)
    return sla_inputs.Workload("scores", B, H, T * 64, d, 64, fr[0], fr[1], T * 64, z, z, z,
                               np.zeros((d, d), np.float32))


@pytest.mark.parametrize("T,G,fr,extra", [
    (16, 2, (0.25, 0.25), (0, 0)),
    (37, 4, (0.10, 0.20), (0, 0)),
    (37, 4, (0.10, 0.20), (3, 1)),
    (128, 8, (0.05, 0.10), (0, 0)),
    (130, 16, (0.05, 0.10), (2, 2)),      # partial last super-block
    (64, 4, (0.0, 0.3), (0, 0)),          # no critical block
    (64, 4, (0.2, 0.0), (0, 0)),          # no negligible block
    (10, 4, (0.3, 0.3), (0, 0)),          # the lists meet: the flat selection
    (1182, 16, (0.10, 0.10), (0, 0)),     # long-sequence counts
])
def test_hierarchical_from_scores_bit_exact(T, G, fr, extra):
    import torch
    import sparse_linear_attention_block_b200 as slab
    B, H = 1, 3
    rng = np.random.default_rng(T * 31 + G)
    TG = -(-T // G)
    fine = rng.standard_normal((B, H, T, T)).astype(np.float32)
    coarse = rng.standard_normal((B, H, T, TG)).astype(np.float32)
    fine[:, 0] = np.round(fine[:, 0] * 4) / 4          # heavy ties
    coarse[:, 0] = np.round(coarse[:, 0] * 2) / 2
    fine[:, 1, :, ::3] = -0.0                           # -0 ties with +0
    fine[:, 1, :, 1::3] = 0.0
    coarse[:, 1, :, ::2] = 0.0
    run = Run(_scores_workload(B, H, T, fr), with_logits=False)
    hz = slab.Hierarchy(G, *extra)
    slab.sla_classify_hierarchical_from_scores(run.shape, to_dev(fine), to_dev(coarse), hz,
                                               run.buf.mask, run.buf.workspace)
    run.check()
    torch.cuda.synchronize()
    n_h, n_l = oracle.block_counts(T, *fr)
    cls_ref = oracle.classify_hierarchical(fine.astype(np.float64), coarse.astype(np.float64),
                                           n_h, n_l, G, *extra)
    check_mask_outputs(run, cls_ref)


def _run_hier(wl, G, extra=(0, 0), n_valid=0):
    import torch
    run = Run(wl, n_valid=n_valid)
    slab = run.slab
    hz = slab.Hierarchy(G, *extra)
    TG, c_hi, c_lo = slab.sla_hierarchy_counts(run.shape, hz)
    coarse = torch.full((wl.B, wl.H, wl.T, TG), float("nan"), dtype=torch.float32,
                        device="cuda")
    run.buf.pooled_logits.fill_(float("nan"))
    slab.sla_classify_hierarchical(run.shape, run.q, run.k, hz, run.buf.mask, coarse,
                                   run.buf.workspace)
    run.check()
    return run, coarse.cpu().numpy().astype(np.float64), (TG, c_hi, c_lo)


def _grid(name, grid, H, k_h, k_l, n_tokens=None):
    return sla_inputs.make_grid(grid, H=H, k_h=k_h, k_l=k_l, name=name, n_tokens=n_tokens)


INPUTS = {
    "mid_G8": (lambda: sla_inputs.make("mid"), 8, (0, 0)),
    "mid_G4_wide": (lambda: sla_inputs.make("mid"), 4, (6, 6)),
    "ragged_T_37": (lambda: _grid("r37", (2, 37, 32), 2, 0.10, 0.20), 4, (0, 0)),
    "long_2h": (lambda: _grid("long", (21, 45, 80), 2, 0.10, 0.10), 16, (0, 0)),
}


@pytest.mark.parametrize("name", list(INPUTS))
def test_hierarchical_from_inputs(name):
    make, G, extra = INPUTS[name]
    wl = make()
    run, coarse, (TG, c_hi, c_lo) = _run_hier(wl, G, extra)
    assert c_hi + c_lo <= TG  # these cases prune
    n_h, n_l = oracle.block_counts(wl.T, wl.k_h, wl.k_l)
    # coarse scores and the fine scores the kernel computed (candidates only)
    co_ref = oracle.coarse_logits(wl.q, wl.k, wl.block, wl.scale, G)
    lg_ref = oracle.pooled_logits(wl.q, wl.k, wl.block, wl.scale)
    tol = 1e-6 * max(1.0, np.abs(lg_ref).max())
    np.testing.assert_allclose(coarse, co_ref, rtol=0, atol=tol)
    lg = run.buf.pooled_logits.cpu().numpy().astype(np.float64)
    seen = np.isfinite(lg)
    np.testing.assert_allclose(lg[seen], lg_ref[seen], rtol=0, atol=tol)
    # the class map is exact on the kernel's own scores (NaN where it computed
    # none: the oracle rejects a NaN it would have to read)
    cls = run.cls()
    assert np.array_equal(cls, oracle.classify_hierarchical(lg, coarse, n_h, n_l, G, *extra))
    check_mask_outputs(run, cls)
    assert ((cls == 1).sum(-1) == n_h).all() and ((cls == -1).sum(-1) == n_l).all()
    # fine scores were computed for exactly (c_hi + c_lo) super-blocks' blocks per row
    per_row = seen.sum(-1)
    assert per_row.max() <= (c_hi + c_lo) * G and per_row.min() >= n_h + n_l


def test_hierarchical_flat_case_is_sla_classify():
    wl = sla_inputs.make("mid")
    run, _, (TG, c_hi, c_lo) = _run_hier(wl, 4, (20, 20))  # 20 + 20 > 32 super-blocks
    assert c_hi == c_lo == TG
    ref = Run(wl)
    ref.classify()
    assert np.array_equal(run.cls(), ref.cls())
    np.testing.assert_array_equal(run.buf.pooled_logits.cpu().numpy(),
                                  ref.buf.pooled_logits.cpu().numpy())


def test_hierarchical_with_key_padding():
    wl = _grid("r37", (2, 37, 32), 2, 0.10, 0.20)
    nv = wl.N - 23
    run, coarse, _ = _run_hier(wl, 4, n_valid=nv)
    co_ref = oracle.coarse_logits(wl.q, wl.k, wl.block, wl.scale, 4, n_valid=nv)
    np.testing.assert_allclose(coarse, co_ref, rtol=0, atol=1e-6 * max(1.0, np.abs(co_ref).max()))
    lg = run.buf.pooled_logits.cpu().numpy().astype(np.float64)
    n_h, n_l = oracle.block_counts(wl.T, wl.k_h, wl.k_l)
    assert np.array_equal(run.cls(), oracle.classify_hierarchical(lg, coarse, n_h, n_l, 4))


def test_forward_on_a_hierarchical_mask():
    wl = sla_inputs.make("mid")
    run, _, _ = _run_hier(wl, 8)
    run.forward()
    cls = run.cls()
    ref = oracle.forward(wl.q, wl.k, wl.v, wl.w_proj, cls, wl.block, wl.scale)
    assert_close(run.np(run.o), ref["o"], "o")
