"""GPU parity of classification and forward against the fp64 oracle, through
the C ABI.  Output parity feeds the oracle the library's own class map, so a
classification tie can never cascade into an output mismatch."""

import math

import numpy as np
import pytest

import oracle
import sla_inputs
from sla_harness import Run, assert_close, check_mask_outputs, errors

pytestmark = pytest.mark.gpu


def _grid(name, grid, H, k_h, k_l, n_tokens=None, d=128):
    return sla_inputs.make_grid(grid, H=H, d=d, k_h=k_h, k_l=k_l, name=name,
                                n_tokens=n_tokens)


WORKLOADS = {
    "tiny": lambda: sla_inputs.make("tiny"),
    "mid": lambda: sla_inputs.make("mid"),
    "wan_slice_2048": lambda: _grid("wan_slice", (21, 30, 52), 12, 0.05, 0.10, n_tokens=2048),
    "odd_T_7": lambda: _grid("odd", (3, 7, 21), 3, 0.25, 0.25),       # 441 tokens -> T = 7
    "ragged_T_37": lambda: _grid("r37", (2, 37, 32), 2, 0.10, 0.20),  # T = 37
}


@pytest.mark.parametrize("T,fr", [(16, (0.25, 0.25)), (37, (0.10, 0.20)), (128, (0.05, 0.10)),
                                  (64, (1.0, 0.0)), (64, (0.0, 1.0)), (64, (0.0, 0.0)),
                                  (33, (0.5, 0.5)), (512, (0.05, 0.10))])
def test_classify_from_scores_bit_exact(T, fr):
    B, H = 1, 3
    rng = np.random.default_rng(T)
    logits = rng.standard_normal((B, H, T, T)).astype(np.float32)
    logits[:, 0] = np.round(logits[:, 0] * 4) / 4       # heavy ties
    logits[:, 1, :, ::3] = -0.0                          # -0 ties with +0
    logits[:, 1, :, 1::3] = 0.0
    wl = sla_inputs.Workload("scores", B, H, T * 64, 64, 64, fr[0], fr[1], T * 64,
                             np.zeros((B, H, T * 64, 64), np.float32),
                             np.zeros((B, H, T * 64, 64), np.float32),
                             np.zeros((B, H, T * 64, 64), np.float32),
                             np.zeros((64, 64), np.float32))
    run = Run(wl, with_logits=False)
    run.classify_from_scores(logits)
    n_h, n_l = oracle.block_counts(T, *fr)
    cls_ref = oracle.classify(logits.astype(np.float64), n_h, n_l)
    check_mask_outputs(run, cls_ref)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_classify_from_inputs(name):
    wl = WORKLOADS[name]()
    run = Run(wl)
    run.classify()
    lg_ref = oracle.pooled_logits(wl.q, wl.k, wl.block, wl.scale)
    lg = run.buf.pooled_logits.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(lg, lg_ref, rtol=0, atol=1e-6 * max(1.0, np.abs(lg_ref).max()))
    n_h, n_l = oracle.block_counts(wl.T, wl.k_h, wl.k_l)
    cls_ref = oracle.classify(lg_ref, n_h, n_l)
    cls = run.cls()
    # differences only at ties: the oracle logit within 1e-6 of a class boundary
    T = wl.T
    srt = -np.sort(-lg_ref, axis=-1)
    bounds = []
    if n_h:
        bounds.append(srt[..., n_h - 1])
    if n_l:
        bounds.append(srt[..., T - n_l])
    diff = np.argwhere(cls != cls_ref)
    for b, h, i, j in diff:
        near = any(abs(lg_ref[b, h, i, j] - tau[b, h, i]) <= 1e-6 * max(1.0, abs(tau[b, h, i]))
                   for tau in bounds)
        assert near, (b, h, i, j)
    # the library's own outputs are consistent with its class map
    check_mask_outputs(run, cls)
    # and its ranking is exact on its own exported fp32 logits
    assert np.array_equal(cls, oracle.classify(lg, n_h, n_l))


def _forward_and_compare(wl, sample_blocks=None):
    run = Run(wl)
    run.classify()
    run.forward()
    cls = run.cls()
    ref = oracle.forward(wl.q, wl.k, wl.v, wl.w_proj, cls, wl.block, wl.scale,
                         query_blocks=sample_blocks)
    o = run.np(run.o)
    o_s = run.np(run.buf.o_s)
    lse = run.np(run.buf.lse)
    den = run.np(run.buf.den)
    if sample_blocks is not None:
        rows = np.concatenate([np.arange(i * 64, (i + 1) * 64) for i in sample_blocks])
        o, o_s, lse, den = o[:, :, rows], o_s[:, :, rows], lse[:, :, rows], den[:, :, rows]
        ref = {k: v[:, :, rows] for k, v in ref.items() if isinstance(v, np.ndarray)}
    res = {"o": assert_close(o, ref["o"], "o"),
           "o_s": assert_close(o_s, ref["o_s"], "o_s", 1e-2, 2e-3)}
    fin = np.isfinite(ref["lse"])
    assert np.array_equal(np.isfinite(lse), fin)
    if fin.any():
        np.testing.assert_allclose(lse[fin], ref["lse"][fin], rtol=1e-4, atol=1e-4)
    np.testing.assert_allclose(den, ref["den"], rtol=2e-3, atol=1e-6)
    return run, res


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_forward_parity(name):
    _forward_and_compare(WORKLOADS[name]())


@pytest.mark.parametrize("fr", [(1.0, 0.0), (0.0, 0.0), (0.0, 1.0), (0.5, 0.5), (0.0, 0.5)])
def test_forward_degenerate_fractions(fr):
    wl = sla_inputs.make("tiny", k_h=fr[0], k_l=fr[1])
    run, _ = _forward_and_compare(wl)
    o = run.np(run.o)
    if fr == (0.0, 1.0):
        assert np.all(o == 0)


def test_forward_all_critical_is_dense_attention():
    import torch
    wl = sla_inputs.make("tiny", k_h=1.0, k_l=0.0)
    run = Run(wl)
    run.classify()
    run.forward()
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.tensor(x, dtype=torch.float64) for x in (wl.q, wl.k, wl.v))).numpy()
    assert_close(run.np(run.o), ref, "o vs SDPA")


def test_forward_zero_projection():
    wl = sla_inputs.make("tiny")
    wl.w_proj = np.zeros_like(wl.w_proj)
    run, _ = _forward_and_compare(wl)
    # O is the bf16 rounding of the saved fp32 sparse output
    o_s = run.buf.o_s.to(__import__("torch").bfloat16).float().cpu().numpy()
    assert np.array_equal(run.np(run.o, np.float32), o_s)


def test_forward_wan_full_size_sampled():
    wl = sla_inputs.make("wan")
    T = wl.T
    blocks = [0, 1, 2, T // 2 - 1, T // 2, T - 2, T - 1]
    _forward_and_compare(wl, sample_blocks=blocks)


def test_forward_mask_reuse_is_deterministic():
    wl = WORKLOADS["wan_slice_2048"]()
    run = Run(wl)
    run.classify()
    run.forward()
    o1 = run.o.clone()
    run.forward()   # same mask, second call
    assert bool((o1 == run.o).all())
