"""GPU parity with key padding (sla_shape.n_valid) against the fp64 oracle:
padded tokens take no part and padded positions come out zero."""

import numpy as np
import pytest

import oracle
import sla_inputs
from sla_harness import Run, assert_close

pytestmark = pytest.mark.gpu


def _padded(grid, H, k_h, k_l, fill_seed, n_tokens=None):
    wl = sla_inputs.make_grid(grid, H=H, k_h=k_h, k_l=k_l, with_grad=True, name="pad",
                              n_tokens=n_tokens)
    assert wl.n_valid < wl.N
    rng = np.random.default_rng(fill_seed)
    for a in (wl.q, wl.k, wl.v, wl.d_o):  # garbage, not zeros, in the padding
        pad = a[:, :, wl.n_valid:]
        pad[...] = sla_inputs.bf16_round((rng.standard_normal(pad.shape) * 3).astype(np.float32))
    return wl


CASES = {
    "grid_3x7x21": lambda seed: _padded((3, 7, 21), 3, 0.25, 0.25, seed),          # 441 of 448
    "wan_slice_2040": lambda seed: _padded((21, 30, 52), 4, 0.05, 0.10, seed, 2040),  # 2040 of 2048
}


def _run(wl):
    run = Run(wl, n_valid=wl.n_valid)
    run.classify()
    run.forward()
    run.backward(wl.d_o)
    return run


@pytest.mark.parametrize("name", list(CASES))
def test_padded_parity(name):
    wl = CASES[name](1)
    nv = wl.n_valid
    run = _run(wl)
    # classification scores from the valid tokens only
    ref_logits = oracle.pooled_logits(wl.q, wl.k, wl.block, wl.scale, nv)
    got_logits = run.np(run.buf.pooled_logits)
    assert np.abs(got_logits - ref_logits).max() <= 1e-5 * np.abs(ref_logits).max()
    cls = run.cls()
    fwd = oracle.forward(wl.q, wl.k, wl.v, wl.w_proj, cls, wl.block, wl.scale, n_valid=nv)
    o = run.np(run.o)
    assert_close(o, fwd["o"], "o")
    assert np.all(o[:, :, nv:] == 0)
    lse = run.np(run.buf.lse)
    fin = np.isfinite(fwd["lse"])
    assert np.array_equal(np.isfinite(lse), fin)
    np.testing.assert_allclose(lse[fin], fwd["lse"][fin], rtol=1e-4, atol=1e-4)
    np.testing.assert_allclose(run.np(run.buf.den), fwd["den"], rtol=2e-3, atol=1e-6)
    g = oracle.backward(wl.q, wl.k, wl.v, wl.w_proj, cls, wl.d_o, wl.block, wl.scale, fwd=fwd,
                        n_valid=nv)
    for n, t in (("dq", run.dq), ("dk", run.dk), ("dv", run.dv), ("dw", run.dw)):
        got = run.np(t)
        assert_close(got, g[n], n)
        if n != "dw":
            assert np.all(got[:, :, nv:] == 0), n


def test_padding_contents_do_not_matter():
    a, b = _run(CASES["grid_3x7x21"](1)), _run(CASES["grid_3x7x21"](2))
    assert np.array_equal(a.cls(), b.cls())
    np.testing.assert_array_equal(a.np(a.o), b.np(b.o))
    for ta, tb, n in ((a.dq, b.dq, "dq"), (a.dk, b.dk, "dk"), (a.dv, b.dv, "dv"), (a.dw, b.dw, "dw")):
        x, y = a.np(ta), b.np(tb)
        assert np.abs(x - y).max() <= 1e-5 * np.abs(y).max(), n  # fp32 reduction order only


def test_full_valid_length_is_unpadded():
    wl = sla_inputs.make("mid", with_grad=True)
    a = Run(wl)
    b = Run(wl, n_valid=wl.N)
    for r in (a, b):
        r.classify()
        r.forward()
    assert np.array_equal(a.cls(), b.cls())
    np.testing.assert_array_equal(a.np(a.o), b.np(b.o))
