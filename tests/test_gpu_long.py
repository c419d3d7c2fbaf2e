"""GPU parity on the long-sequence workload: a 21x45x80 latent grid, N = 75648
tokens (75600 real, zero-padded to whole 64-token blocks), T = 1182 blocks,
d = 128, against the fp64 oracle on two heads.

The forward is checked on sampled query blocks (first, last and interior) at
each critical fraction of the sparsity sweep (k_h = 2.5, 5, 10 % -> 30, 60, 119
critical blocks per row).  The backward runs in full at k_h = 10 %, where the
key-block pairs' unions reach up to 238 query blocks, so the largest union
lists of both attention kernels are exercised."""

import numpy as np
import pytest

import oracle
import sla_inputs
from sla_harness import Run, assert_close

pytestmark = pytest.mark.gpu

HEADS = 2


def _long(k_h, with_grad=False):
    return sla_inputs.make("long", H=HEADS, k_h=k_h, with_grad=with_grad)


@pytest.mark.parametrize("k_h", [0.025, 0.05, 0.10])
def test_long_forward_sampled(k_h):
    wl = _long(k_h)
    T = wl.T
    assert T == 1182
    run = Run(wl)
    run.classify()
    run.forward()
    cls = run.cls()
    n_h, _ = oracle.block_counts(T, wl.k_h, wl.k_l)
    assert int((cls[0, 0, 0] == 1).sum()) == n_h
    blocks = [0, 1, T // 3, T // 2, T - 2, T - 1]
    ref = oracle.forward(wl.q, wl.k, wl.v, wl.w_proj, cls, wl.block, wl.scale,
                         query_blocks=blocks)
    rows = np.concatenate([np.arange(i * 64, (i + 1) * 64) for i in blocks])
    pick = lambda a: a[:, :, rows]
    assert_close(pick(run.np(run.o)), pick(ref["o"]), "o")
    assert_close(pick(run.np(run.buf.o_s)), pick(ref["o_s"]), "o_s")
    lse = pick(run.np(run.buf.lse))
    np.testing.assert_allclose(lse, pick(ref["lse"]), rtol=1e-4, atol=1e-4)


def test_long_backward_full_k10():
    wl = _long(0.10, with_grad=True)
    run = Run(wl)
    run.classify()
    run.forward()
    run.backward(wl.d_o)
    cls = run.cls()
    # the widest unions of two adjacent rows / columns reach past n_crit
    crit = cls == 1
    assert int((crit[..., :-1, :] | crit[..., 1:, :]).sum(-1).max()) > 119
    fwd = oracle.forward(wl.q, wl.k, wl.v, wl.w_proj, cls, wl.block, wl.scale)
    g = oracle.backward(wl.q, wl.k, wl.v, wl.w_proj, cls, wl.d_o, wl.block, wl.scale, fwd=fwd)
    assert_close(run.np(run.o), fwd["o"], "o")
    for name, t in (("dq", run.dq), ("dk", run.dk), ("dv", run.dv), ("dw", run.dw)):
        assert_close(run.np(t), g[name], name)
