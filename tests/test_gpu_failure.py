"""Device-side failure paths, made to happen without a fault, trap or hang.

- A wait that runs out: sla_debug_inject makes the sparse forward's copy warp
  issue none of its copies; every wait on them gives up after its time limit,
  the kernel winds down with nothing in flight, and sla_check reports
  SLA_ERR_TIMEOUT.  The context stays usable: the next forward is correct.
- An index out of range in a caller-given mask: the sparse kernels check the
  block indices before any copy, drop the bad entry and record
  SLA_ERR_DEVICE."""

import numpy as np
import pytest

import oracle
import sla_inputs
from sla_harness import Run, assert_close

pytestmark = pytest.mark.gpu


def _status_of(fn):
    import sparse_linear_attention_block_b200 as slab
    try:
        fn()
    except slab.SlaError as e:
        return e.status
    return 0


def test_withheld_copies_time_out_and_context_survives():
    import sparse_linear_attention_block_b200 as slab
    wl = sla_inputs.make("tiny")
    run = Run(wl)
    run.classify()
    slab.sla_debug_inject(run.buf.workspace, slab.INJECT_WITHHOLD_LOADS)
    slab.sla_forward(run.shape, run.q, run.k, run.v, run.w, run.buf.mask, run.o, run.buf.saved,
                     run.buf.workspace)
    assert _status_of(run.check) == 5  # SLA_ERR_TIMEOUT
    # cleared, the same call is correct again on the same context
    slab.sla_debug_inject(run.buf.workspace, 0)
    run.forward()
    ref = oracle.forward(wl.q, wl.k, wl.v, wl.w_proj, run.cls(), wl.block, wl.scale)
    assert_close(run.np(run.o), ref["o"], "o after the timeout")


def test_out_of_range_block_index_is_reported():
    import torch
    import sparse_linear_attention_block_b200 as slab
    wl = sla_inputs.make("tiny", with_grad=True)
    run = Run(wl)
    run.classify()
    T = wl.T
    # forward: a critical key-block index past the last block
    bad = run.buf.crit_idx.clone()
    run.buf.crit_idx[0, 0, 0, 0] = T + 5
    slab.sla_forward(run.shape, run.q, run.k, run.v, run.w, run.buf.mask, run.o, run.buf.saved,
                     run.buf.workspace)
    assert _status_of(run.check) == 6  # SLA_ERR_DEVICE
    run.buf.crit_idx.copy_(bad)
    run.forward()
    # backward: a query-block index past the last block in the column lists
    run.buf.crit_col_idx[0, 0, 0] = T + 3
    do = torch.from_numpy(wl.d_o).to(torch.bfloat16).cuda()
    dq = torch.empty(run.q.shape, dtype=torch.float32, device="cuda")
    dk, dv = torch.empty_like(dq), torch.empty_like(dq)
    dw = torch.empty(run.w.shape, dtype=torch.float32, device="cuda")
    slab.sla_backward(run.shape, run.q, run.k, run.v, run.w, run.buf.mask, run.buf.saved, do, dq,
                      dk, dv, dw, run.buf.workspace)
    assert _status_of(run.check) == 6
    torch.cuda.synchronize()
    assert np.isfinite(dq.cpu().numpy()).all()
