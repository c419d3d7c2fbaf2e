"""Helpers shared by the GPU tests: run the library through its C ABI on a
workload and compare tensors with the oracle using the acceptance metrics
(max|d| <= 1e-2 max|ref|, sum|d| / sum|ref| <= 3e-3 per tensor)."""

from __future__ import annotations

import numpy as np

MAX_TOL = 1e-2
MEAN_TOL = 3e-3


def to_dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.abs(got - ref)
    mx = float(d.max() / max(np.abs(ref).max(), 1e-300))
    mean = float(d.sum() / max(np.abs(ref).sum(), 1e-300))
    return mx, mean


def assert_close(got, ref, what, max_tol=MAX_TOL, mean_tol=MEAN_TOL):
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    mx, mean = errors(got, ref)
    assert mx <= max_tol and mean <= mean_tol, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


class Run:
    """One library run (classification + forward [+ backward]) on a workload."""

    def __init__(self, wl, with_logits=True, n_valid=0):
        import torch
        import sparse_linear_attention_block_b200 as slab
        self.slab = slab
        self.wl = wl
        self.shape = slab.make_shape(wl.B, wl.H, wl.N, wl.d, wl.block, wl.k_h, wl.k_l,
                                     n_valid=n_valid)
        self.buf = slab.Buffers.allocate(self.shape, with_logits=with_logits)
        self.q = to_dev(wl.q, torch.bfloat16)
        self.k = to_dev(wl.k, torch.bfloat16)
        self.v = to_dev(wl.v, torch.bfloat16)
        self.w = to_dev(wl.w_proj, torch.bfloat16)
        self.o = torch.empty_like(self.q)

    def classify(self):
        self.slab.sla_classify(self.shape, self.q, self.k, self.buf.mask, self.buf.workspace)
        self.check()

    def classify_from_scores(self, logits):
        import torch
        lt = to_dev(np.asarray(logits, dtype=np.float32))
        self.slab.sla_classify_from_scores(self.shape, lt, self.buf.mask, self.buf.workspace)
        self.check()
        torch.cuda.synchronize()

    def forward(self):
        self.slab.sla_forward(self.shape, self.q, self.k, self.v, self.w, self.buf.mask, self.o,
                              self.buf.saved, self.buf.workspace)
        self.check()

    def backward(self, d_o):
        import torch
        self.do = to_dev(d_o, torch.bfloat16)
        self.dq = torch.empty(self.q.shape, dtype=torch.float32, device="cuda")
        self.dk = torch.empty_like(self.dq)
        self.dv = torch.empty_like(self.dq)
        self.dw = torch.empty(self.w.shape, dtype=torch.float32, device="cuda")
        self.slab.sla_backward(self.shape, self.q, self.k, self.v, self.w, self.buf.mask,
                               self.buf.saved, self.do, self.dq, self.dk, self.dv, self.dw,
                               self.buf.workspace)
        self.check()

    def check(self):
        self.slab.sla_check(self.buf.workspace)

    def cls(self):
        return self.buf.cls.cpu().numpy()

    def np(self, t, dtype=np.float64):
        import torch
        if t.dtype == torch.bfloat16:
            t = t.float()
        return t.cpu().numpy().astype(dtype)


def expected_csr(cls):
    B, H, T, _ = cls.shape
    n_crit = int((cls[0, 0, 0] == 1).sum())
    ptr = np.zeros((B, H, T + 1), np.int64)
    idx = np.zeros((B, H, T * max(n_crit, 1)), np.int64)
    for b in range(B):
        for h in range(H):
            pos = 0
            for j in range(T):
                ptr[b, h, j] = pos
                rows = np.nonzero(cls[b, h, :, j] == 1)[0]
                idx[b, h, pos:pos + rows.size] = rows
                pos += rows.size
            ptr[b, h, T] = pos
    return ptr, idx


def check_mask_outputs(run, cls_ref):
    """crit_idx, marg_bits and the column CSR must be consistent with cls."""
    B, H, T, _ = cls_ref.shape
    s = run.buf.sizes
    cls = run.cls()
    assert np.array_equal(cls, cls_ref)
    if s.n_crit > 0:
        crit = run.buf.crit_idx.cpu().numpy()[..., :s.n_crit]
        exp = np.stack([np.nonzero(r == 1)[0] for r in cls_ref.reshape(-1, T)]).reshape(
            B, H, T, s.n_crit)
        assert np.array_equal(crit, exp)
    bits = run.buf.marg_bits.cpu().numpy().view(np.uint32)
    for j in range(T):
        got = (bits[..., j // 32] >> np.uint32(j % 32)) & 1
        assert np.array_equal(got.astype(bool), cls_ref[..., j] == 0)
    ptr, idx = expected_csr(cls_ref)
    assert np.array_equal(run.buf.crit_col_ptr.cpu().numpy(), ptr)
    n = T * s.n_crit
    if n:
        assert np.array_equal(run.buf.crit_col_idx.cpu().numpy()[..., :n], idx[..., :n])
