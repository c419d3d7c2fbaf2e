"""One warm-up and one measured SLA training step (classify + forward +
backward) on a Wan-shaped case with a chosen number of heads, for profiler
captures (e.g. ``ncu ... python -m sparse_linear_attention_block_b200.profile_step
--heads 4``).  Prints "ok" after checking the device error word."""

from __future__ import annotations

import argparse
import os
import sys


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--heads", type=int, default=4)
    ap.add_argument("--grid", type=int, nargs=3, default=(21, 30, 52))
    ap.add_argument("--k-h", type=float, default=0.05)
    ap.add_argument("--k-l", type=float, default=0.10)
    ap.add_argument("--steps", type=int, default=2)
    args = ap.parse_args(argv)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import torch

    import sla_inputs
    import sparse_linear_attention_block_b200 as slab

    wl = sla_inputs.make_grid(tuple(args.grid), H=args.heads, k_h=args.k_h, k_l=args.k_l,
                              with_grad=True, name="profile")
    sh = slab.make_shape(wl.B, wl.H, wl.N, wl.d, wl.block, wl.k_h, wl.k_l)
    buf = slab.Buffers.allocate(sh, with_logits=False)
    dev = lambda a: torch.from_numpy(a).to(torch.bfloat16).cuda()
    q, k, v, w, do = (dev(x) for x in (wl.q, wl.k, wl.v, wl.w_proj, wl.d_o))
    o = torch.empty_like(q)
    dq = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    dk, dv = torch.empty_like(dq), torch.empty_like(dq)
    dw = torch.empty(w.shape, dtype=torch.float32, device="cuda")
    for _ in range(args.steps):
        slab.sla_classify(sh, q, k, buf.mask, buf.workspace)
        slab.sla_forward(sh, q, k, v, w, buf.mask, o, buf.saved, buf.workspace)
        slab.sla_backward(sh, q, k, v, w, buf.mask, buf.saved, do, dq, dk, dv, dw, buf.workspace)
    slab.sla_check(buf.workspace)
    torch.cuda.synchronize()
    print("ok")


if __name__ == "__main__":
    main()
