"""Benchmark of the SLA hot path on B200: one step = classification + forward +
backward of sparse-linear attention on a Wan2.1-1.3B-shaped training
workload (B=1, H=12, N=32768 tokens from a 21x30x52 latent grid padded to
64-token blocks, d=128, k_h=5%, k_l=10%, synthetic inputs, seed = rank).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sla|reference]

Prints one JSON line (rank 0).  ``value`` is executed-block TFLOP/s of the
whole step: (forward 4*b^2*d + backward 10*b^2*d) per critical
(query block, key block) pair, summed over ranks, divided by the max over
ranks of the device time per step.  With N > 1 every rank runs an
independent replica of the step (weak scaling, no collective on the data
path).  ``--impl reference`` times the fp64 CPU oracle on a bounded sample
of the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SLA fwd/bwd ms and executed-block TFLOP/s (% bf16 peak) at N=32768,H=12,d=128"
WORKLOAD = dict(name="train", B=1, H=12, d=128, grid=(21, 30, 52), block=64, k_h=0.05, k_l=0.10)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def workload_config(wl, n_crit):
    kind = ("Wan2.1-1.3B-shaped" if wl.name == "train" else "long-sequence")
    grid = "x".join(str(g) for g in wl.grid) if wl.grid else "none"
    return {
        "workload": f"{kind} SLA training step (classify+forward+backward): B={wl.B} H={wl.H} "
                    f"N={wl.N} ({grid} grid padded) d={wl.d} block={wl.block} "
                    f"k_h={wl.k_h:g} k_l={wl.k_l:g}",
        "B": wl.B, "H": wl.H, "N": wl.N, "d": wl.d, "block": wl.block, "k_h": wl.k_h,
        "k_l": wl.k_l, "n_crit": n_crit, "global_batch": wl.B, "seq_len": wl.N,
        "l2": f"inputs larger than L2 (Q/K/V/dO bf16 = {4 * wl.B * wl.H * wl.N * wl.d * 2 / 1e6:.0f} "
              f"MB per step)",
        "parallelism": "independent replica per GPU",
    }


def executed_block_flops(wl, n_crit):
    pairs = wl.B * wl.H * wl.T * n_crit
    fwd = pairs * 4 * wl.block * wl.block * wl.d
    bwd = pairs * 10 * wl.block * wl.block * wl.d
    return fwd, bwd


# DRAM bytes (read + write) per head of one launch, from an ncu capture of the
# kernel as it is now (dram__bytes_read.sum + dram__bytes_write.sum of the
# 4-head Wan case, divided by 4; the traffic grows with the number of heads).
# A kernel missing here reports traffic null; an entry must be dropped or
# re-measured whenever its kernel changes.
NCU_DRAM_BYTES_PER_HEAD = {
    "bwd_sparse": (395.572224e6 + 233.325056e6) / 4,
    "fwd_sparse": (100.750592e6 + 35.872512e6) / 4,
    "pool": (67.117824e6 + 0.468992e6) / 4,
    "summaries": (67.146496e6 + 79.487232e6) / 4,
}


def kernel_work(wl, n_crit):
    """Algorithmic work per launch of each kernel: ('tensor', FLOP) or ('hbm', bytes)."""
    B, H, N, d, T = wl.B, wl.H, wl.N, wl.d, wl.T
    BH = B * H
    Tp = (T + 127) // 128 * 128
    tok = BH * N
    pairs = BH * T * n_crit
    b = wl.block
    return {
        "pool": ("hbm", 2 * tok * d * 2 + 2 * BH * T * d * 4),
        "summaries": ("hbm", 2 * tok * d * 2 + BH * T * d * d * 4 + BH * T * d * 4),
        "aggregate": ("tensor", 2 * BH * T * T * d * d),
        "aggregate_t": ("tensor", 2 * BH * T * T * d * d),
        "fwd_sparse": ("tensor", pairs * 4 * b * b * d),
        "fwd_linear": ("hbm", tok * d * (2 + 4 + 2) + BH * T * (d * d + d) * 4 + tok * 4),
        "bwd_q": ("hbm", tok * d * (2 + 2 + 4 + 4) + 2 * BH * T * (d * d + d) * 4 + tok * 4 * 2),
        "bwd_sparse": ("tensor", pairs * 10 * b * b * d),
        "bwd_k": ("hbm", tok * d * (2 + 2 + 8 + 8) + BH * T * (d * d + d) * 4),
        "expand_marginal": ("hbm", BH * Tp * Tp * 2),
        "expand_marginal_t": ("hbm", BH * Tp * Tp * 2),
    }


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        self.skip = 0

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return self
        # nvidia-smi takes a moment to start: wait for its first sample so that
        # the timed region is sampled from its start; samples taken before it
        # (the wait itself) are dropped
        t0 = time.time()
        while time.time() - t0 < 5.0 and self.proc.poll() is None:
            with open(self.path) as f:
                n = sum(1 for _ in f)
            if n:
                self.skip = n
                break
            time.sleep(0.01)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        with open(self.path) as f:
            for ln in f:
                parts = [x.strip() for x in ln.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        # the timed region's samples; a region shorter than the sampling
        # interval keeps the sample closest to it
        rows = rows[self.skip:] or rows[-1:]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = [x for x in threadpool_info() if x.get("user_api") == "blas"]
        if info:
            return int(info[0]["num_threads"])
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample_step(wl, heads):
    """classification + forward + backward of the fp64 oracle on `heads`."""
    import oracle
    sub = lambda a: a[:, heads]
    T = wl.T
    n_h, n_l = oracle.block_counts(T, wl.k_h, wl.k_l)
    logits = oracle.pooled_logits(sub(wl.q), sub(wl.k), wl.block, wl.scale)
    cls = oracle.classify(logits, n_h, n_l)
    fwd = oracle.forward(sub(wl.q), sub(wl.k), sub(wl.v), wl.w_proj, cls, wl.block, wl.scale)
    oracle.backward(sub(wl.q), sub(wl.k), sub(wl.v), wl.w_proj, cls, sub(wl.d_o), wl.block,
                    wl.scale, fwd=fwd)
    return n_h


def time_oracle(wl, heads, steps, warmup):
    t_all = []
    n_h = 0
    for i in range(warmup + steps):
        t0 = time.perf_counter()
        n_h = oracle_sample_step(wl, heads)
        if i >= warmup:
            t_all.append(time.perf_counter() - t0)
    sample = wl.B * len(heads) * wl.T * n_h * 14 * wl.block * wl.block * wl.d
    sec = statistics.mean(t_all)
    return sample / sec / 1e12, sec


# ---------------------------------------------------------------- ranks
# One process per GPU; every rank runs an independent replica of the step on
# its own inputs (weak scaling, no collective on the data path).  Timing is the
# maximum over ranks of each rank's device time; the whole-job value counts the
# work of every rank.

def rank_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks_of(x, world, dev):
    """The maximum of a per-rank float over all ranks (a collective when world > 1)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank_step, ms_per_step, world):
    """Executed-block TFLOP/s of all ranks together at the slowest rank's step time."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def run_reference(args, rank, world):
    if rank != 0:
        return
    import sla_inputs
    wl = sla_inputs.make("train", seed=0)
    heads = [0]
    tflops, sec = time_oracle(wl, heads, args.steps, args.warmup)
    n_crit = oracle_n_crit(wl)
    cfg = workload_config(wl, n_crit)
    sample = (f"head 0 of 12 of the same workload per step (classify+forward+backward, fp64 "
              f"numpy on {blas_threads()} BLAS threads), {sec:.2f} s per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def dense_sdpa_context(B, H, N, d, dev, reps=3):
    """Dense attention at the same shape through torch SDPA (context only):
    forward and forward+backward ms per backend, CUDA events on the current
    stream; FLOPs 4 N^2 d (forward) and 14 N^2 d (forward + backward) per head."""
    import torch
    from torch.nn.attention import SDPBackend, sdpa_kernel
    g = torch.Generator(device=dev).manual_seed(0)
    q, k, v = (torch.randn(B, H, N, d, device=dev, dtype=torch.bfloat16, generator=g)
               for _ in range(3))
    fwd_flop = 4.0 * B * H * N * N * d
    out = {}
    for name, backend in (("flash", SDPBackend.FLASH_ATTENTION),
                          ("cudnn", SDPBackend.CUDNN_ATTENTION)):
        try:
            with sdpa_kernel([backend]):
                qq, kk, vv = (x.detach().requires_grad_(True) for x in (q, k, v))
                def fwd():
                    return torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)
                def fwd_bwd():
                    o = fwd()
                    o.backward(torch.ones_like(o))
                for fn in (fwd, fwd_bwd):  # warm-up
                    fn()
                torch.cuda.synchronize()
                res = {}
                for label, fn in (("fwd", fwd), ("fwd_bwd", fwd_bwd)):
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    for _ in range(reps):
                        fn()
                    e1.record()
                    torch.cuda.synchronize()
                    res[label + "_ms"] = e0.elapsed_time(e1) / reps
                res["fwd_tflops"] = fwd_flop / (res["fwd_ms"] * 1e-3) / 1e12
                res["fwd_bwd_tflops"] = 3.5 * fwd_flop / (res["fwd_bwd_ms"] * 1e-3) / 1e12
                out[name] = res
        except Exception as exc:  # a backend this torch build does not offer
            out[name] = {"unavailable": str(exc).splitlines()[0][:160]}
    del q, k, v
    torch.cuda.empty_cache()
    return out


def oracle_n_crit(wl):
    import oracle
    return oracle.block_counts(wl.T, wl.k_h, wl.k_l)[0]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["sla", "reference"], default="sla")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true",
                    help="skip the dense torch SDPA context timing")
    ap.add_argument("--gate-logit", type=float, default=None,
                    help="run the gated entry points with this gate logit (default: ungated)")
    ap.add_argument("--key-padding", action="store_true",
                    help="mask the grid's padding tokens (n_valid) instead of treating them as tokens")
    ap.add_argument("--gate-skip", type=float, default=0.0,
                    help="drop the linear branch when sigmoid(logit) is below this")
    ap.add_argument("--workload", choices=["train", "long"], default="train",
                    help="train: N=32768 (21x30x52 grid); long: N=75648 (21x45x80 grid)")
    ap.add_argument("--k-h", type=float, default=None,
                    help="critical fraction (default: the workload's 0.05)")
    ap.add_argument("--hierarchical", type=int, default=0, metavar="G",
                    help="classify hierarchically with super-blocks of G key blocks (0: flat)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    import sla_inputs
    import sparse_linear_attention_block_b200 as slab

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    over = {"with_grad": True}
    if args.k_h is not None:
        over["k_h"] = args.k_h
    wl = sla_inputs.make(args.workload, seed=rank, **over)
    shape = slab.make_shape(wl.B, wl.H, wl.N, wl.d, wl.block, wl.k_h, wl.k_l,
                            n_valid=wl.n_valid if args.key_padding else 0)
    buf = slab.Buffers.allocate(shape, device=dev, with_logits=False)
    n_crit = buf.sizes.n_crit
    to_dev = lambda a: torch.from_numpy(a).to(torch.bfloat16).to(dev)
    q, k, v, w, do = (to_dev(x) for x in (wl.q, wl.k, wl.v, wl.w_proj, wl.d_o))
    o = torch.empty_like(q)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk, dv = torch.empty_like(dq), torch.empty_like(dq)
    dw = torch.empty(w.shape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    gate = None if args.gate_logit is None else slab.Gate(args.gate_logit, args.gate_skip)
    d_logit = torch.empty(1, dtype=torch.float32, device=dev)

    hier = slab.Hierarchy(args.hierarchical, 0, 0) if args.hierarchical else None

    def step(qq=q, kk=k, vv=v, ww=w, dd=do):
        if hier is None:
            slab.sla_classify(shape, qq, kk, buf.mask, buf.workspace, stream)
        else:
            slab.sla_classify_hierarchical(shape, qq, kk, hier, buf.mask, None, buf.workspace,
                                           stream)
        if gate is None:
            slab.sla_forward(shape, qq, kk, vv, ww, buf.mask, o, buf.saved, buf.workspace,
                             stream)
            slab.sla_backward(shape, qq, kk, vv, ww, buf.mask, buf.saved, dd, dq, dk, dv, dw,
                              buf.workspace, stream)
        else:
            slab.sla_forward_gated(shape, qq, kk, vv, ww, buf.mask, gate, o, buf.saved,
                                   buf.workspace, stream)
            slab.sla_backward_gated(shape, qq, kk, vv, ww, buf.mask, gate, buf.saved, dd, dq, dk,
                                    dv, dw, d_logit, buf.workspace, stream)

    barrier = lambda: rank_barrier(world)
    max_over_ranks = lambda x: max_over_ranks_of(x, world, dev)

    for _ in range(args.warmup):
        step()
    slab.sla_check(buf.workspace, stream)
    torch.cuda.synchronize()
    barrier()

    # ------------------------------------------------------------ timed region
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    slab.sla_check(buf.workspace, stream)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    clocks = clk.summary()

    fwd_flops, bwd_flops = executed_block_flops(wl, n_crit)
    value = whole_job_tflops(fwd_flops + bwd_flops, ms, world)

    # ------------------------------------------------------------ per-kernel times
    slab.sla_profile_begin()
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    prof = slab.sla_profile_end()
    # each profiled call is one kernel launch, except the CSR build (count, scan
    # and, when there are critical blocks, fill kernels)
    kernels_per_call = {"crit_csr": 3 if n_crit > 0 else 2}
    launches_per_step = sum(n * kernels_per_call.get(name, 1)
                            for name, (n, _) in prof.items()) / args.steps
    pk, src = peaks()
    work = kernel_work(wl, n_crit)
    per_kernel = {name: {"launches": n, "ms_per_launch": tot / n,
                         "share": tot / sum(t for _, t in prof.values())}
                  for name, (n, tot) in prof.items()}
    capped_k = bool(clocks) and "sw_power_cap" in clocks.get("reasons", [])
    for name, rec in per_kernel.items():
        if name in work:
            kk, amt = work[name]
            sec = rec["ms_per_launch"] * 1e-3
            if kk == "tensor":
                rec["tflops"] = amt / sec / 1e12
                rec["frac_of_peak"] = rec["tflops"] / (pk["bf16_tflops_sustained"] if capped_k
                                                       else pk["bf16_tflops"])
            else:
                rec["gbs"] = amt / sec / 1e9
                rec["frac_of_peak"] = rec["gbs"] / pk["hbm_gbs"]
    dominant = max(prof, key=lambda n: prof[n][1])
    kind, amount = work.get(dominant, ("tensor", 0))
    traffic = (NCU_DRAM_BYTES_PER_HEAD[dominant] * wl.B * wl.H
               if dominant in NCU_DRAM_BYTES_PER_HEAD and args.workload == "train" else None)
    avg_s = prof[dominant][1] / prof[dominant][0] * 1e-3
    # the tensor peak: the burst figure (a kernel timed at full clock, as the
    # clock record of the timed region shows), the sustained one (measured under
    # the power cap) beside it
    capped = bool(clocks) and "sw_power_cap" in clocks.get("reasons", [])
    tensor_peak = pk["bf16_tflops_sustained"] if capped else pk["bf16_tflops"]
    tensor_src = f"{src} bf16 cuBLAS " + ("sustained (power cap seen)" if capped else "burst")
    if kind == "tensor":
        achieved = amount / avg_s / 1e12
        peak = tensor_peak
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "frac_of_burst": achieved / pk["bf16_tflops"],
                "frac_of_sustained": achieved / pk["bf16_tflops_sustained"],
                "traffic": traffic, "kernel": dominant, "peak_source": tensor_src}
    else:
        achieved = amount / avg_s / 1e9
        peak = pk["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic, "kernel": dominant,
                "peak_source": f"{src} HBM copy"}
    fwd_ms = sum(prof[n][1] for n in ("summaries", "expand_marginal", "aggregate",
                                      "fwd_sparse", "fwd_linear", "os_to_o")
                 if n in prof) / args.steps
    cls_ms = sum(prof[n][1] for n in ("pool", "classify", "coarse_keys", "hier_classify",
                                      "crit_csr") if n in prof) / args.steps
    bwd_ms = sum(t for n, (_, t) in prof.items()) / args.steps - fwd_ms - cls_ms

    # ------------------------------------------------------------ end to end
    e2e = None
    if not args.no_e2e:
        hosts = [torch.from_numpy(x).to(torch.bfloat16).pin_memory()
                 for x in (wl.q, wl.k, wl.v, wl.w_proj, wl.d_o)]
        # two device input sets: step i's inputs cross PCIe on a copy stream
        # while step i-1 computes (every copy is inside the timed region)
        sets = [[torch.empty_like(h, device=dev) for h in hosts] for _ in range(2)]
        copy_stream = torch.cuda.Stream(dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        used = [torch.cuda.Event() for _ in range(2)]
        dw_host = torch.empty(dw.shape, dtype=torch.float32).pin_memory()
        h2d = sum(h.numel() * h.element_size() for h in hosts)
        d2h = dw_host.numel() * dw_host.element_size()

        def e2e_run(nsteps, start=None):
            if start is not None:
                copy_stream.wait_event(start)
            for i in range(nsteps):
                b = i % 2
                with torch.cuda.stream(copy_stream):
                    if i >= 2:
                        copy_stream.wait_event(used[b])
                    for hsrc, ddst in zip(hosts, sets[b]):
                        ddst.copy_(hsrc, non_blocking=True)
                    copied[b].record(copy_stream)
                stream.wait_event(copied[b])
                step(*sets[b])
                used[b].record(stream)
                dw_host.copy_(dw, non_blocking=True)  # the step's result back to the host

        e2e_run(3)
        torch.cuda.synchronize()
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        e2e_run(args.steps, start=a0)
        a1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a0.elapsed_time(a1) / args.steps)
        e2e = {"value": whole_job_tflops(fwd_flops + bwd_flops, e_ms, world),
               "unit": "TFLOP/s", "ms_per_step": e_ms, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}

    # ------------------------------------------------------------ CPU oracle baseline
    cpu = None
    default_run = args.workload == "train" and args.k_h is None and not args.hierarchical
    if rank == 0 and world == 1 and not args.no_cpu_baseline and default_run:
        tfl, sec = time_oracle(wl, [0, 1, 2], 1, 0)
        cpu = {"value": tfl, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"heads 0-2 of 12 of this workload, one classify+forward+backward "
                         f"step of the fp64 oracle ({sec:.1f} s), executed-block FLOPs of "
                         f"those heads"}

    dense = None
    if rank == 0 and world == 1 and not args.no_dense and args.workload == "train":
        dense = dense_sdpa_context(wl.B, wl.H, wl.N, wl.d, dev)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    peak_t = pk["bf16_tflops_sustained"] if (clocks and "sw_power_cap" in clocks.get("reasons", [])) \
        else pk["bf16_tflops"]
    cfg = workload_config(wl, n_crit)
    if args.key_padding:
        cfg["n_valid"] = wl.n_valid
    if hier is not None:
        TG, c_hi, c_lo = slab.sla_hierarchy_counts(shape, hier)
        cfg["classification"] = {"hierarchical_group": args.hierarchical, "super_blocks": TG,
                                 "critical_candidates": c_hi, "negligible_candidates": c_lo}
    if gate is not None:
        g = 1.0 / (1.0 + math.exp(-args.gate_logit))
        cfg["gate"] = {"logit": args.gate_logit, "skip_below": args.gate_skip, "g": g,
                       "linear_branch_dropped": g < args.gate_skip}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": cfg,
        "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "classify_ms": cls_ms,
        "fwd_tflops": fwd_flops / (fwd_ms * 1e-3) / 1e12,
        "bwd_tflops": bwd_flops / (bwd_ms * 1e-3) / 1e12,
        "frac_of_bf16_peak": value / world / peak_t,
        "dense_attention_context": dense,
        "kernels": per_kernel, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "clocks": clocks, "gpu_launches": int(round(launches_per_step * args.steps)),
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
