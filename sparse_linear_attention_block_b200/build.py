"""Build libsla.so (the C-ABI library) in-tree for sm_100a with nvcc.

    python -m sparse_linear_attention_block_b200.build [--verbose]

The library depends only on the CUDA runtime (linked statically) and the
driver entry point for TMA descriptor encoding; it does not link torch.
"""

from __future__ import annotations

import os
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG_DIR, "libsla.so")

SOURCES = ["sla_api.cu", "sla_classify.cu", "sla_linear.cu", "sla_fwd_linear.cu",
           "sla_sparse_fwd.cu", "sla_bwd_linear.cu", "sla_sparse_bwd.cu", "sla_noalloc.cu"]
HEADERS = ["sla_internal.h", "sla_ptx.cuh", "sla_tile.cuh", "sla_union.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--use_fast_math",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "sla.h")]
    return any(os.path.getmtime(f) > t for f in deps if os.path.exists(f))


def build(force: bool = False, verbose: bool = False, extra=None) -> str:
    """Compile the library if any source is newer than it; return its path."""
    if not force and not _stale():
        return LIB
    srcs = [os.path.join(CSRC, f) for f in SOURCES if os.path.exists(os.path.join(CSRC, f))]
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, *(extra or []), "-o", LIB + ".tmp",
           *srcs]
    cmd = [c for c in cmd if c]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas" in sys.argv else None)
