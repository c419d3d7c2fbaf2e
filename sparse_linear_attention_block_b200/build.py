"""Build libsla.so (the C-ABI library) in-tree for sm_100a with nvcc.

    python -m sparse_linear_attention_block_b200.build [--force] [--ptxas]

Each source compiles to its own object under ``_build/`` (in parallel, and only
when the source or a header is newer than its object); the objects are then
linked into ``libsla.so``.  The library depends only on the CUDA runtime
(linked statically) and the driver entry point for TMA descriptor encoding; it
does not link torch.
"""

from __future__ import annotations

import concurrent.futures
import os
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ_DIR = os.path.join(PKG_DIR, "_build")
LIB = os.path.join(PKG_DIR, "libsla.so")

SOURCES = ["sla_api.cu", "sla_classify.cu", "sla_linear.cu", "sla_fwd_linear.cu",
           "sla_sparse_fwd.cu", "sla_bwd_linear.cu", "sla_sparse_bwd.cu", "sla_noalloc.cu"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = ARCH + [
    "-O3", "-lineinfo", "-std=c++17",
    "--use_fast_math",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
]
LINK_FLAGS = ARCH + ["-shared"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _includes(path: str, seen: set) -> set:
    """The project headers `path` includes, transitively."""
    try:
        with open(path) as f:
            lines = f.readlines()
    except OSError:
        return seen
    for ln in lines:
        ln = ln.strip()
        if ln.startswith("#include \""):
            name = ln.split('"')[1]
            for d in (CSRC, INCLUDE):
                dep = os.path.join(d, name)
                if os.path.exists(dep) and dep not in seen:
                    seen.add(dep)
                    _includes(dep, seen)
                    break
    return seen


def _deps_mtime(path: str) -> float:
    return max([os.path.getmtime(path)] + [os.path.getmtime(h) for h in _includes(path, set())])


def _obj(src: str) -> str:
    return os.path.join(OBJ_DIR, os.path.splitext(src)[0] + ".o")


def _stale_objects(force: bool) -> list:
    out = []
    for src in SOURCES:
        path, obj = os.path.join(CSRC, src), _obj(src)
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < _deps_mtime(path):
            out.append(src)
    return out


def _compile(src: str, extra, verbose: bool) -> str:
    cmd = [nvcc(), *COMPILE_FLAGS, "-I", INCLUDE, "-I", CSRC, *(extra or []), "-c",
           os.path.join(CSRC, src), "-o", _obj(src) + ".tmp"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n" + res.stdout + res.stderr)
    os.replace(_obj(src) + ".tmp", _obj(src))
    return (" ".join(cmd) + "\n" if verbose else "") + res.stdout + res.stderr


def build(force: bool = False, verbose: bool = False, extra=None) -> str:
    """Compile the objects whose sources or headers changed and link the
    library if anything is newer than it; return its path."""
    os.makedirs(OBJ_DIR, exist_ok=True)
    todo = _stale_objects(force)
    if todo:
        workers = min(len(todo), os.cpu_count() or 1)
        with concurrent.futures.ThreadPoolExecutor(workers) as ex:
            for log in ex.map(lambda s: _compile(s, extra, verbose), todo):
                if verbose and log:
                    print(log, flush=True)
    objs = [_obj(s) for s in SOURCES]
    if todo or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(map(os.path.getmtime, objs)):
        cmd = [nvcc(), *LINK_FLAGS, "-o", LIB + ".tmp", *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc link failed:\n" + res.stdout + res.stderr)
        os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas" in sys.argv else None)
