"""Python binding of the SLA hot-path C ABI (``include/sla.h``, ``libsla.so``).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  There is no CPU fallback; if the compiled library
is missing, loading it raises.  PyTorch is used for device memory and
streams only.

The entry points mirror the C names (``sla_query_sizes``, ``sla_classify``,
``sla_classify_from_scores``, ``sla_forward``, ``sla_backward``,
``sla_workspace_init``, ``sla_check``, ``sla_strerror``, ``sla_version``) and
take torch tensors where the C ABI takes device pointers.  ``Buffers`` allocates
every caller-owned buffer for a shape with torch.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os

__all__ = [
    "SlaError", "Shape", "Sizes", "MaskStruct", "SavedStruct", "Buffers", "lib", "lib_path",
    "sla_query_sizes", "sla_classify", "sla_classify_from_scores", "sla_forward",
    "sla_backward", "sla_workspace_init", "sla_check", "sla_strerror", "sla_version",
    "sla_profile_begin", "sla_profile_end", "KernelStat", "make_shape", "EXPORTED_SYMBOLS",
    "STATUS", "Gate", "sla_forward_gated", "sla_backward_gated", "Hierarchy",
    "sla_hierarchy_counts", "sla_classify_hierarchical", "sla_classify_hierarchical_from_scores",
    "sla_debug_inject", "INJECT_WITHHOLD_LOADS",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_PKG, "libsla.so")

STATUS = {0: "SLA_OK", 1: "SLA_ERR_INVALID_ARG", 2: "SLA_ERR_UNSUPPORTED", 3: "SLA_ERR_WORKSPACE",
          4: "SLA_ERR_CUDA", 5: "SLA_ERR_TIMEOUT", 6: "SLA_ERR_DEVICE"}

EXPORTED_SYMBOLS = ["sla_query_sizes", "sla_classify", "sla_classify_from_scores",
                    "sla_forward", "sla_backward", "sla_workspace_init", "sla_check",
                    "sla_strerror", "sla_version", "sla_profile_begin", "sla_profile_end",
                    "sla_classify_noalloc", "sla_forward_gated", "sla_backward_gated",
                    "sla_hierarchy_counts", "sla_classify_hierarchical",
                    "sla_classify_hierarchical_from_scores", "sla_debug_inject"]

INJECT_WITHHOLD_LOADS = 1  # SLA_INJECT_WITHHOLD_LOADS of sla.h


class SlaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({_strerror(status)})")


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
                ("d", ctypes.c_int), ("block", ctypes.c_int), ("k_h", ctypes.c_double),
                ("k_l", ctypes.c_double), ("softmax_scale", ctypes.c_float),
                ("n_valid", ctypes.c_int)]


class MaskStruct(ctypes.Structure):
    _fields_ = [("cls", ctypes.c_void_p), ("crit_idx", ctypes.c_void_p),
                ("marg_bits", ctypes.c_void_p), ("crit_col_ptr", ctypes.c_void_p),
                ("crit_col_idx", ctypes.c_void_p), ("pooled_logits", ctypes.c_void_p)]


class SavedStruct(ctypes.Structure):
    _fields_ = [("lse", ctypes.c_void_p), ("o_s", ctypes.c_void_p), ("den", ctypes.c_void_p),
                ("hz_agg", ctypes.c_void_p)]


class Gate(ctypes.Structure):
    """sla_gate: g = sigmoid(logit); the linear branch is dropped when g < skip_below."""
    _fields_ = [("logit", ctypes.c_float), ("skip_below", ctypes.c_float)]


class Hierarchy(ctypes.Structure):
    """sla_hierarchy: super-blocks of `group` key blocks; `top` / `bottom` are
    minimum numbers of critical / negligible candidate super-blocks."""
    _fields_ = [("group", ctypes.c_int), ("top", ctypes.c_int), ("bottom", ctypes.c_int)]


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int),
                ("total_ms", ctypes.c_double)]


class Sizes(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("n_crit", ctypes.c_int), ("n_negl", ctypes.c_int),
                ("n_marg", ctypes.c_int)] + [
        (n, ctypes.c_size_t) for n in (
            "cls_bytes", "crit_idx_bytes", "marg_bits_bytes", "crit_col_ptr_bytes",
            "crit_col_idx_bytes", "pooled_logits_bytes", "lse_bytes", "o_s_bytes", "den_bytes",
            "hz_agg_bytes", "workspace_bytes")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsla.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise OSError(f"libsla.so not built at {lib_path}; run "
                          "python -m sparse_linear_attention_block_b200.build")
        L = ctypes.CDLL(lib_path)
        vp, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        P = ctypes.POINTER
        L.sla_query_sizes.argtypes = [P(Shape), P(Sizes)]
        L.sla_classify.argtypes = [P(Shape), vp, vp, P(MaskStruct), vp, sz, vp]
        L.sla_classify_from_scores.argtypes = [P(Shape), vp, P(MaskStruct), vp, sz, vp]
        L.sla_forward.argtypes = [P(Shape), vp, vp, vp, vp, P(MaskStruct), vp, P(SavedStruct),
                                  vp, sz, vp]
        L.sla_backward.argtypes = [P(Shape), vp, vp, vp, vp, P(MaskStruct), P(SavedStruct), vp,
                                   vp, vp, vp, vp, vp, sz, vp]
        L.sla_forward_gated.argtypes = [P(Shape), vp, vp, vp, vp, P(MaskStruct), P(Gate), vp,
                                        P(SavedStruct), vp, sz, vp]
        L.sla_backward_gated.argtypes = [P(Shape), vp, vp, vp, vp, P(MaskStruct), P(Gate),
                                         P(SavedStruct), vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sla_hierarchy_counts.argtypes = [P(Shape), P(Hierarchy), P(st), P(st), P(st)]
        L.sla_classify_hierarchical.argtypes = [P(Shape), vp, vp, P(Hierarchy), P(MaskStruct), vp,
                                                vp, sz, vp]
        L.sla_classify_hierarchical_from_scores.argtypes = [P(Shape), vp, vp, P(Hierarchy),
                                                            P(MaskStruct), vp, sz, vp]
        L.sla_workspace_init.argtypes = [vp, sz, vp]
        L.sla_check.argtypes = [vp, vp]
        L.sla_debug_inject.argtypes = [vp, st, vp]
        L.sla_strerror.argtypes = [st]
        L.sla_strerror.restype = ctypes.c_char_p
        L.sla_version.argtypes = []
        L.sla_version.restype = ctypes.c_char_p
        L.sla_classify_noalloc.argtypes = [P(Shape), vp, vp, P(MaskStruct), vp]
        L.sla_classify_noalloc.restype = st
        L.sla_profile_begin.argtypes = []
        L.sla_profile_end.argtypes = [P(KernelStat), st, P(st)]
        for n in ("sla_query_sizes", "sla_classify", "sla_classify_from_scores", "sla_forward",
                  "sla_backward", "sla_workspace_init", "sla_check", "sla_profile_begin",
                  "sla_profile_end", "sla_forward_gated", "sla_backward_gated",
                  "sla_hierarchy_counts", "sla_classify_hierarchical",
                  "sla_classify_hierarchical_from_scores", "sla_debug_inject"):
            getattr(L, n).restype = st
        _lib = L
    return _lib


def _strerror(status: int) -> str:
    try:
        return lib().sla_strerror(status).decode()
    except OSError:
        return "library not loaded"


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str):
    if status != 0:
        raise SlaError(status, what)


def make_shape(B, H, N, d, block=64, k_h=0.05, k_l=0.10, softmax_scale=0.0,
               n_valid=0) -> Shape:
    return Shape(B, H, N, d, block, float(k_h), float(k_l), float(softmax_scale), int(n_valid))


def sla_query_sizes(shape: Shape) -> Sizes:
    out = Sizes()
    _check(lib().sla_query_sizes(ctypes.byref(shape), ctypes.byref(out)), "sla_query_sizes")
    return out


def sla_strerror(status: int) -> str:
    return _strerror(status)


def sla_version() -> str:
    return lib().sla_version().decode()


def sla_profile_begin():
    _check(lib().sla_profile_begin(), "sla_profile_begin")


def sla_profile_end(max_out: int = 64) -> dict:
    """Per-kernel {name: (launches, total_ms)} since sla_profile_begin()."""
    arr = (KernelStat * max_out)()
    n = ctypes.c_int(0)
    _check(lib().sla_profile_end(arr, max_out, ctypes.byref(n)), "sla_profile_end")
    return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(n.value)}


def sla_workspace_init(workspace, stream=None):
    _check(lib().sla_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream)), "sla_workspace_init")


def sla_check(workspace, stream=None):
    _check(lib().sla_check(_ptr(workspace), _stream(stream)), "sla_check")


def sla_debug_inject(workspace, what: int, stream=None):
    """Set (what = INJECT_WITHHOLD_LOADS) or clear (what = 0) the workspace's
    fault-injection word; a test hook for the device-side timeout path."""
    _check(lib().sla_debug_inject(_ptr(workspace), int(what), _stream(stream)),
           "sla_debug_inject")


def sla_classify(shape: Shape, q, k, mask: MaskStruct, workspace, stream=None):
    _check(lib().sla_classify(ctypes.byref(shape), _ptr(q), _ptr(k), ctypes.byref(mask),
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream)), "sla_classify")


def sla_classify_noalloc(shape: Shape, q, k, mask: MaskStruct, stream=None):
    """Classification without a workspace, for callers that cannot allocate
    device memory (scratch is a fixed 16 MiB array inside the library; see
    sla.h for the size limit and the one-time per-device set-up)."""
    _check(lib().sla_classify_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k), ctypes.byref(mask),
                                      _stream(stream)), "sla_classify_noalloc")


def sla_classify_from_scores(shape: Shape, logits, mask: MaskStruct, workspace, stream=None):
    _check(lib().sla_classify_from_scores(ctypes.byref(shape), _ptr(logits), ctypes.byref(mask),
                                          _ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          _stream(stream)), "sla_classify_from_scores")


def sla_hierarchy_counts(shape: Shape, hier: Hierarchy) -> tuple[int, int, int]:
    """(TG, c_hi, c_lo) of the hierarchical selection; host only."""
    n, hi, lo = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(lib().sla_hierarchy_counts(ctypes.byref(shape), ctypes.byref(hier), ctypes.byref(n),
                                      ctypes.byref(hi), ctypes.byref(lo)),
           "sla_hierarchy_counts")
    return n.value, hi.value, lo.value


def sla_classify_hierarchical(shape: Shape, q, k, hier: Hierarchy, mask: MaskStruct,
                              coarse_logits, workspace, stream=None):
    _check(lib().sla_classify_hierarchical(ctypes.byref(shape), _ptr(q), _ptr(k),
                                           ctypes.byref(hier), ctypes.byref(mask),
                                           _ptr(coarse_logits), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(),
                                           _stream(stream)), "sla_classify_hierarchical")


def sla_classify_hierarchical_from_scores(shape: Shape, logits, coarse_logits, hier: Hierarchy,
                                          mask: MaskStruct, workspace, stream=None):
    _check(lib().sla_classify_hierarchical_from_scores(
        ctypes.byref(shape), _ptr(logits), _ptr(coarse_logits), ctypes.byref(hier),
        ctypes.byref(mask), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)), "sla_classify_hierarchical_from_scores")


def sla_forward(shape: Shape, q, k, v, w_proj, mask: MaskStruct, o, saved: SavedStruct,
                workspace, stream=None):
    _check(lib().sla_forward(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(w_proj),
                             ctypes.byref(mask), _ptr(o), ctypes.byref(saved), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)),
           "sla_forward")


def sla_backward(shape: Shape, q, k, v, w_proj, mask: MaskStruct, saved: SavedStruct, d_o,
                 dq, dk, dv, dw_proj, workspace, stream=None):
    _check(lib().sla_backward(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(w_proj),
                              ctypes.byref(mask), ctypes.byref(saved), _ptr(d_o), _ptr(dq),
                              _ptr(dk), _ptr(dv), _ptr(dw_proj), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream)),
           "sla_backward")


def sla_forward_gated(shape: Shape, q, k, v, w_proj, mask: MaskStruct, gate: Gate, o,
                      saved: SavedStruct, workspace, stream=None):
    _check(lib().sla_forward_gated(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(w_proj),
                                   ctypes.byref(mask), ctypes.byref(gate), _ptr(o),
                                   ctypes.byref(saved), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "sla_forward_gated")


def sla_backward_gated(shape: Shape, q, k, v, w_proj, mask: MaskStruct, gate: Gate,
                       saved: SavedStruct, d_o, dq, dk, dv, dw_proj, d_logit, workspace,
                       stream=None):
    _check(lib().sla_backward_gated(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(w_proj),
                                    ctypes.byref(mask), ctypes.byref(gate), ctypes.byref(saved),
                                    _ptr(d_o), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dw_proj),
                                    _ptr(d_logit), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "sla_backward_gated")


@dataclasses.dataclass
class Buffers:
    """Every caller-owned device buffer for one shape, allocated with torch.

    Attributes hold torch tensors shaped as documented in ``sla.h``;
    ``mask`` and ``saved`` are the ctypes structs pointing at them.
    """
    shape: Shape
    sizes: Sizes
    cls: object
    crit_idx: object
    marg_bits: object
    crit_col_ptr: object
    crit_col_idx: object
    pooled_logits: object
    lse: object
    o_s: object
    den: object
    hz_agg: object
    workspace: object
    mask: MaskStruct
    saved: SavedStruct

    @classmethod
    def allocate(cls_, shape: Shape, device="cuda", with_logits=True, stream=None):
        import torch
        s = sla_query_sizes(shape)
        B, H, N, d, T = shape.B, shape.H, shape.N, shape.d, s.T
        W = (T + 31) // 32
        dev = torch.device(device)
        e = lambda *sh, dt: torch.empty(*sh, dtype=dt, device=dev)
        nc = max(s.n_crit, 1)
        b = cls_(
            shape=shape, sizes=s,
            cls=e(B, H, T, T, dt=torch.int8),
            crit_idx=e(B, H, T, nc, dt=torch.int32),
            marg_bits=e(B, H, T, W, dt=torch.int32),
            crit_col_ptr=e(B, H, T + 1, dt=torch.int32),
            crit_col_idx=e(B, H, T * nc, dt=torch.int32),
            pooled_logits=e(B, H, T, T, dt=torch.float32) if with_logits else None,
            lse=e(B, H, N, dt=torch.float32),
            o_s=e(B, H, N, d, dt=torch.float32),
            den=e(B, H, N, dt=torch.float32),
            hz_agg=e(2, B, H, T, d * d + d, dt=torch.bfloat16),  # hi plane, lo plane
            workspace=torch.empty(int(s.workspace_bytes) + 1024, dtype=torch.uint8, device=dev),
            mask=MaskStruct(), saved=SavedStruct())
        # the C ABI wants a 1024-byte aligned workspace
        off = (-b.workspace.data_ptr()) % 1024
        b.workspace = b.workspace[off:off + int(s.workspace_bytes)]
        b.mask = MaskStruct(_ptr(b.cls), _ptr(b.crit_idx), _ptr(b.marg_bits),
                            _ptr(b.crit_col_ptr), _ptr(b.crit_col_idx), _ptr(b.pooled_logits))
        b.saved = SavedStruct(_ptr(b.lse), _ptr(b.o_s), _ptr(b.den), _ptr(b.hz_agg))
        sla_workspace_init(b.workspace, stream)
        return b
