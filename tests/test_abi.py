"""Host-side checks of the C ABI: the library builds and loads, exports every
symbol ``include/sla.h`` declares, sizes buffers, and rejects bad arguments
before touching the device (none of these calls launches anything)."""

import ctypes
import os
import re

import pytest

import sparse_linear_attention_block_b200 as slab
from sparse_linear_attention_block_b200 import build as slab_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "sla.h")


@pytest.fixture(scope="module")
def L():
    slab_build.build()
    return slab.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SLA_API\s+[\w\s\*]+?\b(sla_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_symbols() == sorted(slab.EXPORTED_SYMBOLS)


def test_every_declared_symbol_is_exported(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
    # nothing internal leaks out of the shared object
    out = os.popen(f"nm -D --defined-only {slab.lib_path}").read()
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(declared_symbols()) <= exported
    assert not [s for s in exported if "sla" in s and not s.startswith("sla_")]


def test_version_and_strerror(L):
    assert re.fullmatch(r"\d+\.\d+\.\d+", slab.sla_version())
    for code in range(7):
        assert slab.sla_strerror(code) and slab.sla_strerror(code) != "unknown status"
    assert slab.sla_strerror(99) == "unknown status"


def test_query_sizes_wan_shape(L):
    s = slab.sla_query_sizes(slab.make_shape(1, 12, 32768, 128, 64, 0.05, 0.10))
    assert (s.T, s.n_crit, s.n_negl, s.n_marg) == (512, 26, 51, 435)
    assert s.cls_bytes == 12 * 512 * 512
    assert s.crit_idx_bytes == 12 * 512 * 26 * 4
    assert s.marg_bits_bytes == 12 * 512 * 16 * 4
    assert s.o_s_bytes == 12 * 32768 * 128 * 4
    assert s.hz_agg_bytes == 12 * 512 * (128 * 128 + 128) * 4
    assert s.workspace_bytes > 0


@pytest.mark.parametrize("T,k_h,k_l", [(16, 0.25, 0.25), (128, 0.05, 0.10), (1182, 0.025, 0.10),
                                       (1182, 0.10, 0.10), (7, 0.5, 0.5), (10, 0.1, 0.9)])
def test_query_sizes_counts_match_oracle(L, T, k_h, k_l):
    import oracle
    s = slab.sla_query_sizes(slab.make_shape(1, 1, 64 * T, 64, 64, k_h, k_l))
    assert (s.n_crit, s.n_negl) == oracle.block_counts(T, k_h, k_l)


@pytest.mark.parametrize("kw,code", [
    (dict(N=1000), 1),            # N % block != 0
    (dict(block=32, N=1024), 2),  # block != 64
    (dict(d=96), 2),              # unsupported head dim
    (dict(k_h=0.7, k_l=0.4), 1),  # k_h + k_l > 1
    (dict(k_h=-0.1), 1),
    (dict(B=0), 1),
    (dict(N=64 * 4097), 2),       # too many blocks
    (dict(softmax_scale=float("nan")), 1),
])
def test_query_sizes_rejects(L, kw, code):
    args = dict(B=1, H=2, N=1024, d=64, block=64, k_h=0.25, k_l=0.25, softmax_scale=0.0)
    args.update(kw)
    with pytest.raises(slab.SlaError) as e:
        slab.sla_query_sizes(slab.make_shape(**args))
    assert e.value.status == code


def test_entry_points_reject_bad_arguments_without_launching(L):
    sh = slab.make_shape(1, 2, 1024, 64, 64, 0.25, 0.25)
    shp = ctypes.byref(sh)
    m = slab.MaskStruct()
    sv = slab.SavedStruct()
    # null pointers -> invalid argument, before any CUDA call
    assert L.sla_classify(shp, None, None, ctypes.byref(m), None, 0, None) == 1
    assert L.sla_classify_from_scores(shp, None, ctypes.byref(m), None, 0, None) == 1
    assert L.sla_forward(shp, None, None, None, None, ctypes.byref(m), None, ctypes.byref(sv),
                         None, 0, None) == 1
    assert L.sla_backward(shp, None, None, None, None, ctypes.byref(m), ctypes.byref(sv), None,
                          None, None, None, None, None, 0, None) == 1
    assert L.sla_query_sizes(None, None) == 1
    assert L.sla_check(None, None) == 1
    assert L.sla_workspace_init(None, 0, None) == 1
    # misaligned pointers (never dereferenced) -> invalid argument
    fake = 0x10000001
    mk = slab.MaskStruct(fake, fake, fake, fake, fake, None)
    assert L.sla_classify(shp, fake, fake, ctypes.byref(mk), 0x100000, 1 << 40, None) == 1
    # workspace too small -> workspace error
    good = 0x7f0000000000
    mg = slab.MaskStruct(good, good, good, good, good, None)
    assert L.sla_classify(shp, good, good, ctypes.byref(mg), good, 16, None) == 3
    # unsupported shape
    sh2 = slab.make_shape(1, 2, 1024, 96, 64, 0.25, 0.25)
    assert L.sla_classify(ctypes.byref(sh2), good, good, ctypes.byref(mg), good, 1 << 40,
                          None) == 2


def test_gated_entry_points_reject_bad_gates_without_launching(L):
    sh = slab.make_shape(1, 2, 1024, 64, 64, 0.25, 0.25)
    shp = ctypes.byref(sh)
    good = 0x7f0000000000  # aligned, never dereferenced: every check fails first
    m = slab.MaskStruct(good, good, good, good, good, None)
    sv = slab.SavedStruct(good, good, good, good)
    ok_gate = slab.Gate(0.5, 0.1)
    nan_gate = slab.Gate(float("nan"), 0.1)
    nan_skip = slab.Gate(0.5, float("nan"))
    fwd = lambda gate: L.sla_forward_gated(shp, good, good, good, good, ctypes.byref(m), gate,
                                           good, ctypes.byref(sv), good, 16, None)
    assert fwd(None) == 1
    assert fwd(ctypes.byref(nan_gate)) == 1
    assert fwd(ctypes.byref(nan_skip)) == 1
    assert fwd(ctypes.byref(ok_gate)) == 3  # valid gate: the small workspace is reported
    bwd = lambda gate, d_logit: L.sla_backward_gated(
        shp, good, good, good, good, ctypes.byref(m), gate, ctypes.byref(sv), good, good, good,
        good, good, d_logit, good, 16, None)
    assert bwd(ctypes.byref(ok_gate), None) == 1
    assert bwd(ctypes.byref(ok_gate), good + 2) == 1  # d_logit must be 4-byte aligned
    assert bwd(None, good) == 1
    assert bwd(ctypes.byref(nan_gate), good) == 1
    assert bwd(ctypes.byref(ok_gate), good) == 3


@pytest.mark.parametrize("T,k_h,k_l", [(16, 0.25, 0.25), (128, 0.05, 0.10), (512, 0.05, 0.10),
                                       (1182, 0.10, 0.10), (1182, 0.025, 0.10), (10, 0.3, 0.3),
                                       (7, 0.0, 0.0)])
@pytest.mark.parametrize("group,top,bottom", [(2, 0, 0), (4, 0, 0), (16, 0, 0), (16, 12, 3),
                                              (8, 1, 40), (64, 0, 0)])
def test_hierarchy_counts_match_oracle(L, T, k_h, k_l, group, top, bottom):
    import oracle
    sh = slab.make_shape(1, 1, 64 * T, 64, 64, k_h, k_l)
    n_h, n_l = oracle.block_counts(T, k_h, k_l)
    got = slab.sla_hierarchy_counts(sh, slab.Hierarchy(group, top, bottom))
    assert got == oracle.coarse_counts(T, n_h, n_l, group, top, bottom)


def test_hierarchical_entry_points_reject_bad_arguments_without_launching(L):
    sh = slab.make_shape(1, 2, 1024, 64, 64, 0.25, 0.25)
    shp = ctypes.byref(sh)
    good = 0x7f0000000000  # aligned, never dereferenced: every check fails first
    m = slab.MaskStruct(good, good, good, good, good, None)
    n = ctypes.c_int()
    for bad in (slab.Hierarchy(1, 0, 0), slab.Hierarchy(4, -1, 0), slab.Hierarchy(4, 0, -2)):
        assert L.sla_hierarchy_counts(shp, ctypes.byref(bad), ctypes.byref(n), ctypes.byref(n),
                                      ctypes.byref(n)) == 1
        assert L.sla_classify_hierarchical(shp, good, good, ctypes.byref(bad), ctypes.byref(m),
                                           None, good, 1 << 40, None) == 1
    ok = slab.Hierarchy(4, 0, 0)
    assert L.sla_hierarchy_counts(shp, None, ctypes.byref(n), ctypes.byref(n),
                                  ctypes.byref(n)) == 1
    assert L.sla_classify_hierarchical(shp, None, good, ctypes.byref(ok), ctypes.byref(m), None,
                                       good, 1 << 40, None) == 1
    assert L.sla_classify_hierarchical(shp, good, good, ctypes.byref(ok), ctypes.byref(m),
                                       good + 4, good, 1 << 40, None) == 1  # coarse misaligned
    assert L.sla_classify_hierarchical(shp, good, good, ctypes.byref(ok), ctypes.byref(m), None,
                                       good, 16, None) == 3
    fs = lambda lg, co: L.sla_classify_hierarchical_from_scores(
        shp, lg, co, ctypes.byref(ok), ctypes.byref(m), good, 16, None)
    assert fs(good, None) == 1
    assert fs(None, good) == 1
    assert fs(good, good + 8) == 1
    assert fs(good, good) == 3
