"""Seeded synthetic inputs for the SLA hot path.

This module is shared by the tests, the benchmark and the oracle's callers.
It holds input preparation only (random draws, a sinusoidal token-grid
feature, bf16 rounding) and none of the method's arithmetic: no pooling, no
scores, no classification, no attention.

Workloads (sizes and distributions):

* ``tiny``  B=1 H=2 N=1024 d=64, i.i.d. N(0,1) Q/K/V drawn in fp32 from seed 0
  and rounded to bf16; W_proj ~ N(0, 1/64); block 64, k_h=k_l=0.25.
* ``mid``   B=1 H=12 d=128, an 8x32x32 (t,h,w) latent grid (N=8192);
  block 64, k_h=0.05, k_l=0.10.
* ``wan``   B=1 H=12 d=128, a 21x30x52 grid (32760 tokens) zero-padded to
  N=32768; block 64, k_h=0.05, k_l=0.10.  Shaped like Wan2.1-1.3B video
  attention (the SLA paper's evaluation model); no model weights or real
  activations are used, these synthetic tensors stand in for them.
* ``long``  B=1 H=12 d=128, a 21x45x80 grid (75600 tokens) padded to 75648;
  k_h in {0.025, 0.05, 0.10}, k_l=0.10.
* ``train`` the ``wan`` inputs plus an upstream gradient dO ~ N(0,1).

Grid workloads: token n = (t*L_h + h)*L_w + w.  The feature f(n) in R^128
concatenates 1D sinusoid encodings of t (32 dims), h (48 dims) and w (48
dims); an axis with D dims uses the pairs [sin(p*w_k), cos(p*w_k)],
w_k = 10000^(-2k/D), k = 0..D/2-1, so |f|^2 = 64.  Each head draws one
projection R_h with N(0, 1/128) entries; Q = f R_h + E_q, K = f R_h + E_k,
V = f R_h + E_v with independent N(0, 0.5) noise (variances throughout), so
every entry has unit variance and nearby tokens have correlated Q/K, which
concentrates the pooled block scores.  Pad tokens are exact zeros.
W_proj ~ N(0, 1/d); dO ~ N(0, 1).  Draw order from
``numpy.random.default_rng(seed)``: R_0..R_{H-1}, E_q, E_k, E_v, W_proj, dO.
Everything is rounded to bf16 (round to nearest even) after drawing; the
float32 arrays returned hold exactly the bf16 values.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "bf16_bits",
    "bf16_round",
    "bits_to_f32",
    "grid_feature",
    "make",
    "make_iid",
    "make_grid",
]


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp32 values."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 value, returned as fp32."""
    return bits_to_f32(bf16_bits(x))


@dataclasses.dataclass
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    block: int
    k_h: float
    k_l: float
    n_valid: int
    q: np.ndarray  # float32 [B,H,N,d], bf16-exact
    k: np.ndarray
    v: np.ndarray
    w_proj: np.ndarray  # float32 [d,d], bf16-exact
    d_o: np.ndarray | None = None  # float32 [B,H,N,d], bf16-exact
    grid: tuple | None = None

    @property
    def T(self) -> int:
        return self.N // self.block

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


WORKLOADS = {
    "tiny": dict(B=1, H=2, d=64, N=1024, block=64, k_h=0.25, k_l=0.25),
    "mid": dict(B=1, H=12, d=128, grid=(8, 32, 32), block=64, k_h=0.05, k_l=0.10),
    "wan": dict(B=1, H=12, d=128, grid=(21, 30, 52), block=64, k_h=0.05, k_l=0.10),
    "long": dict(B=1, H=12, d=128, grid=(21, 45, 80), block=64, k_h=0.05, k_l=0.10),
    "train": dict(B=1, H=12, d=128, grid=(21, 30, 52), block=64, k_h=0.05, k_l=0.10,
                  with_grad=True),
}


def _axis_encoding(pos: np.ndarray, dims: int) -> np.ndarray:
    k = np.arange(dims // 2, dtype=np.float64)
    omega = 10000.0 ** (-2.0 * k / dims)
    ang = pos[:, None].astype(np.float64) * omega[None, :]
    out = np.empty((pos.shape[0], dims), dtype=np.float64)
    out[:, 0::2] = np.sin(ang)
    out[:, 1::2] = np.cos(ang)
    return out


def grid_feature(grid: tuple) -> np.ndarray:
    """The 128-dim token-grid feature f(n) for a (t,h,w) grid, w fastest."""
    Lt, Lh, Lw = grid
    t, h, w = np.meshgrid(np.arange(Lt), np.arange(Lh), np.arange(Lw), indexing="ij")
    t, h, w = t.reshape(-1), h.reshape(-1), w.reshape(-1)
    return np.concatenate(
        [_axis_encoding(t, 32), _axis_encoding(h, 48), _axis_encoding(w, 48)], axis=1
    )


def _pad_to(n: int, block: int) -> int:
    return ((n + block - 1) // block) * block


def make_grid(grid, B=1, H=12, d=128, block=64, k_h=0.05, k_l=0.10, seed=0,
              with_grad=False, name="grid", n_tokens=None) -> Workload:
    """Sinusoid-grid workload; ``n_tokens`` keeps only the first tokens
    (the "slice" of a larger grid), run as a standalone problem."""
    if d != 128:
        raise ValueError("the grid feature is 128-dimensional")
    rng = np.random.default_rng(seed)
    f = grid_feature(grid)  # [n_valid, 128] fp64
    if n_tokens is not None:
        f = f[:n_tokens]
    n_valid = f.shape[0]
    N = _pad_to(n_valid, block)
    R = [rng.normal(0.0, math.sqrt(1.0 / 128.0), size=(128, d)) for _ in range(H)]
    shape = (B, H, N, d)

    def noise():
        return rng.normal(0.0, math.sqrt(0.5), size=(B, H, n_valid, d))

    signal = np.stack([f @ R[h] for h in range(H)])[None]  # [1,H,n_valid,d]
    outs = []
    for _ in range(3):
        x = np.zeros(shape, dtype=np.float32)
        x[:, :, :n_valid, :] = (signal + noise()).astype(np.float32)
        outs.append(bf16_round(x))
    q, k, v = outs
    w = bf16_round(rng.normal(0.0, math.sqrt(1.0 / d), size=(d, d)).astype(np.float32))
    d_o = None
    if with_grad:
        d_o = bf16_round(rng.normal(0.0, 1.0, size=shape).astype(np.float32))
    return Workload(name, B, H, N, d, block, k_h, k_l, n_valid, q, k, v, w, d_o, grid)


def make_iid(B=1, H=2, N=1024, d=64, block=64, k_h=0.25, k_l=0.25, seed=0,
             with_grad=False, name="iid") -> Workload:
    """i.i.d. N(0,1) Q/K/V (fp32 draws rounded to bf16); W_proj ~ N(0, 1/d)."""
    rng = np.random.default_rng(seed)
    shape = (B, H, N, d)
    q, k, v = (bf16_round(rng.standard_normal(shape, dtype=np.float32)) for _ in range(3))
    w = bf16_round((rng.standard_normal((d, d), dtype=np.float32) / np.float32(math.sqrt(d))))
    d_o = bf16_round(rng.standard_normal(shape, dtype=np.float32)) if with_grad else None
    return Workload(name, B, H, N, d, block, k_h, k_l, N, q, k, v, w, d_o, None)


def make(name: str, seed: int = 0, **overrides) -> Workload:
    """Build one of the named workloads; keyword overrides replace fields
    (for example ``k_h`` for the long-sequence sparsity sweep)."""
    cfg = dict(WORKLOADS[name])
    cfg.update(overrides)
    if "grid" in cfg:
        grid = cfg.pop("grid")
        return make_grid(grid, seed=seed, name=name, **cfg)
    cfg.pop("with_grad", None)
    return make_iid(seed=seed, name=name, with_grad=overrides.get("with_grad", False), **{
        k: v for k, v in cfg.items() if k != "with_grad"})
