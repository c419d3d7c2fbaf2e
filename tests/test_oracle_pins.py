"""Pins for the fp64 oracle: each test checks it against something other than
itself (a library routine, a closed form, a brute force, finite differences
or an invariant), chosen so that a dropped term, a wrong sign or index, or a
transposed operand fails at least one of them."""

import math

import numpy as np
import pytest
import torch

import oracle
import sla_inputs


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------- counts (R3)

@pytest.mark.parametrize("T,k_h,k_l,expect", [
    (16, 0.25, 0.25, (4, 4)),      # tiny
    (128, 0.05, 0.10, (7, 12)),    # mid
    (512, 0.05, 0.10, (26, 51)),   # Wan-shaped
    (1182, 0.025, 0.10, (30, 118)),
    (1182, 0.05, 0.10, (60, 118)),
    (1182, 0.10, 0.10, (119, 118)),
    (10, 0.0, 0.0, (0, 0)),
    (10, 1.0, 0.0, (10, 0)),
    (10, 0.0, 1.0, (0, 10)),
    (10, 0.1, 0.9, (1, 9)),
    (7, 0.5, 0.5, (4, 3)),         # n_l clipped to T - n_h
])
def test_block_counts(T, k_h, k_l, expect):
    assert oracle.block_counts(T, k_h, k_l) == expect


def test_block_counts_rejects_bad_fractions():
    with pytest.raises(ValueError):
        oracle.block_counts(10, 0.6, 0.5)
    with pytest.raises(ValueError):
        oracle.block_counts(10, -0.1, 0.5)


# ---------------------------------------------------------------- classification

@pytest.mark.parametrize("T", [1, 2, 5, 16, 33])
@pytest.mark.parametrize("frac", [(0.0, 0.0), (0.25, 0.25), (0.5, 0.5), (1.0, 0.0), (0.1, 0.6)])
def test_classify_matches_rank_count(T, frac):
    n_h, n_l = oracle.block_counts(T, *frac)
    rng = np.random.default_rng(T * 100 + int(frac[0] * 10))
    # small integer scores force many ties; -0.0 and 0.0 must tie as well
    rows = rng.integers(-3, 4, size=(6, T)).astype(np.float64)
    rows[0, ::2] = -0.0
    got = oracle.classify(rows, n_h, n_l)
    for r in range(rows.shape[0]):
        assert got[r].tolist() == oracle.classify_rows_bruteforce(rows[r].tolist(), n_h, n_l)
        assert (got[r] == 1).sum() == n_h and (got[r] == -1).sum() == n_l


def test_classify_ranks_softmax_like_logits():
    # ranking the row softmax (the pooled probabilities) gives the same classes
    rows = _rand((20, 64), 1, 2.0)
    p = np.exp(rows - rows.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    assert np.array_equal(oracle.classify(rows, 5, 9), oracle.classify(p, 5, 9))


def test_classify_rejects_nan():
    with pytest.raises(ValueError):
        oracle.classify(np.array([[0.0, np.nan]]), 1, 0)


def test_pool_is_block_mean():
    x = _rand((1, 1, 8, 3), 2)
    got = oracle.pool(x, 4)
    assert np.allclose(got[0, 0, 0], x[0, 0, :4].sum(0) / 4)
    assert np.allclose(got[0, 0, 1], x[0, 0, 4:].sum(0) / 4)


def test_pooled_logits_closed_form():
    q, k = _rand((1, 1, 4, 2), 3), _rand((1, 1, 4, 2), 4)
    s = oracle.pooled_logits(q, k, 2, 0.5)
    qb = [(q[0, 0, 0] + q[0, 0, 1]) / 2, (q[0, 0, 2] + q[0, 0, 3]) / 2]
    kb = [(k[0, 0, 0] + k[0, 0, 1]) / 2, (k[0, 0, 2] + k[0, 0, 3]) / 2]
    for i in range(2):
        for j in range(2):
            assert math.isclose(s[0, 0, i, j], 0.5 * float(qb[i] @ kb[j]), rel_tol=1e-12)


def test_phi_closed_form():
    x = np.array([-2.0, -0.5, 0.0, 0.5, 3.0])
    assert np.allclose(oracle.phi(x), [math.exp(-2), math.exp(-0.5), 1.0, 1.5, 4.0])
    assert np.allclose(oracle.phi_prime(x), [math.exp(-2), math.exp(-0.5), 1.0, 1.0, 1.0])
    # elu(x) + 1 from torch's own elu
    xt = torch.tensor(x)
    assert np.allclose(oracle.phi(x), (torch.nn.functional.elu(xt) + 1).numpy())


# ---------------------------------------------------------------- forward special cases

def _small(B=1, H=2, N=256, d=16, seed=0):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, H, N, d))
    k = g.standard_normal((B, H, N, d))
    v = g.standard_normal((B, H, N, d))
    w = g.standard_normal((d, d)) / math.sqrt(d)
    return q, k, v, w


def _cls_from(q, k, block, k_h, k_l):
    T = q.shape[2] // block
    n_h, n_l = oracle.block_counts(T, k_h, k_l)
    return oracle.classify(oracle.pooled_logits(q, k, block, 1 / math.sqrt(q.shape[-1])), n_h, n_l)


def test_all_critical_is_dense_softmax_attention():
    q, k, v, w = _small(N=256, d=16)
    out = oracle.sla(q, k, v, w, 32, 1.0, 0.0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k), torch.tensor(v)).numpy()
    assert np.all(out["cls"] == 1)
    np.testing.assert_allclose(out["o"], ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out["o_s"], ref, rtol=1e-10, atol=1e-12)
    assert np.all(out["o_l"] == 0)


def test_all_marginal_is_dense_linear_attention():
    q, k, v, w = _small(N=256, d=16, seed=5)
    out = oracle.sla(q, k, v, w, 32, 0.0, 0.0)
    assert np.all(out["cls"] == 0)
    # Katharopoulos-style normalised linear attention with an explicit N x N
    # kernel matrix, computed with torch (elu + 1 feature map)
    tq, tk, tv, tw = (torch.tensor(a) for a in (q, k, v, w))
    fq = torch.nn.functional.elu(tq) + 1
    fk = torch.nn.functional.elu(tk) + 1
    A = fq @ fk.transpose(-1, -2)
    lin = (A @ tv) / A.sum(-1, keepdim=True)
    np.testing.assert_allclose(out["o_l"], lin.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out["o"], (lin @ tw).numpy(), rtol=1e-10, atol=1e-12)
    assert np.all(out["o_s"] == 0)


def test_all_negligible_gives_zero():
    q, k, v, w = _small(N=128, d=8, seed=6)
    out = oracle.sla(q, k, v, w, 16, 0.0, 1.0)
    assert np.all(out["cls"] == -1)
    assert np.all(out["o"] == 0)
    assert np.all(np.isneginf(out["lse"]))


def test_zero_projection_leaves_sparse_output():
    q, k, v, w = _small(N=256, d=16, seed=7)
    out = oracle.sla(q, k, v, np.zeros_like(w), 32, 0.25, 0.25)
    assert np.array_equal(out["o"], out["o_s"])
    assert np.abs(out["o_l"]).max() > 0


def test_projection_is_right_multiplied():
    # W_proj a cyclic column shift: O - O_s must be O_l with its columns rotated
    q, k, v, _ = _small(N=256, d=16, seed=8)
    d = 16
    w = np.zeros((d, d))
    for a in range(d):
        w[a, (a + 3) % d] = 1.0
    out = oracle.sla(q, k, v, w, 32, 0.25, 0.25)
    np.testing.assert_allclose(out["o"] - out["o_s"], np.roll(out["o_l"], 3, axis=-1),
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("block,k_h,k_l", [(64, 0.25, 0.25), (16, 0.25, 0.25),
                                           (16, 0.1, 0.5), (32, 0.0, 0.25)])
def test_blockwise_equals_bruteforce(block, k_h, k_l):
    q, k, v, w = _small(B=1, H=1, N=256, d=8, seed=block)
    cls = _cls_from(q, k, block, k_h, k_l)
    fast = oracle.forward(q, k, v, w, cls, block)["o"]
    slow = oracle.forward_bruteforce(q, k, v, w, cls, block)
    np.testing.assert_allclose(fast, slow, rtol=1e-10, atol=1e-12)


def test_query_block_subset_matches_full():
    q, k, v, w = _small(N=256, d=16, seed=9)
    cls = _cls_from(q, k, 32, 0.25, 0.25)
    full = oracle.forward(q, k, v, w, cls, 32)
    part = oracle.forward(q, k, v, w, cls, 32, query_blocks=[1, 6])
    for i in (1, 6):
        sl = slice(i * 32, (i + 1) * 32)
        np.testing.assert_array_equal(part["o"][:, :, sl], full["o"][:, :, sl])


def test_in_block_token_permutation():
    q, k, v, w = _small(N=256, d=16, seed=10)
    block = 32
    rng = np.random.default_rng(11)
    perm = np.concatenate([i * block + rng.permutation(block) for i in range(256 // block)])
    base = oracle.sla(q, k, v, w, block, 0.25, 0.25)
    # permuting keys/values inside their blocks changes nothing
    kv = oracle.sla(q, k[:, :, perm], v[:, :, perm], w, block, 0.25, 0.25)
    assert np.array_equal(kv["cls"], base["cls"])
    np.testing.assert_allclose(kv["o"], base["o"], rtol=1e-10, atol=1e-12)
    # permuting queries inside their blocks permutes the output rows
    qp = oracle.sla(q[:, :, perm], k, v, w, block, 0.25, 0.25)
    assert np.array_equal(qp["cls"], base["cls"])
    np.testing.assert_allclose(qp["o"], base["o"][:, :, perm], rtol=1e-10, atol=1e-12)


def test_key_shift_invariance_of_sparse_branch():
    q, k, v, w = _small(N=256, d=16, seed=12)
    c = np.random.default_rng(13).standard_normal(16) * 3
    a = oracle.sla(q, k, v, w, 32, 0.25, 0.25)
    b = oracle.sla(q, k + c, v, w, 32, 0.25, 0.25)
    assert np.array_equal(a["cls"], b["cls"])
    np.testing.assert_allclose(a["o_s"], b["o_s"], rtol=1e-9, atol=1e-12)


def test_output_linear_in_v_with_mask_fixed():
    q, k, v, w = _small(N=256, d=16, seed=14)
    v2 = np.random.default_rng(15).standard_normal(v.shape)
    cls = _cls_from(q, k, 32, 0.25, 0.25)
    f = lambda vv: oracle.forward(q, k, vv, w, cls, 32)["o"]
    np.testing.assert_allclose(f(v + 2.5 * v2), f(v) + 2.5 * f(v2), rtol=1e-9, atol=1e-11)


def test_summaries_closed_form():
    k = _rand((1, 1, 4, 3), 16)
    v = _rand((1, 1, 4, 3), 17)
    h, z = oracle.key_block_summaries(k, v, 2)
    for j in range(2):
        hh = np.zeros((3, 3))
        zz = np.zeros(3)
        for u in (2 * j, 2 * j + 1):
            fk = [kk + 1 if kk > 0 else math.exp(kk) for kk in k[0, 0, u]]
            zz += fk
            for a in range(3):
                for c in range(3):
                    hh[a, c] += fk[a] * v[0, 0, u, c]
        np.testing.assert_allclose(h[0, 0, j], hh, rtol=1e-12)
        np.testing.assert_allclose(z[0, 0, j], zz, rtol=1e-12)


# ---------------------------------------------------------------- backward

def _loss(q, k, v, w, cls, do, block):
    return float(np.sum(oracle.forward(q, k, v, w, cls, block)["o"] * do))


@pytest.mark.parametrize("block,k_h,k_l,d", [(64, 0.25, 0.25, 8), (16, 0.25, 0.25, 8),
                                             (16, 0.1, 0.3, 4)])
def test_backward_matches_central_differences(block, k_h, k_l, d):
    q, k, v, w = _small(B=1, H=1, N=256, d=d, seed=20 + block)
    do = np.random.default_rng(21).standard_normal(q.shape)
    cls = _cls_from(q, k, block, k_h, k_l)  # frozen at the unperturbed point
    assert set(np.unique(cls)) == {-1, 0, 1}
    g = oracle.backward(q, k, v, w, cls, do, block)
    rng = np.random.default_rng(22)
    eps = 1e-6
    for name, arr, grad in (("q", q, g["dq"]), ("k", k, g["dk"]),
                            ("v", v, g["dv"]), ("w", w, g["dw"])):
        for _ in range(12):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            xp, xm = arr.copy(), arr.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v, "w": w}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd = (_loss(args_p["q"], args_p["k"], args_p["v"], args_p["w"], cls, do, block)
                  - _loss(args_m["q"], args_m["k"], args_m["v"], args_m["w"], cls, do, block)) / (2 * eps)
            assert math.isclose(fd, grad[idx], rel_tol=2e-6, abs_tol=2e-8), (name, idx, fd, grad[idx])


def test_sparse_key_gradient_sums_to_zero():
    # with no marginal pairs only the softmax branch carries gradient, and its
    # invariance under K -> K + c makes the key gradients sum to zero
    q, k, v, w = _small(N=256, d=16, seed=30)
    do = np.random.default_rng(31).standard_normal(q.shape)
    cls = _cls_from(q, k, 32, 0.5, 0.5)
    assert not np.any(cls == 0)
    g = oracle.backward(q, k, v, w, cls, do, 32)
    np.testing.assert_allclose(g["dk"].sum(axis=2), 0.0, atol=1e-10)
    assert np.all(g["dw"] == 0)


def test_workload_generators_shapes_and_stats():
    t = sla_inputs.make("tiny")
    assert t.q.shape == (1, 2, 1024, 64) and t.w_proj.shape == (64, 64)
    assert np.array_equal(sla_inputs.bf16_round(t.q), t.q)
    g = sla_inputs.make_grid((2, 8, 8), H=2, name="g")
    assert g.N == 128 and g.n_valid == 128
    f = sla_inputs.grid_feature((2, 3, 4))
    np.testing.assert_allclose((f ** 2).sum(1), 64.0)
    # zero padding past the grid
    p = sla_inputs.make_grid((1, 3, 7), H=1, name="p")
    assert p.N == 64 and p.n_valid == 21 and np.all(p.q[:, :, 21:] == 0)


# ---------------------------------------------------------------- gated linear branch (R12)

def test_gate_factor_closed_form():
    assert oracle.gate_factor(None) == (1.0, False)
    g, dropped = oracle.gate_factor((0.0, 0.25))
    assert g == 0.5 and not dropped
    g, dropped = oracle.gate_factor((math.log(3.0), 0.0))  # sigmoid(log 3) = 3/4
    assert math.isclose(g, 0.75, rel_tol=1e-15) and not dropped
    assert oracle.gate_factor((-math.log(9.0), 0.2)) == pytest.approx((0.1, True))
    assert oracle.gate_factor((float("inf"), 0.5)) == (1.0, False)


def test_gate_open_is_ungated():
    q, k, v, w = _small(N=256, d=16, seed=40)
    cls = _cls_from(q, k, 32, 0.25, 0.25)
    do = np.random.default_rng(41).standard_normal(q.shape)
    a = oracle.forward(q, k, v, w, cls, 32)
    b = oracle.forward(q, k, v, w, cls, 32, gate=(float("inf"), 0.5))
    assert np.array_equal(a["o"], b["o"])
    ga = oracle.backward(q, k, v, w, cls, do, 32)
    gb = oracle.backward(q, k, v, w, cls, do, 32, gate=(float("inf"), 0.5))
    for n in ("dq", "dk", "dv", "dw"):
        assert np.array_equal(ga[n], gb[n]), n
    assert gb["d_gamma"] == 0.0  # g (1 - g) = 0


def test_gate_scales_only_the_linear_share():
    q, k, v, w = _small(N=256, d=16, seed=42)
    cls = _cls_from(q, k, 32, 0.25, 0.25)
    a = oracle.forward(q, k, v, w, cls, 32)
    b = oracle.forward(q, k, v, w, cls, 32, gate=(-0.7, 0.05))
    g = 1.0 / (1.0 + math.exp(0.7))
    np.testing.assert_allclose(b["o"] - b["o_s"], g * (a["o"] - a["o_s"]), rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(a["o_s"], b["o_s"])


def test_dropped_gate_equals_no_marginal_blocks():
    # dropping the branch must give exactly the problem in which every
    # marginal block is negligible instead (outputs and all gradients)
    q, k, v, w = _small(N=256, d=16, seed=44)
    cls = _cls_from(q, k, 32, 0.25, 0.25)
    assert np.any(cls == 0)
    do = np.random.default_rng(45).standard_normal(q.shape)
    cls_nm = np.where(cls == 0, -1, cls).astype(cls.dtype)
    gate = (-3.0, 0.1)  # g = 0.047 < 0.1
    a = oracle.forward(q, k, v, w, cls, 32, gate=gate)
    b = oracle.forward(q, k, v, w, cls_nm, 32)
    np.testing.assert_array_equal(a["o"], b["o"])
    ga = oracle.backward(q, k, v, w, cls, do, 32, gate=gate)
    gb = oracle.backward(q, k, v, w, cls_nm, do, 32)
    for n in ("dq", "dk", "dv", "dw"):
        np.testing.assert_array_equal(ga[n], gb[n], err_msg=n)
    assert ga["d_gamma"] == 0.0


@pytest.mark.parametrize("gamma", [-1.3, 0.4, 2.0])
def test_gate_gradient_matches_central_difference(gamma):
    q, k, v, w = _small(B=1, H=1, N=256, d=8, seed=46)
    cls = _cls_from(q, k, 16, 0.25, 0.25)
    do = np.random.default_rng(47).standard_normal(q.shape)

    def loss(gm):
        return float(np.sum(oracle.forward(q, k, v, w, cls, 16, gate=(gm, 0.0))["o"] * do))

    eps = 1e-5
    fd = (loss(gamma + eps) - loss(gamma - eps)) / (2 * eps)
    got = oracle.backward(q, k, v, w, cls, do, 16, gate=(gamma, 0.0))
    assert math.isclose(fd, got["d_gamma"], rel_tol=1e-7, abs_tol=1e-10), (fd, got["d_gamma"])
    # and the other gradients still match finite differences with the gate on
    rng = np.random.default_rng(48)
    for name in ("q", "w"):
        arr = {"q": q, "w": w}[name]
        grad = got["d" + name]
        for _ in range(6):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            xp, xm = arr.copy(), arr.copy()
            xp[idx] += 1e-6
            xm[idx] -= 1e-6
            argp = {"q": q, "w": w}
            argm = dict(argp)
            argp[name], argm[name] = xp, xm
            lp = np.sum(oracle.forward(argp["q"], k, v, argp["w"], cls, 16, gate=(gamma, 0.0))["o"] * do)
            lm = np.sum(oracle.forward(argm["q"], k, v, argm["w"], cls, 16, gate=(gamma, 0.0))["o"] * do)
            assert math.isclose((lp - lm) / 2e-6, grad[idx], rel_tol=2e-6, abs_tol=2e-8)


# ---------------------------------------------------------------- key padding (R13)

def test_pool_with_padding_is_mean_of_valid_tokens():
    x = _rand((1, 2, 128, 4), 60)
    got = oracle.pool(x, 32, n_valid=101)
    np.testing.assert_allclose(got[:, :, :3], x.reshape(1, 2, 4, 32, 4)[:, :, :3].mean(axis=3),
                               rtol=1e-14)
    np.testing.assert_allclose(got[:, :, 3], x[:, :, 96:101].mean(axis=2), rtol=1e-14)
    with pytest.raises(ValueError):
        oracle.pool(x, 32, n_valid=96)  # a whole block of padding


def test_padding_at_full_length_is_unpadded():
    q, k, v, w = _small(N=256, d=16, seed=61)
    cls = _cls_from(q, k, 32, 0.25, 0.25)
    do = np.random.default_rng(62).standard_normal(q.shape)
    a = oracle.forward(q, k, v, w, cls, 32)
    b = oracle.forward(q, k, v, w, cls, 32, n_valid=256)
    for n in ("o", "o_s", "o_l", "lse", "den"):
        assert np.array_equal(a[n], b[n]), n
    ga = oracle.backward(q, k, v, w, cls, do, 32)
    gb = oracle.backward(q, k, v, w, cls, do, 32, n_valid=256)
    for n in ("dq", "dk", "dv", "dw"):
        assert np.array_equal(ga[n], gb[n]), n


def test_padded_tokens_do_not_matter():
    # two different fillings of the padding: identical outputs and gradients,
    # zero at the padded positions
    nv = 229
    q, k, v, w = _small(N=256, d=16, seed=63)
    do = np.random.default_rng(64).standard_normal(q.shape)
    q2, k2, v2, do2 = (a.copy() for a in (q, k, v, do))
    rng = np.random.default_rng(65)
    for a in (q2, k2, v2, do2):
        a[:, :, nv:] = rng.standard_normal(a[:, :, nv:].shape) * 7.0
    n_h, n_l = oracle.block_counts(8, 0.25, 0.25)
    cls = oracle.classify(oracle.pooled_logits(q, k, 32, 0.25, nv), n_h, n_l)
    cls2 = oracle.classify(oracle.pooled_logits(q2, k2, 32, 0.25, nv), n_h, n_l)
    assert np.array_equal(cls, cls2)
    f1 = oracle.forward(q, k, v, w, cls, 32, n_valid=nv)
    f2 = oracle.forward(q2, k2, v2, w, cls, 32, n_valid=nv)
    for n in ("o", "o_s", "o_l", "lse", "den"):
        assert np.array_equal(f1[n], f2[n]), n
    assert np.all(f1["o"][:, :, nv:] == 0) and np.all(np.isposinf(f1["lse"][:, :, nv:]))
    g1 = oracle.backward(q, k, v, w, cls, do, 32, n_valid=nv)
    g2 = oracle.backward(q2, k2, v2, w, cls, do2, 32, n_valid=nv)
    for n in ("dq", "dk", "dv", "dw"):
        assert np.array_equal(g1[n], g2[n]), n
    for n in ("dq", "dk", "dv"):
        assert np.all(g1[n][:, :, nv:] == 0), n


@pytest.mark.parametrize("nv", [113, 127])
def test_padded_blockwise_equals_bruteforce(nv):
    q, k, v, w = _small(B=1, H=2, N=128, d=8, seed=66)
    cls = oracle.classify(oracle.pooled_logits(q, k, 16, 0.3, nv), *oracle.block_counts(8, 0.25, 0.25))
    got = oracle.forward(q, k, v, w, cls, 16, 0.3, n_valid=nv)["o"]
    ref = oracle.forward_bruteforce(q, k, v, w, cls, 16, 0.3, n_valid=nv)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_padded_backward_matches_central_differences():
    nv = 247
    q, k, v, w = _small(B=1, H=1, N=256, d=8, seed=67)
    do = np.random.default_rng(68).standard_normal(q.shape)
    cls = oracle.classify(oracle.pooled_logits(q, k, 16, 1 / math.sqrt(8), nv),
                          *oracle.block_counts(16, 0.25, 0.25))
    g = oracle.backward(q, k, v, w, cls, do, 16, n_valid=nv)

    def loss(qq, kk, vv, ww):
        o = oracle.forward(qq, kk, vv, ww, cls, 16, n_valid=nv)["o"]
        return float(np.sum(o[:, :, :nv] * do[:, :, :nv]))

    rng = np.random.default_rng(69)
    for name in ("q", "k", "v", "w"):
        arr = {"q": q, "k": k, "v": v, "w": w}[name]
        grad = g["d" + name]
        for _ in range(8):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            xp, xm = arr.copy(), arr.copy()
            xp[idx] += 1e-6
            xm[idx] -= 1e-6
            a = {"q": q, "k": k, "v": v, "w": w}
            bp, bm = dict(a), dict(a)
            bp[name], bm[name] = xp, xm
            fd = (loss(bp["q"], bp["k"], bp["v"], bp["w"]) - loss(bm["q"], bm["k"], bm["v"], bm["w"])) / 2e-6
            assert math.isclose(fd, grad[idx], rel_tol=2e-6, abs_tol=2e-8), (name, idx, fd, grad[idx])


# ---------------------------------------------------------------- hierarchical selection (R14)

@pytest.mark.parametrize("args,expect", [
    ((1182, 119, 118, 16), (74, 9, 9)),     # long sequence, partial last super-block
    ((1182, 30, 118, 16), (74, 3, 9)),
    ((512, 26, 51, 16), (32, 2, 4)),        # whole super-blocks only
    ((16, 4, 4, 4), (4, 1, 1)),
    ((16, 4, 4, 4, 3), (4, 3, 1)),          # a caller's minimum
    ((16, 4, 4, 4, 3, 2), (4, 4, 4)),       # the lists would meet: flat
    ((16, 0, 0, 4), (4, 0, 0)),
    ((10, 3, 3, 4), (3, 3, 3)),             # 2 + 2 > 3: flat
    ((10, 1, 0, 4), (3, 2, 0)),             # partial: one more than ceil(1/4)
])
def test_coarse_counts(args, expect):
    assert oracle.coarse_counts(*args) == expect


def test_coarse_counts_rejects_bad_group():
    with pytest.raises(ValueError):
        oracle.coarse_counts(16, 4, 4, 1)
    with pytest.raises(ValueError):
        oracle.coarse_counts(16, 4, 4, 4, -1)


def test_coarse_keys_are_pooling_at_the_coarser_block():
    # whole super-blocks: the mean of G block means is the mean of their G*b tokens
    k = _rand((2, 3, 16 * 8, 5), 40)
    kb = oracle.pool(k, 8)
    np.testing.assert_allclose(oracle.coarse_keys(kb, 4), oracle.pool(k, 32), rtol=0, atol=1e-13)
    # partial last super-block (T = 7, G = 3): blocks 6 alone
    k7 = _rand((1, 1, 7 * 4, 3), 41)
    kc = oracle.coarse_keys(oracle.pool(k7, 4), 3)
    assert kc.shape == (1, 1, 3, 3)
    np.testing.assert_allclose(kc[0, 0, 2], k7[0, 0, 24:28].mean(axis=0), atol=1e-14)
    np.testing.assert_allclose(kc[0, 0, 1], k7[0, 0, 12:24].mean(axis=0), atol=1e-14)


def test_coarse_logits_closed_form():
    q, k = _rand((1, 2, 12 * 8, 6), 42), _rand((1, 2, 12 * 8, 6), 43)
    got = oracle.coarse_logits(q, k, 8, 0.3, 3)
    want = np.einsum("bhid,bhjd->bhij", oracle.pool(q, 8), oracle.pool(k, 24)) * 0.3
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def _hier_case(T, G, seed, ties=True):
    rng = np.random.default_rng(seed)
    TG = -(-T // G)
    if ties:
        fine = rng.integers(-3, 4, size=(2, T, T)).astype(np.float64)
        coarse = rng.integers(-2, 3, size=(2, T, TG)).astype(np.float64)
        fine[0, :, ::3] = -0.0
    else:
        fine, coarse = rng.standard_normal((2, T, T)), rng.standard_normal((2, T, TG))
    return fine, coarse


@pytest.mark.parametrize("T,G", [(1, 2), (5, 2), (16, 4), (21, 4), (33, 8), (40, 3)])
@pytest.mark.parametrize("frac", [(0.0, 0.0), (0.1, 0.2), (0.25, 0.25), (0.05, 0.5)])
@pytest.mark.parametrize("extra", [(0, 0), (1, 0), (0, 2)])
def test_hierarchical_matches_rank_count(T, G, frac, extra):
    n_h, n_l = oracle.block_counts(T, *frac)
    fine, coarse = _hier_case(T, G, T * 7 + G)
    got = oracle.classify_hierarchical(fine, coarse, n_h, n_l, G, *extra)
    for r in range(fine.shape[0]):
        for i in range(T):
            want = oracle.classify_hierarchical_rows_bruteforce(
                fine[r, i].tolist(), coarse[r, i].tolist(), n_h, n_l, G, *extra)
            assert got[r, i].tolist() == want, (r, i)


@pytest.mark.parametrize("T,G", [(16, 4), (21, 4), (40, 3)])
def test_hierarchical_with_every_candidate_is_flat(T, G):
    n_h, n_l = oracle.block_counts(T, 0.2, 0.3)
    fine, coarse = _hier_case(T, G, 5 + T)
    TG = coarse.shape[-1]
    got = oracle.classify_hierarchical(fine, coarse, n_h, n_l, G, TG, TG)
    np.testing.assert_array_equal(got, oracle.classify(fine, n_h, n_l))


@pytest.mark.parametrize("T,G,frac", [(64, 8, (0.1, 0.2)), (61, 4, (0.05, 0.1)),
                                      (100, 16, (0.1, 0.1))])
def test_hierarchical_counts_and_candidate_sets(T, G, frac):
    n_h, n_l = oracle.block_counts(T, *frac)
    fine, coarse = _hier_case(T, G, 11 * T, ties=False)
    TG, c_hi, c_lo = oracle.coarse_counts(T, n_h, n_l, G)
    assert c_hi + c_lo <= TG  # a pruning case
    got = oracle.classify_hierarchical(fine, coarse, n_h, n_l, G)
    assert ((got == 1).sum(-1) == n_h).all() and ((got == -1).sum(-1) == n_l).all()
    for r in range(2):
        for i in range(T):
            c = coarse[r, i]
            rank = np.array([(c > c[J]).sum() for J in range(TG)])  # distinct scores
            crit = np.flatnonzero(got[r, i] == 1)
            neg = np.flatnonzero(got[r, i] == -1)
            assert (rank[crit // G] < c_hi).all()
            assert (rank[neg // G] >= TG - c_lo).all()
            # inside its candidates the critical set is the top of the fine scores
            cand = np.flatnonzero(rank[np.arange(T) // G] < c_hi)
            rest = np.setdiff1d(cand, crit)
            if len(rest) and len(crit):
                assert fine[r, i, crit].min() >= fine[r, i, rest].max()


@pytest.mark.parametrize("frac", [(0.1, 0.2), (0.05, 0.4), (0.3, 0.3)])
def test_hierarchical_equals_flat_when_blocks_follow_their_super_block(frac):
    # fine score = coarse score of the block's super-block: the coarse order
    # agrees with the fine one (ties by index on both levels), so pruning to
    # the candidates loses nothing
    T, G = 48, 4
    n_h, n_l = oracle.block_counts(T, *frac)
    rng = np.random.default_rng(3)
    coarse = rng.integers(-4, 5, size=(3, T, T // G)).astype(np.float64)
    fine = np.repeat(coarse, G, axis=-1)
    TG, c_hi, c_lo = oracle.coarse_counts(T, n_h, n_l, G)
    assert c_hi + c_lo <= TG
    np.testing.assert_array_equal(oracle.classify_hierarchical(fine, coarse, n_h, n_l, G),
                                  oracle.classify(fine, n_h, n_l))
