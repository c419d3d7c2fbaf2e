"""Plain fp64 CPU oracle for SLA (Sparse-Linear Attention).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  It shares no code with the CUDA path
and never calls it.  It is slow on purpose: every step is the definition
written out, with numpy matrix products as the only library primitive.

Sources.  "SLA" below is the paper page "SLA: Beyond Sparsity in Diffusion
Transformers via Fine-Tunable Sparse-Linear Attention" (arXiv 2509.24006):
its English abstract and the Chinese card's technical-framework steps 1-4
fix that attention weights fall into critical / marginal / negligible groups,
that critical pairs get exact O(N^2) softmax attention, marginal pairs get
O(N) linear attention and negligible pairs are skipped, and that a backward
pass exists.  The pages leave open how the classes are chosen, the feature
map, the combination and the backward math; this oracle takes these readings
(each restated where it is used):

* R1  classes come from block mean-pooled Q and K: pooled logits
      s_ij = mean(Q_i) . mean(K_j) * scale; per row, order j by
      (s_ij descending, j ascending); the first n_h are critical (+1), the
      last n_l negligible (-1), the rest marginal (0).  Ranking logits is the
      same as ranking the row softmax of the pooled scores (softmax is
      strictly increasing within a row).
* R3  n_h = ceil(k_h*T - 1e-9), n_l = min(floor(k_l*T + 1e-9), T - n_h).
* R4  phi(x) = elu(x) + 1 (alpha 1): x + 1 for x > 0, exp(x) otherwise.
* R5  a query block with no critical key block has O_s = 0 and LSE = -inf.
* R6  linear branch: O_l,t = phi(Q_t)^T H_i / (phi(Q_t) . Z_i) with
      H_i = sum_{j marginal} phi(K_j)^T V_j and Z_i = sum_{j marginal}
      sum_{u in j} phi(K_u); no epsilon; 0 when row i has no marginal block.
* R7  O = O_s + O_l W_proj, W_proj one d x d matrix for all heads.
* R8  gradients treat the classification as a constant.
* R13 optional key padding (valid length n_valid, only the last block may be
      partial): tokens t >= n_valid do not exist for the method.  Block means,
      softmax keys and key-block summaries use valid tokens only; padded query
      rows output O = O_s = O_l = 0 and den = 0, and LSE = +inf (no token, so
      exp(s - LSE) = 0 for every key; -inf stays the mark of a real row with no
      critical block); their dO is ignored and every padded position gets zero
      gradient.  Without n_valid, padding
      tokens are ordinary tokens.
* R12 optional gate on the linear branch, after the page "SALAD: Achieve
      High-Sparsity Attention via Efficient Linear Attention Tuning for Video
      Diffusion Transformer", section "Methodologie: SALAD", items 2 (a global
      factor in (0, 1) from a sigmoid scales the linear branch) and 3 (branches
      with a very low factor are dropped at inference): with a caller-given
      logit gamma and threshold tau, g = sigmoid(gamma) and
      O = O_s + g * O_l W_proj; when g < tau the branch is dropped, O = O_s,
      and neither the branch nor gamma gets a gradient.
* R14 optional hierarchical selection for long sequences, after the page
      "Trainable Log-linear Sparse Attention for Efficient Diffusion
      Transformers" (abstract: top-K is taken at a coarse level first and the
      next level's top-K is restricted to the indices found there): blocks
      are grouped into super-blocks of G consecutive blocks (the last may be
      partial) with mean key Kc_J (equal-weight mean of its blocks' mean
      keys); a query block's coarse scores are sc_iJ = mean(Q_i) . Kc_J *
      scale; in the order (sc desc, J asc) its first c_hi super-blocks are the
      critical candidates and its last c_lo the negligible candidates.  c_hi is
      at least a caller's minimum and at least ceil(n_h / G) (+1 when T % G,
      since the partial super-block may be chosen), so the candidates hold
      n_h blocks; c_lo likewise for n_l; when c_hi + c_lo > TG both become
      TG.  Critical: the first n_h candidate blocks in the order (s desc,
      j asc) of the fine scores; negligible: the last n_l, in that order, of
      the negligible candidates that are not critical; the rest marginal.
      Counts are exactly n_h and n_l, and with every super-block a candidate
      this is R1.

Arrays are [B, H, N, d]; blocks are consecutive runs of ``block`` tokens.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "block_counts",
    "pool",
    "pooled_logits",
    "classify",
    "classify_rows_bruteforce",
    "coarse_counts",
    "coarse_keys",
    "coarse_logits",
    "classify_hierarchical",
    "classify_hierarchical_rows_bruteforce",
    "phi",
    "phi_prime",
    "key_block_summaries",
    "gate_factor",
    "forward",
    "forward_bruteforce",
    "backward",
    "sla",
]


def block_counts(T: int, k_h: float, k_l: float) -> tuple[int, int]:
    """Critical and negligible block counts per row (reading R3)."""
    if not (0.0 <= k_h and 0.0 <= k_l and k_h + k_l <= 1.0 + 1e-12):
        raise ValueError("need 0 <= k_h, k_l and k_h + k_l <= 1")
    n_h = min(T, max(0, math.ceil(k_h * T - 1e-9)))
    n_l = max(0, min(math.floor(k_l * T + 1e-9), T - n_h))
    return n_h, n_l


def _n_valid(N: int, block: int, n_valid) -> int:
    """Checked valid length (reading R13): N when not given."""
    if n_valid is None:
        return N
    n_valid = int(n_valid)
    if not (N - block < n_valid <= N):
        raise ValueError("n_valid must leave only the last block partially padded")
    return n_valid


def pool(x: np.ndarray, block: int, n_valid=None) -> np.ndarray:
    """Mean of each block's valid tokens (R1, R13): [B,H,N,d] -> [B,H,T,d]."""
    B, H, N, d = x.shape
    if N % block:
        raise ValueError("N must be a multiple of the block size")
    nv = _n_valid(N, block, n_valid)
    w = (np.arange(N) < nv).astype(np.float64).reshape(N // block, block)
    xb = x.astype(np.float64).reshape(B, H, N // block, block, d)
    return np.einsum("bhtud,tu->bhtd", xb, w) / w.sum(axis=1)[:, None]


def pooled_logits(q: np.ndarray, k: np.ndarray, block: int, scale: float,
                  n_valid=None) -> np.ndarray:
    """s_ij = mean(Q_i) . mean(K_j) * scale, [B,H,T,T] (reading R1)."""
    qb, kb = pool(q, block, n_valid), pool(k, block, n_valid)
    return np.einsum("bhid,bhjd->bhij", qb, kb) * scale


def classify(logits: np.ndarray, n_h: int, n_l: int) -> np.ndarray:
    """Three-way block classes from score rows (reading R1): int8 in {+1,0,-1}.

    Each row is ordered by (score descending, key-block index ascending); the
    first n_h entries are critical, the last n_l negligible.
    """
    logits = np.asarray(logits, dtype=np.float64)
    if np.isnan(logits).any():
        raise ValueError("NaN scores have no ordering")
    *lead, T = logits.shape
    flat = logits.reshape(-1, T)
    cls = np.zeros(flat.shape, dtype=np.int8)
    idx = np.arange(T)
    for r in range(flat.shape[0]):
        order = np.lexsort((idx, -flat[r]))  # primary: -score, secondary: index
        cls[r, order[:n_h]] = 1
        if n_l:
            cls[r, order[T - n_l:]] = -1
    return cls.reshape(*lead, T)


def classify_rows_bruteforce(row: list[float], n_h: int, n_l: int) -> list[int]:
    """Pure-Python per-entry rank count; the independent check of ``classify``.

    rank(j) = #{k : s_k > s_j} + #{k < j : s_k == s_j}; critical iff
    rank < n_h, negligible iff rank >= T - n_l.
    """
    T = len(row)
    out = []
    for j in range(T):
        rank = sum(1 for k in range(T) if row[k] > row[j] or (row[k] == row[j] and k < j))
        out.append(1 if rank < n_h else (-1 if rank >= T - n_l else 0))
    return out


def coarse_counts(T: int, n_h: int, n_l: int, group: int, top: int = 0, bottom: int = 0):
    """(TG, c_hi, c_lo) of the hierarchical selection (reading R14).

    TG = ceil(T / group) super-blocks.  c_hi is at least top and at least the
    number of super-blocks that always hold n_h blocks (ceil(n_h / group),
    plus one when the last super-block is partial, since it may be chosen);
    c_lo likewise for n_l.  When the two candidate lists could meet
    (c_hi + c_lo > TG) every super-block is a candidate of both, which is the
    flat selection.
    """
    if group < 2:
        raise ValueError("group must be at least 2")
    if top < 0 or bottom < 0:
        raise ValueError("candidate counts must be non-negative")
    TG = -(-T // group)
    partial = 1 if T % group else 0

    def floor(n):
        return 0 if n == 0 else -(-n // group) + partial

    c_hi = min(TG, max(top, floor(n_h)))
    c_lo = min(TG, max(bottom, floor(n_l)))
    if c_hi + c_lo > TG:
        c_hi = c_lo = TG
    return TG, c_hi, c_lo


def coarse_keys(kbar: np.ndarray, group: int) -> np.ndarray:
    """Kc_J = equal-weight mean of the block means of super-block J: [.., T, d] -> [.., TG, d]."""
    T = kbar.shape[-2]
    TG = -(-T // group)
    return np.stack([kbar[..., J * group:min((J + 1) * group, T), :].mean(axis=-2)
                     for J in range(TG)], axis=-2)


def coarse_logits(q: np.ndarray, k: np.ndarray, block: int, scale: float, group: int,
                  n_valid=None) -> np.ndarray:
    """sc_iJ = mean(Q_i) . Kc_J * scale, [B,H,T,ceil(T/group)] (reading R14)."""
    qb = pool(q, block, n_valid)
    kc = coarse_keys(pool(k, block, n_valid), group)
    return np.einsum("bhid,bhjd->bhij", qb, kc) * scale


def _order(scores: np.ndarray, among: np.ndarray) -> np.ndarray:
    """Indices ``among`` sorted by (score desc, index asc)."""
    among = np.asarray(among)
    return among[np.lexsort((among, -scores[among]))]


def classify_hierarchical(logits: np.ndarray, coarse: np.ndarray, n_h: int, n_l: int,
                          group: int, top: int = 0, bottom: int = 0) -> np.ndarray:
    """Three-way classes by the two-level selection of reading R14.

    logits [.., T, T] fine scores s_ij and coarse [.., T, TG] scores sc_iJ;
    only the fine scores of candidate blocks are read.  int8 in {+1, 0, -1}.
    """
    T = logits.shape[-1]
    TG, c_hi, c_lo = coarse_counts(T, n_h, n_l, group, top, bottom)
    if coarse.shape[-1] != TG or coarse.shape[:-1] != logits.shape[:-1]:
        raise ValueError("coarse scores must be [.., T, ceil(T / group)]")
    if np.isnan(coarse).any():
        raise ValueError("NaN scores have no ordering")
    lead = logits.shape[:-2]
    L = np.asarray(logits, dtype=np.float64).reshape(-1, T, T)
    C = np.asarray(coarse, dtype=np.float64).reshape(-1, T, TG)
    out = np.zeros(L.shape, dtype=np.int8)
    blocks_of = [np.arange(J * group, min((J + 1) * group, T)) for J in range(TG)]
    for r in range(L.shape[0]):
        for i in range(T):
            sb = _order(C[r, i], np.arange(TG))
            hi = np.concatenate([blocks_of[J] for J in sb[:c_hi]] + [np.zeros(0, int)])
            lo = np.concatenate([blocks_of[J] for J in sb[TG - c_lo:]] + [np.zeros(0, int)])
            if np.isnan(L[r, i, np.union1d(hi, lo)]).any():
                raise ValueError("NaN scores have no ordering")
            crit = _order(L[r, i], hi)[:n_h]
            rest = np.setdiff1d(lo, crit)
            neg = _order(L[r, i], rest)[len(rest) - n_l:] if n_l else rest[:0]
            out[r, i, crit] = 1
            out[r, i, neg] = -1
    return out.reshape(*lead, T, T)


def classify_hierarchical_rows_bruteforce(row, crow, n_h, n_l, group, top=0, bottom=0):
    """Pure-Python check of ``classify_hierarchical`` for one row: membership
    by counting, for every entry, how many entries of its set precede it."""
    T, TG = len(row), len(crow)
    _, c_hi, c_lo = coarse_counts(T, n_h, n_l, group, top, bottom)

    def rank(vals, idxs, x):  # position of x in (value desc, index asc) among idxs
        return sum(1 for y in idxs if vals[y] > vals[x] or (vals[y] == vals[x] and y < x))

    allJ = list(range(TG))
    hi_sb = {J for J in allJ if rank(crow, allJ, J) < c_hi}
    lo_sb = {J for J in allJ if rank(crow, allJ, J) >= TG - c_lo}
    hi = [j for j in range(T) if j // group in hi_sb]
    crit = {j for j in hi if rank(row, hi, j) < n_h}
    lo = [j for j in range(T) if j // group in lo_sb and j not in crit]
    neg = {j for j in lo if rank(row, lo, j) >= len(lo) - n_l}
    return [1 if j in crit else (-1 if j in neg else 0) for j in range(T)]


def phi(x: np.ndarray) -> np.ndarray:
    """elu(x) + 1 with alpha = 1 (reading R4)."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def phi_prime(x: np.ndarray) -> np.ndarray:
    """Derivative of phi: 1 for x > 0, exp(x) otherwise."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))


def key_block_summaries(k: np.ndarray, v: np.ndarray, block: int, n_valid=None):
    """Per key block j: h_j = phi(K_j)^T V_j [d,d] and z_j = sum_u phi(K_u) [d]
    over the block's valid tokens u.

    These are the per-key-block summaries through which marginal pairs get
    O(N) linear attention (SLA abstract; framework step 3).
    """
    B, H, N, d = k.shape
    T = N // block
    nv = _n_valid(N, block, n_valid)
    valid = (np.arange(N) < nv).astype(np.float64)[:, None]
    fk = (phi(k) * valid).reshape(B, H, T, block, d)
    vb = (v.astype(np.float64) * valid).reshape(B, H, T, block, d)
    h = np.einsum("bhtua,bhtuc->bhtac", fk, vb)
    z = fk.sum(axis=3)
    return h, z


def gate_factor(gate) -> tuple[float, bool]:
    """(g, dropped) for gate = (gamma, tau) or None (reading R12).

    g = 1 / (1 + exp(-gamma)); None means no gate (g = 1, never dropped).
    """
    if gate is None:
        return 1.0, False
    gamma, tau = float(gate[0]), float(gate[1])
    g = 1.0 / (1.0 + math.exp(-gamma)) if gamma > -700 else 0.0
    return g, g < tau


def _tokens(blocks: np.ndarray, block: int) -> np.ndarray:
    return (blocks[:, None] * block + np.arange(block)[None, :]).reshape(-1)


def forward(q, k, v, w_proj, cls, block: int, scale: float | None = None,
            query_blocks=None, gate=None, n_valid=None):
    """SLA forward with a given class map ``cls`` [B,H,T,T].

    Returns a dict with o, o_s, o_l [B,H,N,d], lse and den [B,H,N] (fp64),
    and the gate factor g.  ``query_blocks``, if given, restricts the work to
    those query-block indices (other rows stay zero / -inf); used to sample
    large problems.  ``gate`` = (gamma, tau) gates the linear branch (R12); a
    dropped branch leaves o_l and den zero.  ``n_valid`` masks the padding
    tokens (R13).
    """
    g, dropped = gate_factor(gate)
    B, H, N, d = q.shape
    T = N // block
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    q64, k64, v64 = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    w64 = np.asarray(w_proj, dtype=np.float64)
    nv = _n_valid(N, block, n_valid)
    h, z = key_block_summaries(k64, v64, block, nv)
    o_s = np.zeros((B, H, N, d))
    o_l = np.zeros((B, H, N, d))
    lse = np.full((B, H, N), -np.inf)
    den = np.zeros((B, H, N))
    rows = range(T) if query_blocks is None else query_blocks
    for b in range(B):
        for hh in range(H):
            # H_i = sum_{j marginal in row i} h_j for every i, written as the
            # product with the 0/1 marginal indicator matrix of this head
            marg_ind = (cls[b, hh] == 0).astype(np.float64)
            H_all = np.tensordot(marg_ind, h[b, hh], axes=(1, 0))
            Z_all = marg_ind @ z[b, hh]
            for i in rows:
                t0, t1 = i * block, min((i + 1) * block, nv)  # valid query rows
                qi = q64[b, hh, t0:t1]
                crit = np.nonzero(cls[b, hh, i] == 1)[0]
                marg = np.nonzero(cls[b, hh, i] == 0)[0]
                # critical pairs: exact softmax attention over all their valid key tokens
                if crit.size:
                    keys = _tokens(crit, block)
                    keys = keys[keys < nv]
                    s = (qi @ k64[b, hh, keys].T) * scale
                    m = s.max(axis=1, keepdims=True)
                    e = np.exp(s - m)
                    l = e.sum(axis=1, keepdims=True)
                    o_s[b, hh, t0:t1] = (e @ v64[b, hh, keys]) / l
                    lse[b, hh, t0:t1] = (m + np.log(l))[:, 0]
                # marginal pairs: linear attention through the key-block summaries
                if marg.size and not dropped:
                    Hi, Zi = H_all[i], Z_all[i]
                    fq = phi(qi)
                    num = fq @ Hi
                    dn = fq @ Zi
                    o_l[b, hh, t0:t1] = num / dn[:, None]
                    den[b, hh, t0:t1] = dn
                # negligible pairs contribute nothing
    lse[:, :, nv:] = np.inf  # padded rows (R13)
    o = o_s + g * np.einsum("bhta,ac->bhtc", o_l, w64)
    return {"o": o, "o_s": o_s, "o_l": o_l, "lse": lse, "den": den, "g": g}


def forward_bruteforce(q, k, v, w_proj, cls, block: int, scale: float | None = None,
                       n_valid=None):
    """Per-token loops over every key with the class looked up per key.

    The linear branch is written per key token,
    O_l,t = sum_u (phi(Q_t).phi(K_u)) V_u / sum_u phi(Q_t).phi(K_u),
    u over marginal tokens, so agreement with ``forward`` pins the summary
    reassociation.  Meant for N <= 256.  With ``n_valid`` (R13) keys and
    queries at t >= n_valid are skipped (padded rows stay 0).
    """
    B, H, N, d = q.shape
    nv = N if n_valid is None else int(n_valid)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    q64, k64, v64 = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    w64 = np.asarray(w_proj, dtype=np.float64)
    o = np.zeros((B, H, N, d))
    for b in range(B):
        for hh in range(H):
            for t in range(nv):
                i = t // block
                crit_w, crit_v = [], []
                lin_num = np.zeros(d)
                lin_den = 0.0
                fq = phi(q64[b, hh, t])
                for u in range(nv):
                    c = cls[b, hh, i, u // block]
                    if c == 1:
                        crit_w.append(float(q64[b, hh, t] @ k64[b, hh, u]) * scale)
                        crit_v.append(v64[b, hh, u])
                    elif c == 0:
                        a = float(fq @ phi(k64[b, hh, u]))
                        lin_num += a * v64[b, hh, u]
                        lin_den += a
                os_t = np.zeros(d)
                if crit_w:
                    mx = max(crit_w)
                    ex = [math.exp(x - mx) for x in crit_w]
                    tot = sum(ex)
                    for e_u, v_u in zip(ex, crit_v):
                        os_t += (e_u / tot) * v_u
                ol_t = lin_num / lin_den if lin_den > 0 else np.zeros(d)
                for c_out in range(d):
                    o[b, hh, t, c_out] = os_t[c_out] + sum(
                        ol_t[a] * w64[a, c_out] for a in range(d))
    return o


def backward(q, k, v, w_proj, cls, d_o, block: int, scale: float | None = None,
             fwd=None, gate=None, n_valid=None):
    """Gradients of sum(O * dO) w.r.t. Q, K, V and W_proj, classes held fixed (R8).

    Sparse branch (standard softmax-attention backward over critical pairs):
      D_t = dO_t . O_s,t;  P = exp(S - LSE);  dV_u += P_tu dO_t;
      dP_tu = dO_t . V_u;  dS = P (dP - D);  dQ_t += scale dS_tu K_u;
      dK_u += scale dS_tu Q_t.
    Linear branch (O_l = num/den, num = phi(Q) H_i, den = phi(Q) . Z_i):
      dO_l = dO W^T; dnum = dO_l / den; dden = -(dO_l . O_l) / den;
      dphi(Q_t) = H_i dnum_t + Z_i dden_t;  dQ_t += dphi(Q_t) * phi'(Q_t);
      dH_i = sum_t phi(Q_t) dnum_t^T;  dZ_i = sum_t phi(Q_t) dden_t;
      dh_j = sum_{i: j marginal in row i} dH_i (likewise dz_j);
      dphi(K_u) = dh_j V_u + dz_j;  dK_u += dphi(K_u) * phi'(K_u);
      dV_u += dh_j^T phi(K_u).
    Projection: dW = sum over b, h, t of O_l,t dO_t^T.
    Gate (R12): the linear branch sees g dO, so dO_l, dW and everything
    downstream of them carry the factor g, and
      d gamma = g (1 - g) sum over b, h, t of (O_l,t W) . dO_t;
    a dropped branch contributes nothing and d gamma = 0.
    Key padding (R13): dO of padded rows is ignored, padded positions get 0.
    """
    g, dropped = gate_factor(gate)
    B, H, N, d = q.shape
    T = N // block
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    nv = _n_valid(N, block, n_valid)
    if fwd is None:
        fwd = forward(q, k, v, w_proj, cls, block, scale, gate=gate, n_valid=nv)
    q64, k64, v64, do64 = (np.asarray(a, dtype=np.float64) for a in (q, k, v, d_o))
    do64 = do64 * (np.arange(N) < nv)[:, None]  # padded rows carry no gradient
    w64 = np.asarray(w_proj, dtype=np.float64)
    h, z = key_block_summaries(k64, v64, block, nv)
    dq = np.zeros_like(q64)
    dk = np.zeros_like(k64)
    dv = np.zeros_like(v64)
    dw = g * np.einsum("bhta,bhtc->ac", fwd["o_l"], do64)
    do_l = g * np.einsum("bhtc,ac->bhta", do64, w64)
    d_gamma = 0.0 if dropped else (
        g * (1.0 - g) * float(np.einsum("bhta,ac,bhtc->", fwd["o_l"], w64, do64)))
    for b in range(B):
        for hh in range(H):
            marg_ind = (cls[b, hh] == 0).astype(np.float64)
            H_all = np.tensordot(marg_ind, h[b, hh], axes=(1, 0))
            Z_all = marg_ind @ z[b, hh]
            dH_all = np.zeros((T, d, d))  # dL/dH_i per query block
            dZ_all = np.zeros((T, d))
            for i in range(T):
                t0, t1 = i * block, min((i + 1) * block, nv)  # valid query rows
                qi = q64[b, hh, t0:t1]
                doi = do64[b, hh, t0:t1]
                crit = np.nonzero(cls[b, hh, i] == 1)[0]
                marg = np.nonzero(cls[b, hh, i] == 0)[0]
                if crit.size:
                    keys = _tokens(crit, block)
                    keys = keys[keys < nv]
                    kc, vc = k64[b, hh, keys], v64[b, hh, keys]
                    s = (qi @ kc.T) * scale
                    p = np.exp(s - fwd["lse"][b, hh, t0:t1, None])
                    D = np.sum(doi * fwd["o_s"][b, hh, t0:t1], axis=1, keepdims=True)
                    dv[b, hh, keys] += p.T @ doi
                    dp = doi @ vc.T
                    ds = p * (dp - D)
                    dq[b, hh, t0:t1] += scale * (ds @ kc)
                    dk[b, hh, keys] += scale * (ds.T @ qi)
                if marg.size and not dropped:
                    Hi, Zi = H_all[i], Z_all[i]
                    dn = fwd["den"][b, hh, t0:t1]
                    dol = do_l[b, hh, t0:t1]
                    dnum = dol / dn[:, None]
                    dden = -np.sum(dol * fwd["o_l"][b, hh, t0:t1], axis=1) / dn
                    fq = phi(qi)
                    dfq = dnum @ Hi.T + dden[:, None] * Zi[None, :]
                    dq[b, hh, t0:t1] += dfq * phi_prime(qi)
                    dH_all[i] = fq.T @ dnum
                    dZ_all[i] = fq.T @ dden
            # dh_j = sum over rows i in which j is marginal of dL/dH_i
            dh = np.tensordot(marg_ind.T, dH_all, axes=(1, 0))
            dz = marg_ind.T @ dZ_all
            for j in range(T):
                u0, u1 = j * block, min((j + 1) * block, nv)  # valid key rows
                kj, vj = k64[b, hh, u0:u1], v64[b, hh, u0:u1]
                dfk = vj @ dh[j].T + dz[j][None, :]
                dk[b, hh, u0:u1] += dfk * phi_prime(kj)
                dv[b, hh, u0:u1] += phi(kj) @ dh[j]
    return {"dq": dq, "dk": dk, "dv": dv, "dw": dw, "d_gamma": d_gamma}


def sla(q, k, v, w_proj, block: int, k_h: float, k_l: float, scale: float | None = None,
        n_valid=None):
    """Classification from the inputs followed by the forward."""
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    T = q.shape[2] // block
    n_h, n_l = block_counts(T, k_h, k_l)
    logits = pooled_logits(q, k, block, scale, n_valid)
    cls = classify(logits, n_h, n_l)
    out = forward(q, k, v, w_proj, cls, block, scale, n_valid=n_valid)
    out.update(cls=cls, logits=logits)
    return out
