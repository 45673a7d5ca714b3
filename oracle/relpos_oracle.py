"""Plain fp64 CPU oracle for exact relative-position attention, forward and backward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run
this module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it.  It shares no code, table or helper with the CUDA library.

What it computes
----------------
"Fast and Exact Relative-Position Attention via Structure-Aware Kernels"
(Abstract) adds a relative-position term to FlashAttention-style attention and
keeps the result exact.  The article "结构感知内核让相对位置注意力加速21倍",
section "为什么相对位置注意力难做快", writes the score as

    S_ij = Q_i K_j^T / sqrt(d) + B_ij

and notes that a naive implementation materialises B (an [L, L] fp32 matrix,
256 MiB at L = 8K).  This oracle does exactly that, on purpose: it builds B for
each (batch, head) explicitly, applies the row softmax, and differentiates the
result by the textbook chain rule.  Because the method is exact, this plain
definition is the result the fast path must reproduce up to rounding.

The four mechanisms named on the Hugging Face page of the paper (Community
comment: DeBERTa, Shaw, Transformer-XL and T5) are written out from their
original papers, because the pages print none of their formulas:

  T5 (Raffel et al.)           S_ij = s q_i.k_j + t[h, bucket(j - i)]
  Shaw (Shaw et al., key side) S_ij = s (q_i.k_j + q_i.a[h, clip(j - i, -c, c) + c])
  Transformer-XL (Dai et al.)  S_ij = s ((q_i + u).k_j + (q_i + v).r[h, row(i - j)])
  DeBERTa (He et al.)          S_ij = s (q_i.k_j + q_i.Kr[h, clip(i - j + k, 0, 2k-1)]
                                          + k_j.Qr[h, clip(j - i + k, 0, 2k-1)])

with s the caller's scale (1/sqrt(d) for the first three, 1/sqrt(3d) for DeBERTa
by default).  Shaw's value-side term (the second relative table of Shaw et al.,
optional: ``RelCfg.shaw_value``) adds the same clipped offset's table row to every
value a query averages:

  O_i = sum_j P_ij (v_j + aV[h, clip(j - i, -c, c) + c])

ALiBi, the further bias named by the article (section "工程权衡与适用边界", in its
list of models the method suits), is written from its own paper (Press et al.,
"Train Short, Test Long"):

  ALiBi                        S_ij = s q_i.k_j - m[h] |j - i|

a fixed per-head slope m[h] times the distance, added unscaled (the causal model of
that paper sees only j <= i, so -m (i - j); without a causal mask the symmetric
distance is the plain reading).  The slopes are the caller's input; their gradient
sum_ij dS_ij (-|j - i|) is returned like a table gradient.

Transformer-XL rows: row(delta) = delta when causal (delta in [0, L)), delta + L - 1
otherwise (delta in (-L, L)).  Causal masking removes j > i.

Backward (textbook softmax chain rule):
  dP = dO V^T,  D_i = sum_c dO_ic O_ic,  dS = P o (dP - D),  dV = P^T dO,
and every parameter theta of the score gets  sum_ij dS_ij dS_ij/dtheta.
Table gradients are formed by scatter-adding dS into explicit index maps
(``np.add.at``): the gradient-sharding of the paper (Abstract, technique (3);
article section "3. 基于偏移的梯度分片") is what the fast path does, not this.

Readings where the pages are silent (listed again in the design notes):
  * T5 buckets: bidirectional, 32 buckets, max_distance 128; the logarithmic
    part 8 + floor(2 log2(a/8)) is taken in exact integer arithmetic,
    8 + floor(log2(a^2)) - 6 (a float log may land either side of the exact
    boundaries a = 16, 32, 64).
  * Shaw: the scale multiplies the whole logit (content and position parts).
  * T5: the bias is added unscaled.
  * Variable-length batches (the speech batches of the article, section "为什么
    相对位置注意力难做快"): an optional per-batch key length ``seqlens_k[b]``
    masks keys j >= seqlens_k[b] of that batch (after causal masking); queries are
    all computed.  Relative positions keep their meaning (j - i over the padded
    length L), so the tables and index maps do not change.
  * Transformer-XL memory (``txl_memory_forward`` / ``txl_memory_backward``): the L
    queries of the current segment sit at absolute positions M .. M + L - 1 over the M
    cached keys / values followed by the segment's L; causal, r has M + L rows.
  * Fully masked rows (an empty key set: seqlens_k[b] = 0, or a causal row whose
    keys are all padding) give O = 0 and LSE = -inf and zero gradients.
  * LSE is the natural log of the softmax denominator.

All arithmetic is float64.  Inputs given in bf16 are expected to be upcast by
the caller (the oracle then sees exactly the values the GPU sees).

Pins (tests/test_oracle_pins.py, tests/test_oracle_autograd.py; none of them calls
this module to make its expected values):
  * ``t5_bucket``: a hand-written golden table (tests/golden), the float formula away
    from the exact ties, the unidirectional variant;
  * ``forward`` / ``backward`` / ``backward_rows`` for every mechanism, with key
    lengths and the Shaw value table: scalar Python loops written from each formula
    (forward and scalar chain rule) on tiny shapes, central finite differences, and
    torch.autograd of a dense torch restatement (1e-11);
  * closed forms: L = 1, causal row 0, ALiBi geometric sums; zero relative term ==
    torch's scaled_dot_product_attention; row-constant terms; query-side table
    gradients summing to zero; batch sums; padding keys;
  * ``txl_memory_forward`` / ``txl_memory_backward``: scalar loops with the explicit
    memory offset, finite differences, autograd of a direct restatement.
Parity unpinned: no function.  The conventions the pages leave open (listed above
under "Readings") are pinned only as readings: the pages print no worked example.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

T5, SHAW, TXL, DEBERTA, ALIBI = 0, 1, 2, 3, 4
MECH_NAMES = {T5: "t5", SHAW: "shaw", TXL: "txl", DEBERTA: "deberta", ALIBI: "alibi"}


@dataclass(frozen=True)
class RelCfg:
    """Mechanism hyper-parameters (defaults are the workloads' values)."""

    t5_num_buckets: int = 32
    t5_max_distance: int = 128
    t5_bidirectional: bool = True
    shaw_clip: int = 64
    deberta_span: int = 256
    shaw_value: bool = False  # Shaw: rel[1] = aV, the value-side table


def default_scale(mech: int, d: int) -> float:
    """1/sqrt(d) as in the article's score formula; DeBERTa uses 1/sqrt(3d)
    (its three score terms, He et al.)."""
    return 1.0 / math.sqrt(3 * d) if mech == DEBERTA else 1.0 / math.sqrt(d)


def table_rows(mech: int, L: int, causal: bool, cfg: RelCfg) -> int:
    """Number of rows of the relative table of each head (ALiBi: one slope)."""
    if mech == ALIBI:
        return 1
    if mech == T5:
        return cfg.t5_num_buckets
    if mech == SHAW:
        return 2 * cfg.shaw_clip + 1
    if mech == TXL:
        return L if causal else 2 * L - 1
    return 2 * cfg.deberta_span


# --------------------------------------------------------------------------
# T5 bucket of a relative position n = j - i (T5 paper, relative attention bias)
# --------------------------------------------------------------------------
def t5_bucket(n, num_buckets: int = 32, max_distance: int = 128, bidirectional: bool = True):
    """Bucket of relative position n = key - query.

    Half of the buckets (bidirectional) hold exact small distances, the other
    half logarithmically spaced distances up to max_distance, beyond which the
    last bucket is used.  Positive n (key after query) uses the upper half.

    The logarithmic index is max_exact + floor(log(a/max_exact) /
    log(max_distance/max_exact) * (nb - max_exact)).  It is evaluated in exact
    integer arithmetic: for the standard (32, 128) setting this is
    floor(log2(a^2)) + 2; in general the test a^e >= max_exact^e * ratio^t is
    done on Python integers (no float rounding at the ties).
    """
    n = np.asarray(n, dtype=np.int64)
    if n.size > 4096:
        # evaluate once per distinct offset, then look up (same values)
        uniq, inv = np.unique(n, return_inverse=True)
        return _t5_bucket_direct(uniq, num_buckets, max_distance, bidirectional)[inv].reshape(n.shape)
    return _t5_bucket_direct(n, num_buckets, max_distance, bidirectional)


def _t5_bucket_direct(n, num_buckets, max_distance, bidirectional):
    nb = num_buckets
    out = np.zeros(n.shape, dtype=np.int64)
    if bidirectional:
        nb //= 2
        out += np.where(n > 0, nb, 0)
        a = np.abs(n)
    else:
        # unidirectional (causal T5): only keys at or before the query count
        a = np.maximum(-n, 0)
    max_exact = nb // 2
    flat_a = a.reshape(-1)
    flat_out = out.reshape(-1)
    for idx in range(flat_a.size):
        ai = int(flat_a[idx])
        if ai < max_exact:
            flat_out[idx] += ai
            continue
        # largest t in [0, nb - max_exact) with
        #   log(ai/me) / log(md/me) * (nb - me) >= t
        # <=> (ai/me)^(nb-me) >= (md/me)^t   (all positive)
        span = nb - max_exact
        t = 0
        while t + 1 < span + 1 and (ai ** span) * (max_exact ** (t + 1)) >= (max_exact ** span) * (max_distance ** (t + 1)):
            t += 1
        flat_out[idx] += min(max_exact + t, nb - 1)
    return out


# --------------------------------------------------------------------------
# Index maps: which table row each (query i, key j) pair reads
# --------------------------------------------------------------------------
def _rel(rows_i: np.ndarray, L: int) -> np.ndarray:
    """Matrix of j - i for the given query rows and all keys."""
    return np.arange(L, dtype=np.int64)[None, :] - rows_i[:, None]


def index_map(mech: int, L: int, causal: bool, cfg: RelCfg, rows_i: np.ndarray, side: str = "row") -> np.ndarray:
    """Table row index of every pair (i in rows_i, j in [0, L)).

    side="row" is the query-side table (T5 bucket, Shaw a, TXL r, DeBERTa Kr);
    side="col" is DeBERTa's key-side table Qr.
    """
    n = _rel(rows_i, L)  # j - i
    if mech == T5:
        return t5_bucket(n, cfg.t5_num_buckets, cfg.t5_max_distance, cfg.t5_bidirectional)
    if mech == SHAW:
        c = cfg.shaw_clip
        return np.clip(n, -c, c) + c
    if mech == TXL:
        delta = -n  # i - j
        return delta if causal else delta + (L - 1)
    k = cfg.deberta_span
    if side == "row":
        return np.clip(-n + k, 0, 2 * k - 1)  # delta(i, j) = clip(i - j + k)
    return np.clip(n + k, 0, 2 * k - 1)  # delta(j, i) = clip(j - i + k)


def _mask(L: int, causal: bool, rows_i: np.ndarray, lk=None) -> np.ndarray:
    """True where the pair is allowed: j <= i when causal, and j < lk (the batch's
    key length) when one is given."""
    allowed = np.ones((rows_i.size, L), dtype=bool) if not causal else _rel(rows_i, L) <= 0
    if lk is not None:
        allowed &= np.arange(L)[None, :] < int(lk)
    return allowed


# --------------------------------------------------------------------------
# Scores of one (batch, head): S = s q k^T + B, with B materialised
# --------------------------------------------------------------------------
def head_bias(mech, q, k, rel_h, scale, cfg, causal, rows_i):
    """The additive term B (as it enters S) for rows_i of one (b, h).

    q, k: [L, d] float64; rel_h: this head's tables.  Returns [len(rows_i), L].
    The (q+u).k part of Transformer-XL is returned here too (as u.k_j), so that
    S = scale * q k^T + B for every mechanism.
    """
    L = k.shape[0]
    qi = q[rows_i]
    if mech == ALIBI:
        (m,) = rel_h
        return -float(m) * np.abs(_rel(rows_i, L)).astype(np.float64)
    if mech == T5:
        (t,) = rel_h
        return t[index_map(T5, L, causal, cfg, rows_i)]
    if mech == SHAW:
        a = rel_h[0]  # rel_h[1], the value-side table, does not enter the scores
        qa = qi @ a.T  # [rows, 2c+1]: every q_i . a_r
        idx = index_map(SHAW, L, causal, cfg, rows_i)
        return scale * np.take_along_axis(qa, idx, axis=1)
    if mech == TXL:
        r, u, v = rel_h
        idx = index_map(TXL, L, causal, cfg, rows_i)
        valid = (idx >= 0) & (idx < r.shape[0])
        qr = (qi + v) @ r.T  # [rows, n_off]
        pos = np.where(valid, np.take_along_axis(qr, np.clip(idx, 0, r.shape[0] - 1), axis=1), 0.0)
        uk = k @ u  # [L]
        return scale * (uk[None, :] + pos)
    Kr, Qr = rel_h
    idx_c2p = index_map(DEBERTA, L, causal, cfg, rows_i, "row")
    idx_p2c = index_map(DEBERTA, L, causal, cfg, rows_i, "col")
    c2p = np.take_along_axis(qi @ Kr.T, idx_c2p, axis=1)  # q_i . Kr[delta(i,j)]
    kq = k @ Qr.T  # [L, 2k]: k_j . Qr_r
    p2c = kq[np.arange(L)[None, :], idx_p2c]  # k_j . Qr[delta(j,i)]
    return scale * (c2p + p2c)


def head_scores(mech, q, k, rel_h, scale, cfg, causal, rows_i, lk=None):
    """S rows for one (b, h): scale q_i.k_j + B_ij, -inf where masked."""
    S = scale * (q[rows_i] @ k.T) + head_bias(mech, q, k, rel_h, scale, cfg, causal, rows_i)
    return np.where(_mask(k.shape[0], causal, rows_i, lk), S, -np.inf)


def _lk(seqlens_k, b):
    return None if seqlens_k is None else int(seqlens_k[b])


def _softmax_rows(S):
    """Row softmax and natural-log LSE; fully masked rows give P = 0, LSE = -inf."""
    m = np.max(S, axis=1, keepdims=True)
    finite = np.isfinite(m)
    m0 = np.where(finite, m, 0.0)
    e = np.exp(S - m0)
    z = e.sum(axis=1, keepdims=True)
    P = np.where(finite, e / np.where(z > 0, z, 1.0), 0.0)
    lse = np.where(finite[:, 0], m0[:, 0] + np.log(np.where(z[:, 0] > 0, z[:, 0], 1.0)), -np.inf)
    return P, lse


def _head_tables(mech, rel, h):
    return tuple(np.asarray(x[h], dtype=np.float64) for x in rel)


def _value_term(mech, cfg):
    return mech == SHAW and cfg.shaw_value


def _by_offset(X, mech, L, causal, cfg, rows_i, nrows):
    """Pe[r, rho] = sum of X[r, j] over the keys j whose pair (rows_i[r], j) reads
    table row rho (X is zero on masked pairs)."""
    idx = index_map(mech, L, causal, cfg, rows_i)
    Pe = np.zeros((rows_i.size, nrows))
    np.add.at(Pe, (np.repeat(np.arange(rows_i.size), L), idx.ravel()), X.ravel())
    return Pe


# --------------------------------------------------------------------------
# Public entry points
# --------------------------------------------------------------------------
def forward(mech, q, k, v, rel, causal, scale=None, cfg=RelCfg(), rows=None, seqlens_k=None):
    """O [B,H,R,d] and LSE [B,H,R] for the query rows ``rows`` (default: all);
    ``seqlens_k`` (optional, [B]) masks each batch's keys j >= seqlens_k[b].

    q, k, v: [B, H, L, d]; rel: list of per-head tables (see module docstring):
    T5 [t (H,nb)], Shaw [a (H,2c+1,d)], TXL [r (H,n_off,d), u (H,d), v (H,d)],
    DeBERTa [Kr (H,2k,d), Qr (H,2k,d)], ALiBi [m (H,)].
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, H, L, d = q.shape
    scale = default_scale(mech, d) if scale is None else scale
    rows_i = np.arange(L) if rows is None else np.asarray(rows, dtype=np.int64)
    O = np.zeros((B, H, rows_i.size, d))
    LSE = np.zeros((B, H, rows_i.size))
    for b in range(B):
        for h in range(H):
            rh = _head_tables(mech, rel, h)
            S = head_scores(mech, q[b, h], k[b, h], rh, scale, cfg, causal, rows_i, _lk(seqlens_k, b))
            P, lse = _softmax_rows(S)
            O[b, h] = P @ v[b, h]
            if _value_term(mech, cfg):
                O[b, h] += _by_offset(P, mech, L, causal, cfg, rows_i, rh[1].shape[0]) @ rh[1]
            LSE[b, h] = lse
    return O, LSE


def backward(mech, q, k, v, rel, causal, dO, scale=None, cfg=RelCfg(), seqlens_k=None):
    """Exact gradients (dq, dk, dv, drel) of  sum(O * dO).

    drel matches rel's structure: T5 [dt], Shaw [da] (+ daV with the value term), TXL [dr, du, dv],
    DeBERTa [dKr, dQr], ALiBi [dm]; table gradients sum over the batch (tables
    are per head).
    """
    q, k, v, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dO))
    B, H, L, d = q.shape
    scale = default_scale(mech, d) if scale is None else scale
    rows_i = np.arange(L)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    drel = [np.zeros(np.shape(x), dtype=np.float64) for x in rel]
    for b in range(B):
        for h in range(H):
            rh = _head_tables(mech, rel, h)
            qh, kh, vh, gh = q[b, h], k[b, h], v[b, h], dO[b, h]
            S = head_scores(mech, qh, kh, rh, scale, cfg, causal, rows_i, _lk(seqlens_k, b))
            P, _ = _softmax_rows(S)
            O = P @ vh
            dP = gh @ vh.T
            if _value_term(mech, cfg):  # O_i += sum_j P_ij aV_rho: dP_ij += dO_i . aV_rho, daV += Pe^T dO
                aV = rh[1]
                Pe = _by_offset(P, mech, L, causal, cfg, rows_i, aV.shape[0])
                O = O + Pe @ aV
                dP = dP + np.take_along_axis(gh @ aV.T, index_map(mech, L, causal, cfg, rows_i), axis=1)
                drel[1][h] += Pe.T @ gh
            D = np.sum(gh * O, axis=1)
            dS = P * (dP - D[:, None])
            dv[b, h] = P.T @ gh
            # content term scale * q_i . k_j
            dq[b, h] = scale * (dS @ kh)
            dk[b, h] = scale * (dS.T @ qh)
            if mech == ALIBI:
                drel[0][h] += np.sum(dS * -np.abs(_rel(rows_i, L)))
            elif mech == T5:
                idx = index_map(T5, L, causal, cfg, rows_i)
                np.add.at(drel[0][h], idx.ravel(), dS.ravel())
            elif mech == SHAW:
                a = rh[0]
                idx = index_map(SHAW, L, causal, cfg, rows_i)
                M = np.zeros((L, a.shape[0]))  # M[i, r] = sum_{j: idx=r} dS_ij
                np.add.at(M, (np.repeat(rows_i, L), idx.ravel()), dS.ravel())
                dq[b, h] += scale * (M @ a)
                drel[0][h] += scale * (M.T @ qh)
            elif mech == TXL:
                r, u, vv = rh
                idx = index_map(TXL, L, causal, cfg, rows_i)
                allowed = _mask(L, causal, rows_i, _lk(seqlens_k, b))
                M = np.zeros((L, r.shape[0]))
                sel = allowed.ravel()
                np.add.at(M, (np.repeat(rows_i, L)[sel], idx.ravel()[sel]), dS.ravel()[sel])
                dq[b, h] += scale * (M @ r)
                dk[b, h] += scale * np.outer(dS.sum(axis=0), u)  # (q_i + u) . k_j
                drel[0][h] += scale * (M.T @ (qh + vv))
                drel[1][h] += scale * (dS.sum(axis=0) @ kh)
                drel[2][h] += scale * (M.sum(axis=0) @ r)
            else:
                Kr, Qr = rh
                idx_r = index_map(DEBERTA, L, causal, cfg, rows_i, "row")
                idx_c = index_map(DEBERTA, L, causal, cfg, rows_i, "col")
                M = np.zeros((L, Kr.shape[0]))  # query side: M[i, r]
                np.add.at(M, (np.repeat(rows_i, L), idx_r.ravel()), dS.ravel())
                N = np.zeros((L, Qr.shape[0]))  # key side: N[j, r] = sum_{i: idx_c=r} dS_ij
                np.add.at(N, (np.tile(np.arange(L), L), idx_c.ravel()), dS.ravel())
                dq[b, h] += scale * (M @ Kr)
                dk[b, h] += scale * (N @ Qr)
                drel[0][h] += scale * (M.T @ qh)
                drel[1][h] += scale * (N.T @ kh)
    return dq, dk, dv, drel


def backward_rows(mech, q, k, v, rel, causal, dO, rows, scale=None, cfg=RelCfg(), seqlens_k=None):
    """dq for the query rows ``rows`` only (each is a function of its own row of
    dS, which needs only that row's O, so no full pass is required)."""
    q, k, v, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dO))
    B, H, L, d = q.shape
    scale = default_scale(mech, d) if scale is None else scale
    rows_i = np.asarray(rows, dtype=np.int64)
    dq = np.zeros((B, H, rows_i.size, d))
    for b in range(B):
        for h in range(H):
            rh = _head_tables(mech, rel, h)
            qh, kh, vh, gh = q[b, h], k[b, h], v[b, h], dO[b, h]
            S = head_scores(mech, qh, kh, rh, scale, cfg, causal, rows_i, _lk(seqlens_k, b))
            P, _ = _softmax_rows(S)
            O = P @ vh
            dP = gh[rows_i] @ vh.T
            if _value_term(mech, cfg):
                aV = rh[1]
                O = O + _by_offset(P, mech, L, causal, cfg, rows_i, aV.shape[0]) @ aV
                dP = dP + np.take_along_axis(gh[rows_i] @ aV.T, index_map(mech, L, causal, cfg, rows_i), axis=1)
            D = np.sum(gh[rows_i] * O, axis=1)
            dS = P * (dP - D[:, None])
            g = scale * (dS @ kh)
            if mech in (SHAW, TXL, DEBERTA):
                tab = rh[0]
                idx = index_map(mech, L, causal, cfg, rows_i, "row")
                allowed = _mask(L, causal, rows_i, _lk(seqlens_k, b))
                M = np.zeros((rows_i.size, tab.shape[0]))
                sel = allowed.ravel()
                np.add.at(M, (np.repeat(np.arange(rows_i.size), L)[sel], idx.ravel()[sel]), dS.ravel()[sel])
                g += scale * (M @ tab)
            dq[b, h] = g
    return dq


# --------------------------------------------------------------------------
# Transformer-XL with memory (Dai et al.): the current segment's L queries attend to the
# cached previous segment's M keys / values followed by the segment's own L; query i sits
# at absolute position M + i, so S_ij = s ((q_i + u).k_j + (q_i + v).r[M + i - j]) for
# keys j <= M + i (causal), and r has M + L rows.  This is exactly the causal attention of
# the concatenated M + L positions read at its last L query rows, which is how it is
# computed here (the first M query rows are placeholders with zero output gradient).
# --------------------------------------------------------------------------
def _with_memory(q, m_len):
    B, H, L, d = q.shape
    return np.concatenate([np.zeros((B, H, m_len, d)), np.asarray(q, dtype=np.float64)], axis=2)


def txl_memory_forward(q, k, v, rel, scale=None, cfg=RelCfg()):
    """O [B,H,L,d] and LSE [B,H,L] of Transformer-XL with memory: q [B,H,L,d] is the
    current segment, k and v [B,H,M+L,d] the memory followed by the segment, rel =
    [r (H, M+L, d), u (H, d), v (H, d)]."""
    m_len = np.shape(k)[2] - np.shape(q)[2]
    assert m_len >= 0, "keys must cover the memory and the segment"
    qf = _with_memory(q, m_len)
    rows = np.arange(m_len, qf.shape[2])
    return forward(TXL, qf, k, v, rel, True, scale, cfg, rows=rows)


def txl_memory_backward(q, k, v, rel, dO, scale=None, cfg=RelCfg()):
    """Gradients (dq [B,H,L,d], dk, dv [B,H,M+L,d], drel) of sum(O * dO) for
    txl_memory_forward; the memory's keys and values get gradients like any key."""
    m_len = np.shape(k)[2] - np.shape(q)[2]
    assert m_len >= 0, "keys must cover the memory and the segment"
    qf = _with_memory(q, m_len)
    gf = _with_memory(dO, m_len)
    dq, dk, dv, drel = backward(TXL, qf, k, v, rel, True, gf, scale, cfg)
    return dq[:, :, m_len:], dk, dv, drel
