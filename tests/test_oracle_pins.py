"""Pins of the fp64 oracle against things other than itself.

* hand-written T5 bucket table (tests/golden),
* brute force: scalar Python loops straight from each mechanism's formula,
  forward and scalar chain-rule backward, on tiny shapes with small clip /
  span / bucket parameters so that clipping and bucketing are exercised,
* central finite differences of sum(O * dO) for every input and parameter,
* closed forms (L = 1; causal row 0; ALiBi with q.k = 0: geometric sums),
* zero relative term == plain softmax attention, checked against
  torch.nn.functional.scaled_dot_product_attention (fp64, CPU) and autograd,
* row-constant terms leave O unchanged and shift LSE; the gradient of every
  query-side table sums to zero (because each row of dS sums to zero).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle as orc
from oracle import ALIBI, DEBERTA, SHAW, T5, TXL, RelCfg

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SMALL = RelCfg(t5_num_buckets=8, t5_max_distance=6, t5_bidirectional=True, shaw_clip=2, deberta_span=2)


def rnd(rng, *shape, std=1.0):
    return rng.standard_normal(shape) * std


def make_case(mech, B, H, L, d, causal, cfg, seed=0, zero_rel=False):
    rng = np.random.default_rng(seed)
    q, k, v, do = (rnd(rng, B, H, L, d) for _ in range(4))
    nrows = orc.table_rows(mech, L, causal, cfg)
    sc = 0.0 if zero_rel else 1.0
    if mech == ALIBI:
        rel = [sc * (0.05 + np.abs(rnd(rng, H, std=0.5)))]
    elif mech == T5:
        rel = [sc * rnd(rng, H, nrows, std=0.5)]
    elif mech == SHAW:
        rel = [sc * rnd(rng, H, nrows, d, std=0.5)]
    elif mech == TXL:
        rel = [sc * rnd(rng, H, nrows, d, std=0.5), sc * rnd(rng, H, d, std=0.5), sc * rnd(rng, H, d, std=0.5)]
    else:
        rel = [sc * rnd(rng, H, nrows, d, std=0.5), sc * rnd(rng, H, nrows, d, std=0.5)]
    return q, k, v, do, rel


# ----------------------------------------------------------------------------
# golden T5 buckets
# ----------------------------------------------------------------------------
def test_t5_buckets_golden():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "t5_buckets_nb32_md128.txt")) if ln.strip() and not ln.startswith("#")]
    n = np.array([int(a) for a, _ in rows])
    want = np.array([int(b) for _, b in rows])
    got = orc.t5_bucket(n, 32, 128, True)
    assert np.array_equal(got, want), list(zip(n[got != want], got[got != want], want[got != want]))
    # the vectorised (look-up) branch gives the same values as the direct branch
    big = np.arange(-9000, 9000)
    direct = np.concatenate([orc.t5_bucket(big[i:i + 4000], 32, 128, True) for i in range(0, big.size, 4000)])
    assert np.array_equal(orc.t5_bucket(big, 32, 128, True), direct)


def test_t5_buckets_match_float_formula_away_from_ties():
    """Away from the exact boundaries a = 16, 32, 64 the integer form equals the
    float formula of the T5 paper."""
    for n in range(-300, 301):
        a = abs(n)
        if a in (16, 32, 64):
            continue
        base = 16 if n > 0 else 0
        if a < 8:
            want = base + a
        else:
            want = base + min(15, 8 + int(math.log(a / 8) / math.log(128 / 8) * 8))
        assert int(orc.t5_bucket(np.array([n]))[0]) == want, n


def test_t5_unidirectional():
    # causal T5: only n <= 0 distinguishes buckets; nb = 32 all on one side
    got = orc.t5_bucket(np.array([5, 1, 0, -1, -15, -16, -200]), 32, 128, False)
    # max_exact = 16: a < 16 exact; a >= 16 -> 16 + floor(log(a/16)/log(8) * 16)
    want = [0, 0, 0, 1, 15, 16, 31]
    assert got.tolist() == want


# ----------------------------------------------------------------------------
# brute force
# ----------------------------------------------------------------------------
def bf_bucket(n, cfg):
    nb = cfg.t5_num_buckets // 2
    base = nb if n > 0 else 0
    a = abs(n)
    me = nb // 2
    if a < me:
        return base + a
    return base + min(nb - 1, me + int(math.log(a / me) / math.log(cfg.t5_max_distance / me) * (nb - me)))


def dot(x, y):
    return sum(float(a) * float(b) for a, b in zip(x, y))


def bf_score(mech, q, k, rel, h, i, j, L, causal, s, cfg):
    """S_ij straight from the mechanism's formula."""
    if mech == ALIBI:
        return s * dot(q[i], k[j]) - rel[0][h] * abs(j - i)
    if mech == T5:
        return s * dot(q[i], k[j]) + rel[0][h][bf_bucket(j - i, cfg)]
    if mech == SHAW:
        c = cfg.shaw_clip
        return s * (dot(q[i], k[j]) + dot(q[i], rel[0][h][max(-c, min(c, j - i)) + c]))
    if mech == TXL:
        r, u, vv = rel
        row = (i - j) if causal else (i - j + L - 1)
        return s * (dot(q[i] + u[h], k[j]) + dot(q[i] + vv[h], r[h][row]))
    sp = cfg.deberta_span
    c2p = max(0, min(2 * sp - 1, i - j + sp))
    p2c = max(0, min(2 * sp - 1, j - i + sp))
    return s * (dot(q[i], k[j]) + dot(q[i], rel[0][h][c2p]) + dot(k[j], rel[1][h][p2c]))


def bf_value_row(cfg, i, j):
    c = cfg.shaw_clip
    return max(-c, min(c, j - i)) + c


def brute(mech, q, k, v, rel, causal, do, s, cfg, lk=None):
    """Scalar loops over (i, j) from the mechanism formulas; lk[b] (optional) is the
    batch's key length: keys j >= lk[b] do not take part.  With Shaw's value term
    (cfg.shaw_value) every value v_j is read as v_j + aV[row(i, j)]."""
    val = mech == SHAW and cfg.shaw_value
    B, H, L, d = q.shape
    O = np.zeros_like(q)
    LSE = np.zeros((B, H, L))
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    drel = [np.zeros_like(x) for x in rel]
    for b in range(B):
        for h in range(H):
            qb, kb, vb, gb = q[b, h], k[b, h], v[b, h], do[b, h]
            P = np.zeros((L, L))
            for i in range(L):
                keys = [j for j in range(L) if not (causal and j > i) and (lk is None or j < lk[b])]
                if not keys:  # empty key set: O = 0, LSE = -inf, no gradient
                    LSE[b, h, i] = -math.inf
                    continue
                sc = {j: bf_score(mech, qb, kb, rel, h, i, j, L, causal, s, cfg) for j in keys}
                m = max(sc.values())
                z = sum(math.exp(x - m) for x in sc.values())
                LSE[b, h, i] = m + math.log(z)
                for j in keys:
                    P[i, j] = math.exp(sc[j] - m) / z
                for c in range(d):
                    O[b, h, i, c] = sum(P[i, j] * (vb[j, c] + (rel[1][h][bf_value_row(cfg, i, j)][c] if val else 0.0))
                                        for j in keys)
            for i in range(L):
                Di = dot(gb[i], O[b, h, i])
                for j in range(L):
                    if (causal and j > i) or (lk is not None and j >= lk[b]):
                        continue
                    vj = vb[j] + (rel[1][h][bf_value_row(cfg, i, j)] if val else 0.0)
                    dS = P[i, j] * (dot(gb[i], vj) - Di)
                    dv[b, h, j] += P[i, j] * gb[i]
                    if val:
                        drel[1][h][bf_value_row(cfg, i, j)] += P[i, j] * gb[i]
                    dq[b, h, i] += s * dS * kb[j]
                    dk[b, h, j] += s * dS * qb[i]
                    if mech == ALIBI:
                        drel[0][h] += dS * -abs(j - i)
                    elif mech == T5:
                        drel[0][h][bf_bucket(j - i, cfg)] += dS
                    elif mech == SHAW:
                        c = cfg.shaw_clip
                        rr = max(-c, min(c, j - i)) + c
                        dq[b, h, i] += s * dS * rel[0][h][rr]
                        drel[0][h][rr] += s * dS * qb[i]
                    elif mech == TXL:
                        r, u, vv = rel
                        row = (i - j) if causal else (i - j + L - 1)
                        dq[b, h, i] += s * dS * r[h][row]
                        dk[b, h, j] += s * dS * u[h]
                        drel[0][h][row] += s * dS * (qb[i] + vv[h])
                        drel[1][h] += s * dS * kb[j]
                        drel[2][h] += s * dS * r[h][row]
                    else:
                        sp = cfg.deberta_span
                        c2p = max(0, min(2 * sp - 1, i - j + sp))
                        p2c = max(0, min(2 * sp - 1, j - i + sp))
                        dq[b, h, i] += s * dS * rel[0][h][c2p]
                        dk[b, h, j] += s * dS * rel[1][h][p2c]
                        drel[0][h][c2p] += s * dS * qb[i]
                        drel[1][h][p2c] += s * dS * kb[j]
    return O, LSE, dq, dk, dv, drel


MECHS = (T5, SHAW, TXL, DEBERTA, ALIBI)
CASES = [(mech, causal, L, d) for mech in MECHS for causal in (False, True)
         for (L, d) in ((1, 2), (2, 1), (3, 4), (5, 2), (8, 4))]


@pytest.mark.parametrize("mech,causal,L,d", CASES)
def test_oracle_vs_brute_force(mech, causal, L, d):
    q, k, v, do, rel = make_case(mech, 2, 2, L, d, causal, SMALL, seed=L * 10 + d)
    s = 0.37
    O, LSE = orc.forward(mech, q, k, v, rel, causal, s, SMALL)
    dq, dk, dv, drel = orc.backward(mech, q, k, v, rel, causal, do, s, SMALL)
    bO, bL, bdq, bdk, bdv, bdrel = brute(mech, q, k, v, rel, causal, do, s, SMALL)
    for got, want in [(O, bO), (LSE, bL), (dq, bdq), (dk, bdk), (dv, bdv)] + list(zip(drel, bdrel)):
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    # the row-subset entry points agree with the full ones
    rows = np.arange(L)[::2]
    O2, L2 = orc.forward(mech, q, k, v, rel, causal, s, SMALL, rows=rows)
    np.testing.assert_allclose(O2, O[:, :, rows], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(L2, LSE[:, :, rows], rtol=1e-13, atol=1e-13)
    dq2 = orc.backward_rows(mech, q, k, v, rel, causal, do, rows, s, SMALL)
    np.testing.assert_allclose(dq2, dq[:, :, rows], rtol=1e-12, atol=1e-12)


SEQ_CASES = [(mech, causal, L, lk) for mech in MECHS for causal in (False, True)
             for (L, lk) in ((3, (2, 0)), (5, (5, 1)), (8, (3, 7)))]


@pytest.mark.parametrize("mech,causal,L,lk", SEQ_CASES)
def test_oracle_key_lengths_vs_brute_force(mech, causal, L, lk):
    """Variable key lengths: the oracle's masked path against the scalar loops."""
    q, k, v, do, rel = make_case(mech, 2, 2, L, 2, causal, SMALL, seed=L * 7 + lk[0])
    s = 0.41
    O, LSE = orc.forward(mech, q, k, v, rel, causal, s, SMALL, seqlens_k=lk)
    dq, dk, dv, drel = orc.backward(mech, q, k, v, rel, causal, do, s, SMALL, seqlens_k=lk)
    bO, bL, bdq, bdk, bdv, bdrel = brute(mech, q, k, v, rel, causal, do, s, SMALL, lk=lk)
    np.testing.assert_array_equal(np.isneginf(LSE), np.isneginf(bL))
    fin = np.isfinite(bL)
    np.testing.assert_allclose(LSE[fin], bL[fin], rtol=1e-12, atol=1e-12)
    for got, want in [(O, bO), (dq, bdq), (dk, bdk), (dv, bdv)] + list(zip(drel, bdrel)):
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    rows = np.arange(L)[1::2]
    dq2 = orc.backward_rows(mech, q, k, v, rel, causal, do, rows, s, SMALL, seqlens_k=lk)
    np.testing.assert_allclose(dq2, dq[:, :, rows], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mech", MECHS)
def test_padding_keys_do_not_matter(mech):
    """Keys past a batch's length change nothing but get zero dk, dv; an empty key
    set gives O = 0, LSE = -inf and zero gradients; a full length is no mask."""
    L = 7
    q, k, v, do, rel = make_case(mech, 2, 2, L, 4, False, SMALL, seed=11)
    lk = (4, 0)
    base = orc.forward(mech, q, k, v, rel, False, 0.3, SMALL, seqlens_k=lk)
    gb = orc.backward(mech, q, k, v, rel, False, do, 0.3, SMALL, seqlens_k=lk)
    k2, v2 = k.copy(), v.copy()
    rng = np.random.default_rng(5)
    k2[0, :, 4:] = rng.standard_normal(k2[0, :, 4:].shape)
    v2[0, :, 4:] = rng.standard_normal(v2[0, :, 4:].shape)
    k2[1] = rng.standard_normal(k2[1].shape)
    v2[1] = rng.standard_normal(v2[1].shape)
    alt = orc.forward(mech, q, k2, v2, rel, False, 0.3, SMALL, seqlens_k=lk)
    ga = orc.backward(mech, q, k2, v2, rel, False, do, 0.3, SMALL, seqlens_k=lk)
    np.testing.assert_allclose(alt[0], base[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(alt[1], base[1])
    np.testing.assert_allclose(ga[0], gb[0], rtol=1e-12, atol=1e-13)  # dq
    for t in range(len(rel)):  # table gradients (TXL du = s sum_j c_j k_j: masked keys have c_j = 0)
        np.testing.assert_allclose(ga[3][t], gb[3][t], rtol=1e-12, atol=1e-13)
    assert np.all(gb[1][0, :, 4:] == 0) and np.all(gb[2][0, :, 4:] == 0)
    assert np.all(base[0][1] == 0) and np.all(np.isneginf(base[1][1]))
    assert all(np.all(g[1] == 0) for g in gb[:3])
    full = orc.forward(mech, q, k, v, rel, False, 0.3, SMALL, seqlens_k=(L, L))
    plain = orc.forward(mech, q, k, v, rel, False, 0.3, SMALL)
    np.testing.assert_array_equal(full[0], plain[0])
    np.testing.assert_array_equal(full[1], plain[1])


# ----------------------------------------------------------------------------
# Shaw's value-side term
# ----------------------------------------------------------------------------
VAL = RelCfg(shaw_clip=2, shaw_value=True)


def value_case(B, H, L, d, seed):
    rng = np.random.default_rng(seed)
    q, k, v, do = (rnd(rng, B, H, L, d) for _ in range(4))
    rel = [rnd(rng, H, 2 * VAL.shaw_clip + 1, d, std=0.5), rnd(rng, H, 2 * VAL.shaw_clip + 1, d, std=0.5)]
    return q, k, v, do, rel


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L,lk", [(1, None), (3, None), (7, None), (8, (8, 3))])
def test_shaw_value_term_vs_brute_force(causal, L, lk):
    q, k, v, do, rel = value_case(2, 2, L, 3, seed=L + 5)
    s = 0.45
    O, LSE = orc.forward(SHAW, q, k, v, rel, causal, s, VAL, seqlens_k=lk)
    dq, dk, dv, drel = orc.backward(SHAW, q, k, v, rel, causal, do, s, VAL, seqlens_k=lk)
    bO, bL, bdq, bdk, bdv, bdrel = brute(SHAW, q, k, v, rel, causal, do, s, VAL, lk=lk)
    for got, want in [(O, bO), (LSE, bL), (dq, bdq), (dk, bdk), (dv, bdv)] + list(zip(drel, bdrel)):
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    rows = np.arange(L)[::2]
    dq2 = orc.backward_rows(SHAW, q, k, v, rel, causal, do, rows, s, VAL, seqlens_k=lk)
    np.testing.assert_allclose(dq2, dq[:, :, rows], rtol=1e-12, atol=1e-12)
    O2, _ = orc.forward(SHAW, q, k, v, rel, causal, s, VAL, rows=rows, seqlens_k=lk)
    np.testing.assert_allclose(O2, O[:, :, rows], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_shaw_value_term_finite_differences(causal):
    q, k, v, do, rel = value_case(1, 2, 11, 4, seed=3)
    s = 0.4

    def loss(rel_):
        return float(np.sum(orc.forward(SHAW, q, k, v, rel_, causal, s, VAL)[0] * do))

    _, _, _, drel = orc.backward(SHAW, q, k, v, rel, causal, do, s, VAL)
    rng = np.random.default_rng(8)
    for n in range(2):
        e = rng.standard_normal(rel[n].shape)
        rp, rm = list(rel), list(rel)
        rp[n] = rel[n] + 1e-6 * e
        rm[n] = rel[n] - 1e-6 * e
        fd = (loss(rp) - loss(rm)) / 2e-6
        an = float(np.sum(drel[n] * e))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (n, fd, an)


def test_shaw_value_term_constant_rows_shift_the_output():
    """aV rows all equal to w: each row of P sums to one, so O = O_plain + w, the
    scores (LSE, dq, dk) do not change, and the daV rows add up to sum_i dO_i."""
    q, k, v, do, rel = value_case(2, 2, 9, 4, seed=4)
    w = np.random.default_rng(1).standard_normal((2, 4))
    aV = np.repeat(w[:, None, :], 2 * VAL.shaw_clip + 1, axis=1)
    plain = RelCfg(shaw_clip=2)
    O0, L0 = orc.forward(SHAW, q, k, v, rel[:1], False, 0.5, plain)
    O1, L1 = orc.forward(SHAW, q, k, v, [rel[0], aV], False, 0.5, VAL)
    np.testing.assert_allclose(O1, O0 + w[None, :, None, :], atol=1e-12)
    np.testing.assert_array_equal(L1, L0)
    g0 = orc.backward(SHAW, q, k, v, rel[:1], False, do, 0.5, plain)
    g1 = orc.backward(SHAW, q, k, v, [rel[0], aV], False, do, 0.5, VAL)
    for a, b in zip(list(g0[:3]) + [g0[3][0]], list(g1[:3]) + [g1[3][0]]):
        np.testing.assert_allclose(b, a, atol=1e-11)
    np.testing.assert_allclose(g1[3][1].sum(axis=1), do.sum(axis=(0, 2)), atol=1e-11)


# ----------------------------------------------------------------------------
# finite differences
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mech", MECHS)
@pytest.mark.parametrize("causal", [False, True])
def test_oracle_finite_differences(mech, causal):
    L, d = 13, 4
    q, k, v, do, rel = make_case(mech, 2, 2, L, d, causal, SMALL, seed=7 + mech)
    s = 0.41

    def loss(q_, k_, v_, rel_):
        O, _ = orc.forward(mech, q_, k_, v_, rel_, causal, s, SMALL)
        return float(np.sum(O * do))

    dq, dk, dv, drel = orc.backward(mech, q, k, v, rel, causal, do, s, SMALL)
    rng = np.random.default_rng(123)
    eps = 1e-6
    params = [("q", q, dq), ("k", k, dk), ("v", v, dv)] + [(f"rel{n}", rel[n], drel[n]) for n in range(len(rel))]
    for name, x, g in params:
        e = rng.standard_normal(x.shape)

        def at(sign, name=name, e=e):
            args = {"q": q, "k": k, "v": v}
            rr = list(rel)
            if name in args:
                args[name] = args[name] + sign * eps * e
            else:
                n = int(name[3:])
                rr[n] = rr[n] + sign * eps * e
            return loss(args["q"], args["k"], args["v"], rr)

        fd = (at(+1) - at(-1)) / (2 * eps)
        an = float(np.sum(g * e))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


# ----------------------------------------------------------------------------
# closed forms
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mech", MECHS)
def test_closed_form_L1(mech):
    q, k, v, do, rel = make_case(mech, 1, 3, 1, 8, False, RelCfg(), seed=3)
    s = orc.default_scale(mech, 8)
    O, LSE = orc.forward(mech, q, k, v, rel, False, s)
    np.testing.assert_allclose(O, v, rtol=0, atol=1e-15)
    S00 = np.array([[bf_score(mech, q[0, h], k[0, h], rel, h, 0, 0, 1, False, s, RelCfg()) for h in range(3)]])
    np.testing.assert_allclose(LSE[..., 0], S00, rtol=1e-13, atol=1e-13)
    dq, dk, dv, drel = orc.backward(mech, q, k, v, rel, False, do, s)
    np.testing.assert_allclose(dv, do, atol=1e-15)
    for g in [dq, dk] + drel:
        np.testing.assert_allclose(g, 0.0, atol=1e-13)


@pytest.mark.parametrize("mech", MECHS)
def test_closed_form_causal_row0(mech):
    q, k, v, do, rel = make_case(mech, 1, 2, 6, 4, True, SMALL, seed=5)
    O, _ = orc.forward(mech, q, k, v, rel, True, 0.5, SMALL)
    np.testing.assert_allclose(O[:, :, 0], v[:, :, 0], atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_alibi_geometric_closed_form(causal):
    """q = 0 leaves only the ALiBi term: row i's softmax weights are e^{-m |j - i|},
    so LSE_i = ln(sum_{t=0}^{i} e^{-m t} + [not causal] sum_{t=1}^{L-1-i} e^{-m t})
    (geometric sums), and with v_j = e^{-m j} (causal) every key contributes
    e^{-m i} / Z_i, so O_i = (i + 1) e^{-m i} / Z_i."""
    L, H = 50, 3
    m = np.array([0.03, 0.5, 2.0])
    q = np.zeros((1, H, L, 1))
    k = np.random.default_rng(2).standard_normal((1, H, L, 1))
    j = np.arange(L, dtype=np.float64)
    v = np.broadcast_to(np.exp(-m[:, None] * j[None, :])[None, :, :, None], (1, H, L, 1)).copy()
    O, LSE = orc.forward(ALIBI, q, k, v, [m], causal, 1.0)

    def geo(n, mm):  # sum_{t=0}^{n-1} e^{-mm t}
        return (1.0 - np.exp(-mm * n)) / (1.0 - np.exp(-mm))

    for h in range(H):
        i = np.arange(L)
        Z = geo(i + 1, m[h]) + (0.0 if causal else geo(L - i, m[h]) - 1.0)
        np.testing.assert_allclose(LSE[0, h], np.log(Z), rtol=1e-13, atol=1e-13)
        if causal:
            np.testing.assert_allclose(O[0, h, :, 0], (i + 1) * np.exp(-m[h] * i) / Z, rtol=1e-12)


# ----------------------------------------------------------------------------
# zero relative term == plain attention (independent library routine)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mech", MECHS)
@pytest.mark.parametrize("causal", [False, True])
def test_zero_term_is_plain_attention(mech, causal):
    L, d = 37, 16
    q, k, v, do, rel = make_case(mech, 2, 3, L, d, causal, RelCfg(), seed=11, zero_rel=True)
    s = orc.default_scale(mech, d)
    O, LSE = orc.forward(mech, q, k, v, rel, causal, s)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=s)
    np.testing.assert_allclose(O, ref.detach().numpy(), rtol=1e-12, atol=1e-12)
    lse_ref = torch.logsumexp(s * tq @ tk.transpose(-1, -2) + (torch.triu(torch.full((L, L), -math.inf, dtype=torch.float64), 1) if causal else 0.0), dim=-1)
    np.testing.assert_allclose(LSE, lse_ref.detach().numpy(), rtol=1e-12, atol=1e-12)
    ref.backward(torch.tensor(do))
    dq, dk, dv, _ = orc.backward(mech, q, k, v, rel, causal, do, s)
    for got, want in [(dq, tq.grad), (dk, tk.grad), (dv, tv.grad)]:
        np.testing.assert_allclose(got, want.numpy(), rtol=1e-10, atol=1e-11)


# ----------------------------------------------------------------------------
# row-constant invariants and gradient sums
# ----------------------------------------------------------------------------
def test_row_constant_terms_leave_output_unchanged():
    L, d, H = 29, 8, 2
    cfg = RelCfg(shaw_clip=5, deberta_span=4)
    rng = np.random.default_rng(9)
    q, k, v = (rnd(rng, 1, H, L, d) for _ in range(3))
    s = 0.3
    # T5: constant table -> every score shifted by the same constant
    t = np.full((H, 32), 0.7)
    O0, L0 = orc.forward(T5, q, k, v, [np.zeros((H, 32))], False, s)
    O1, L1 = orc.forward(T5, q, k, v, [t], False, s)
    np.testing.assert_allclose(O1, O0, atol=1e-13)
    np.testing.assert_allclose(L1, L0 + 0.7, atol=1e-12)
    # Shaw: all rows equal -> q_i . a is row-constant
    a_row = rnd(rng, H, d)
    a = np.repeat(a_row[:, None, :], 2 * cfg.shaw_clip + 1, axis=1)
    O2, L2 = orc.forward(SHAW, q, k, v, [a], False, s, cfg)
    O3, L3 = orc.forward(SHAW, q, k, v, [np.zeros_like(a)], False, s, cfg)
    np.testing.assert_allclose(O2, O3, atol=1e-13)
    np.testing.assert_allclose(L2, L3 + s * np.einsum("bhld,hd->bhl", q, a_row), atol=1e-12)
    # DeBERTa c2p rows equal -> row-constant (Qr zero)
    Kr = np.repeat(rnd(rng, H, d)[:, None, :], 8, axis=1)
    O4, _ = orc.forward(DEBERTA, q, k, v, [Kr, np.zeros_like(Kr)], False, s, cfg)
    O5, _ = orc.forward(DEBERTA, q, k, v, [np.zeros_like(Kr), np.zeros_like(Kr)], False, s, cfg)
    np.testing.assert_allclose(O4, O5, atol=1e-13)
    # Transformer-XL: constant r -> (q_i + v) . r is row-constant
    for causal in (False, True):
        n_off = orc.table_rows(TXL, L, causal, cfg)
        r = np.repeat(rnd(rng, H, d)[:, None, :], n_off, axis=1)
        u, vv = rnd(rng, H, d), rnd(rng, H, d)
        O6, _ = orc.forward(TXL, q, k, v, [r, u, vv], causal, s)
        O7, _ = orc.forward(TXL, q, k, v, [np.zeros_like(r), u, vv], causal, s)
        np.testing.assert_allclose(O6, O7, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_query_side_table_grads_sum_to_zero(causal):
    L, d, H = 33, 8, 2
    cfg = RelCfg(shaw_clip=5, deberta_span=4)
    for mech in (T5, SHAW, TXL, DEBERTA):
        q, k, v, do, rel = make_case(mech, 2, H, L, d, causal, cfg, seed=21 + mech)
        _, _, _, drel = orc.backward(mech, q, k, v, rel, causal, do, 0.35, cfg)
        tot = drel[0].sum(axis=1)
        scale_ref = np.abs(drel[0]).sum(axis=1).max()
        assert scale_ref > 1e-3
        np.testing.assert_allclose(tot, 0.0, atol=1e-12 * max(1.0, scale_ref))


def test_batch_sums_table_grads():
    """Per-head tables are shared across the batch: their gradient with B = 2 is
    the sum of the two single-batch gradients."""
    cfg = RelCfg(shaw_clip=3, deberta_span=3)
    for mech in MECHS:
        q, k, v, do, rel = make_case(mech, 2, 2, 9, 4, False, cfg, seed=31)
        _, _, _, dr = orc.backward(mech, q, k, v, rel, False, do, 0.5, cfg)
        parts = [orc.backward(mech, q[b:b + 1], k[b:b + 1], v[b:b + 1], rel, False, do[b:b + 1], 0.5, cfg)[3] for b in range(2)]
        for n in range(len(rel)):
            np.testing.assert_allclose(dr[n], parts[0][n] + parts[1][n], rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------
# Transformer-XL with memory (keys: M cached positions, then the L of the segment)
# ----------------------------------------------------------------------------
def brute_txl_memory(q, k, v, rel, do, s):
    """Scalar loops: query i at absolute position M + i, keys j <= M + i,
    S_ij = s ((q_i + u).k_j + (q_i + v).r[M + i - j])."""
    r, u, vv = rel
    B, H, L, d = q.shape
    LK = k.shape[2]
    M = LK - L
    O = np.zeros_like(q)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    drel = [np.zeros_like(x) for x in rel]
    for b in range(B):
        for h in range(H):
            for i in range(L):
                a = M + i
                keys = list(range(a + 1))
                sc = [s * (dot(q[b, h, i] + u[h], k[b, h, j]) + dot(q[b, h, i] + vv[h], r[h][a - j])) for j in keys]
                mx = max(sc)
                z = sum(math.exp(x - mx) for x in sc)
                P = [math.exp(x - mx) / z for x in sc]
                O[b, h, i] = sum(pj * v[b, h, j] for pj, j in zip(P, keys))
                Di = dot(do[b, h, i], O[b, h, i])
                for pj, j in zip(P, keys):
                    dS = pj * (dot(do[b, h, i], v[b, h, j]) - Di)
                    dv[b, h, j] += pj * do[b, h, i]
                    dq[b, h, i] += s * dS * (k[b, h, j] + r[h][a - j])
                    dk[b, h, j] += s * dS * (q[b, h, i] + u[h])
                    drel[0][h][a - j] += s * dS * (q[b, h, i] + vv[h])
                    drel[1][h] += s * dS * k[b, h, j]
                    drel[2][h] += s * dS * r[h][a - j]
    return O, dq, dk, dv, drel


@pytest.mark.parametrize("M,L", [(0, 5), (3, 4), (6, 2), (5, 1)])
def test_txl_memory_vs_brute_force(M, L):
    rng = np.random.default_rng(M * 10 + L)
    d, H = 3, 2
    q, do = rnd(rng, 2, H, L, d), rnd(rng, 2, H, L, d)
    k, v = rnd(rng, 2, H, M + L, d), rnd(rng, 2, H, M + L, d)
    rel = [rnd(rng, H, M + L, d, std=0.5), rnd(rng, H, d, std=0.5), rnd(rng, H, d, std=0.5)]
    s = 0.43
    O, _ = orc.txl_memory_forward(q, k, v, rel, s)
    dq, dk, dv, drel = orc.txl_memory_backward(q, k, v, rel, do, s)
    bO, bdq, bdk, bdv, bdrel = brute_txl_memory(q, k, v, rel, do, s)
    for got, want in [(O, bO), (dq, bdq), (dk, bdk), (dv, bdv)] + list(zip(drel, bdrel)):
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_txl_memory_finite_differences():
    rng = np.random.default_rng(17)
    M, L, d, H = 4, 5, 3, 2
    q, do = rnd(rng, 1, H, L, d), rnd(rng, 1, H, L, d)
    k, v = rnd(rng, 1, H, M + L, d), rnd(rng, 1, H, M + L, d)
    rel = [rnd(rng, H, M + L, d, std=0.5), rnd(rng, H, d, std=0.5), rnd(rng, H, d, std=0.5)]
    s = 0.37
    dq, dk, dv, drel = orc.txl_memory_backward(q, k, v, rel, do, s)

    def loss(q_, k_, v_, rel_):
        return float(np.sum(orc.txl_memory_forward(q_, k_, v_, rel_, s)[0] * do))

    e = np.random.default_rng(2)
    for name, x, g in [("q", q, dq), ("k", k, dk), ("v", v, dv), ("r", rel[0], drel[0])]:
        dirn = e.standard_normal(x.shape)
        args = {"q": q, "k": k, "v": v, "r": rel[0]}
        plus, minus = dict(args), dict(args)
        plus[name] = x + 1e-6 * dirn
        minus[name] = x - 1e-6 * dirn
        fd = (loss(plus["q"], plus["k"], plus["v"], [plus["r"]] + rel[1:]) -
              loss(minus["q"], minus["k"], minus["v"], [minus["r"]] + rel[1:])) / 2e-6
        an = float(np.sum(g * dirn))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)
