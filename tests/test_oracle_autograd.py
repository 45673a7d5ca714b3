"""The oracle's hand-derived backward against torch.autograd (fp64, CPU).

Each mechanism's forward is restated here as a dense torch expression, with
S = s q k^T + B and B materialised from its definition:
* T5: a bucket per offset j - i (buckets from the pinned golden table's function);
* Shaw: q_i . a[clip(j - i) + c], plus, with the value table, sum_j P_ij aV[...];
* Transformer-XL: s((q_i + u) . k_j + (q_i + v) . r[row(i - j)]), with an optional
  memory of M keys before the segment;
* DeBERTa: s(q_i . Kr[clip(i - j + k)] + k_j . Qr[clip(j - i + k)]);
* ALiBi: -m_h |j - i|.
Autograd of sum(O * dO) then gives every gradient, which must match the oracle's
chain-rule backward to fp64 rounding. This pins the backward to ~1e-12, where the
finite differences of test_oracle_pins.py reach ~1e-6.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from oracle import ALIBI, DEBERTA, SHAW, T5, TXL, RelCfg

CFG = RelCfg(t5_num_buckets=8, t5_max_distance=12, t5_bidirectional=True, shaw_clip=3, deberta_span=4)


def _tables(mech, H, L, d, causal, cfg, rng):
    rows = orc.table_rows(mech, L, causal, cfg)
    if mech == ALIBI:
        return [0.05 + np.abs(rng.standard_normal(H)) * 0.3]
    if mech == T5:
        return [rng.standard_normal((H, rows)) * 0.5]
    if mech == SHAW:
        t = [rng.standard_normal((H, rows, d)) * 0.5]
        return t + [rng.standard_normal((H, rows, d)) * 0.5] if cfg.shaw_value else t
    if mech == TXL:
        return [rng.standard_normal((H, rows, d)) * 0.5, rng.standard_normal((H, d)) * 0.5,
                rng.standard_normal((H, d)) * 0.5]
    return [rng.standard_normal((H, rows, d)) * 0.5, rng.standard_normal((H, rows, d)) * 0.5]


def _gather_rows(x, idx):
    """x [B, H, Lq, R], idx [Lq, Lk] -> [B, H, Lq, Lk] with out[..., i, j] = x[..., i, idx[i, j]]."""
    B, H, Lq, _ = x.shape
    return torch.gather(x, 3, idx[None, None].expand(B, H, Lq, idx.shape[1]))


def torch_forward(mech, q, k, v, rel, causal, s, cfg, seqlens_k=None, mem=0):
    """O, LSE of the dense restatement; queries sit at positions mem .. mem + Lq - 1."""
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    i = torch.arange(Lq)[:, None] + mem
    j = torch.arange(Lk)[None, :]
    n = j - i  # j - i, [Lq, Lk]
    S = s * q @ k.transpose(-1, -2)
    if mech == ALIBI:
        S = S - rel[0][None, :, None, None] * n.abs().to(torch.float64)
    elif mech == T5:
        bkt = torch.from_numpy(orc.t5_bucket(n.numpy(), cfg.t5_num_buckets, cfg.t5_max_distance,
                                             cfg.t5_bidirectional)).long()
        S = S + rel[0][:, bkt][None]
    elif mech == SHAW:
        c = cfg.shaw_clip
        idx = n.clamp(-c, c) + c
        S = S + s * _gather_rows(torch.einsum("bhid,hrd->bhir", q, rel[0]), idx)
    elif mech == TXL:
        r, u, vb = rel
        row = (i - j) if causal else (i - j) + (Lk - 1)
        valid = (row >= 0) & (row < r.shape[1])
        qr = torch.einsum("bhid,hrd->bhir", q + vb[None, :, None, :], r)
        pos = torch.where(valid, _gather_rows(qr, row.clamp(0, r.shape[1] - 1)), torch.zeros((), dtype=q.dtype))
        uk = torch.einsum("bhjd,hd->bhj", k, u)
        S = S + s * (uk[:, :, None, :] + pos)
    else:
        Kr, Qr = rel
        kk = cfg.deberta_span
        c2p = _gather_rows(torch.einsum("bhid,hrd->bhir", q, Kr), (i - j + kk).clamp(0, 2 * kk - 1))
        kq = torch.einsum("bhjd,hrd->bhjr", k, Qr)  # [B, H, Lk, R]
        p2c = kq[:, :, j.expand(Lq, Lk), (j - i + kk).clamp(0, 2 * kk - 1)]
        S = S + s * (c2p + p2c)
    allowed = torch.ones(B, 1, Lq, Lk, dtype=torch.bool)
    if causal:
        allowed = allowed & (n <= 0)[None, None]
    if seqlens_k is not None:
        allowed = allowed & (j[None, None] < torch.tensor(seqlens_k)[:, None, None, None])
    S = S.masked_fill(~allowed, -float("inf"))
    P = torch.softmax(S, dim=-1)
    O = P @ v
    if mech == SHAW and cfg.shaw_value:
        c = cfg.shaw_clip
        aV = rel[1][:, n.clamp(-c, c) + c]  # [H, Lq, Lk, d]
        O = O + torch.einsum("bhij,hijd->bhid", P, aV)
    return O, torch.logsumexp(S, dim=-1)


def autograd_case(mech, q, k, v, rel, do, causal, s, cfg, seqlens_k=None, mem=0):
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    trel = [torch.tensor(np.asarray(x, dtype=np.float64), requires_grad=True) for x in rel]
    O, LSE = torch_forward(mech, tq, tk, tv, trel, causal, s, cfg, seqlens_k, mem)
    (O * torch.tensor(do)).sum().backward()
    return O.detach().numpy(), LSE.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy(), \
        [t.grad.numpy() for t in trel]


def assert_close(got, want, what):
    scale = max(1.0, float(np.abs(want).max()))
    err = float(np.abs(np.asarray(got) - want).max())
    assert err <= 1e-11 * scale, f"{what}: max |diff| {err:.3g}"


CASES = [(T5, CFG), (ALIBI, CFG), (SHAW, CFG), (SHAW, RelCfg(shaw_clip=3, shaw_value=True)), (TXL, CFG),
         (DEBERTA, CFG)]


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("mech,cfg", CASES, ids=["t5", "alibi", "shaw", "shaw_value", "txl", "deberta"])
def test_backward_matches_autograd(mech, cfg, causal):
    B, H, L, d = 2, 2, 19, 5
    rng = np.random.default_rng(31 + 7 * mech + causal)
    q, k, v, do = (rng.standard_normal((B, H, L, d)) for _ in range(4))
    rel = _tables(mech, H, L, d, causal, cfg, rng)
    s = 0.4
    O, LSE, dq, dk, dv, drel = autograd_case(mech, q, k, v, rel, do, causal, s, cfg)
    O2, LSE2 = orc.forward(mech, q, k, v, rel, causal, s, cfg)
    dq2, dk2, dv2, drel2 = orc.backward(mech, q, k, v, rel, causal, do, s, cfg)
    assert_close(O2, O, "O")
    assert_close(LSE2, LSE, "LSE")
    for name, got, want in [("dq", dq2, dq), ("dk", dk2, dk), ("dv", dv2, dv)]:
        assert_close(got, want, name)
    assert len(drel2) == len(drel)
    for t, (got, want) in enumerate(zip(drel2, drel)):
        assert_close(got, want, f"drel[{t}]")


@pytest.mark.parametrize("mech", [T5, SHAW, TXL, DEBERTA, ALIBI], ids=["t5", "shaw", "txl", "deberta", "alibi"])
def test_key_lengths_backward_matches_autograd(mech):
    B, H, L, d = 3, 2, 17, 4
    rng = np.random.default_rng(5 + mech)
    q, k, v, do = (rng.standard_normal((B, H, L, d)) for _ in range(4))
    rel = _tables(mech, H, L, d, False, CFG, rng)
    lens = [17, 9, 1]
    O, LSE, dq, dk, dv, drel = autograd_case(mech, q, k, v, rel, do, False, 0.3, CFG, seqlens_k=lens)
    O2, _ = orc.forward(mech, q, k, v, rel, False, 0.3, CFG, seqlens_k=lens)
    dq2, dk2, dv2, drel2 = orc.backward(mech, q, k, v, rel, False, do, 0.3, CFG, seqlens_k=lens)
    assert_close(O2, O, "O")
    for name, got, want in [("dq", dq2, dq), ("dk", dk2, dk), ("dv", dv2, dv)] + \
            [(f"drel[{t}]", a, b) for t, (a, b) in enumerate(zip(drel2, drel))]:
        assert_close(got, want, name)


@pytest.mark.parametrize("M,L", [(7, 11), (1, 5), (12, 3)])
def test_txl_memory_backward_matches_autograd(M, L):
    """Transformer-XL with memory: queries at positions M .. M + L - 1 over M + L keys,
    table row (M + i) - j; restated directly here (the oracle computes it by padding)."""
    B, H, d = 2, 2, 4
    rng = np.random.default_rng(100 + M + L)
    q, do = (rng.standard_normal((B, H, L, d)) for _ in range(2))
    k, v = (rng.standard_normal((B, H, M + L, d)) for _ in range(2))
    rel = [rng.standard_normal((H, M + L, d)) * 0.5, rng.standard_normal((H, d)) * 0.5,
           rng.standard_normal((H, d)) * 0.5]
    s = 0.45
    O, LSE, dq, dk, dv, drel = autograd_case(TXL, q, k, v, rel, do, True, s, RelCfg(), mem=M)
    O2, LSE2 = orc.txl_memory_forward(q, k, v, rel, s)
    dq2, dk2, dv2, drel2 = orc.txl_memory_backward(q, k, v, rel, do, s)
    assert_close(O2, O, "O")
    assert_close(LSE2, LSE, "LSE")
    for name, got, want in [("dq", dq2, dq), ("dk", dk2, dk), ("dv", dv2, dv)] + \
            [(f"drel[{t}]", a, b) for t, (a, b) in enumerate(zip(drel2, drel))]:
        assert_close(got, want, name)
