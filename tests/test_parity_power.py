"""The GPU parity cases for Shaw and DeBERTa can fail: CPU proof with the oracle alone.

The GPU parity tests draw the Shaw table a and the DeBERTa tables Kr, Qr at std 1.0
(``Workload.rel_std``), not at the workloads' 0.02.  At 0.02 the whole relative term
moves O, LSE and the content gradients by about the bf16 tolerance (2e-2), so a kernel
that gathered the wrong table row, or left a term out, could still pass.  Here the
oracle is run on the GPU tests' own shapes and seeds twice, once with the true tables
and once with tables that reproduce a plausible kernel mistake, and the two results
must differ by several tolerances in at least one compared output:

  * Shaw: the band gather one offset off (rows 1 .. 2c - 1 read their neighbour), the
    sign of the offset flipped (the table read mirrored), the term dropped;
  * DeBERTa: either term dropped (c2p: Kr = 0, p2c: Qr = 0), either gather one offset
    off, and the two tables swapped (the operands of c2p and p2c transposed).

The relative term is the article's B of "结构感知内核让相对位置注意力加速21倍" (section
"为什么相对位置注意力难做快", S = Q K^T / sqrt(d) + B); its forward and backward both
have to be checked (section "开发者落地建议", item 3).
"""
import numpy as np
import pytest
import torch

import oracle as orc
from attention_fwd_bwd_flashattention_b200.inputs import DEBERTA, SHAW, Workload, make_inputs, to_f64

from _parity import TOL, maxabs, oracle_cfg, rel_l2

O1_STD = 1.0  # the std the GPU parity cases draw the Shaw / DeBERTa tables at
MARGIN = 5.0  # a planted mistake must move some output by this many tolerances


def shaw_wl(clip, causal, L, std=O1_STD):
    return Workload("shaw_o1", SHAW, torch.bfloat16, causal, 2, 2, L, shaw_clip=clip, rel_std=std)


def deberta_wl(span, causal, L, std=O1_STD):
    return Workload("deb_o1", DEBERTA, torch.bfloat16, causal, 2, 2, L, deberta_span=span, rel_std=std)


def _run(wl, inp, rel):
    q, k, v, do = (to_f64(inp[n]) for n in ("q", "k", "v", "do"))
    cfg = oracle_cfg(wl)
    O, LSE = orc.forward(wl.mech, q, k, v, rel, wl.causal, wl.scale, cfg)
    dq, dk, dv, _ = orc.backward(wl.mech, q, k, v, rel, wl.causal, do, wl.scale, cfg)
    return O, LSE, dq, dk, dv


def _effect(a, b):
    """Largest change, in units of the bf16 tolerance, over the outputs the parity
    tests compare (max-abs on O and LSE, relative L2 on dQ, dK, dV)."""
    tol = TOL[torch.bfloat16]
    e = [maxabs(a[0], b[0]), maxabs(a[1], b[1]), rel_l2(a[2], b[2]), rel_l2(a[3], b[3]), rel_l2(a[4], b[4])]
    return max(e) / tol


def _shift_interior(t, rows):
    """Rows 1 .. rows - 2 read their upper neighbour (a gather one offset off inside the
    band; the clipped end rows unchanged)."""
    s = t.copy()
    s[:, 1:rows - 1] = t[:, 2:rows]
    return s


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("clip", [1, 7, 64, 100])
def test_shaw_mistakes_exceed_tolerance(clip, causal):
    L = 300
    wl = shaw_wl(clip, causal, L)
    inp = make_inputs(wl, seed=clip + L)  # the GPU case's seed
    rel = [to_f64(r) for r in inp["rel"]]
    base = _run(wl, inp, rel)
    a = rel[0]
    mistakes = {"mirror": a[:, ::-1].copy(), "drop": np.zeros_like(a)}
    if clip > 1:  # with c = 1 the band is the diagonal alone: its shift is checked by the mirror
        mistakes["shift"] = _shift_interior(a, 2 * clip + 1)
    for name, bad in mistakes.items():
        eff = _effect(_run(wl, inp, [bad]), base)
        assert eff > MARGIN, (clip, causal, name, eff)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("span", [32, 96, 256, 40])
def test_deberta_mistakes_exceed_tolerance(span, causal):
    L = 300
    wl = deberta_wl(span, causal, L)
    inp = make_inputs(wl, seed=span + L)  # the GPU case's seed
    Kr, Qr = (to_f64(r) for r in inp["rel"])
    base = _run(wl, inp, [Kr, Qr])
    mistakes = {
        "drop_c2p": [np.zeros_like(Kr), Qr],
        "drop_p2c": [Kr, np.zeros_like(Qr)],
        "shift_c2p": [_shift_interior(Kr, 2 * span), Qr],
        "shift_p2c": [Kr, _shift_interior(Qr, 2 * span)],
        "swap": [Qr, Kr],
    }
    for name, bad in mistakes.items():
        eff = _effect(_run(wl, inp, bad), base)
        assert eff > MARGIN, (span, causal, name, eff)


def test_workload_scale_is_too_small_to_discriminate():
    """Why the parity cases raise the scale: at the workloads' std 0.02 a Shaw gather
    one offset off moves no compared output by even one tolerance (c = 7, non-causal)."""
    wl = shaw_wl(7, False, 300, std=0.02)
    inp = make_inputs(wl, seed=307)
    rel = [to_f64(r) for r in inp["rel"]]
    eff = _effect(_run(wl, inp, [_shift_interior(rel[0], 15)]), _run(wl, inp, rel))
    assert eff < 1.0, eff
