"""The identity behind Shaw's wide-clip route, checked with the oracle alone.

Shaw's key-side term s q_i . a[clip(j - i, -c, c) + c] is the Transformer-XL term
s (q_i + v) . r_{i-j} with v = 0 for the table with one row per offset,
r[rho] = a[clip(off - rho, -c, c) + c] (rho = i - j + off, off = 0 causal, L - 1
otherwise), and u = 0 removes Transformer-XL's content bias.  So both mechanisms give
the same O, LSE, dQ, dK and dV, and the gradient of a row of a is the sum of the
expanded table's gradient over the offsets that row stands for.  The tensor-core
library runs Shaw with c > 64 this way; this test pins the identity and the two index
maps (expansion, summation) in plain NumPy, independent of the CUDA code.
"""
import numpy as np
import pytest

import oracle as orc


def expand(a, L, causal, c):
    off = 0 if causal else L - 1
    rows = L if causal else 2 * L - 1
    rho = np.arange(rows)
    return a[:, np.clip(off - rho, -c, c) + c, :]


def collapse(dr, L, causal, c):
    off = 0 if causal else L - 1
    rows = dr.shape[1]
    da = np.zeros((dr.shape[0], 2 * c + 1, dr.shape[2]))
    for rho in range(rows):
        da[:, int(np.clip(off - rho, -c, c)) + c, :] += dr[:, rho, :]
    return da


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("c", [1, 5, 30, 70])  # 30 and 70 reach past L - 1 = 22
def test_shaw_equals_txl_on_the_expanded_table(c, causal):
    rng = np.random.default_rng(c + 7 * causal)
    B, H, L, d = 2, 2, 23, 8
    q, k, v, dO = (rng.standard_normal((B, H, L, d)) for _ in range(4))
    a = rng.standard_normal((H, 2 * c + 1, d))
    scale = 0.4
    zero = np.zeros((H, d))
    r = expand(a, L, causal, c)
    Os, Ls = orc.forward(orc.SHAW, q, k, v, [a], causal, scale, orc.RelCfg(shaw_clip=c))
    Ot, Lt = orc.forward(orc.TXL, q, k, v, [r, zero, zero], causal, scale, orc.RelCfg())
    np.testing.assert_allclose(Os, Ot, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Ls, Lt, rtol=0, atol=1e-12)
    dqs, dks, dvs, (da,) = orc.backward(orc.SHAW, q, k, v, [a], causal, dO, scale, orc.RelCfg(shaw_clip=c))
    dqt, dkt, dvt, (dr, du, dv_bias) = orc.backward(orc.TXL, q, k, v, [r, zero, zero], causal, dO, scale, orc.RelCfg())
    for x, y in ((dqs, dqt), (dks, dkt), (dvs, dvt)):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-12)
    np.testing.assert_allclose(da, collapse(dr, L, causal, c), rtol=0, atol=1e-12)
    # causal: only j - i <= 0 occurs, so the rows of positive offsets get no gradient
    if causal:
        assert np.all(da[:, c + 1:, :] == 0)
