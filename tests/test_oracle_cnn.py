"""Pins for the oracle's retention CNN (no GPU).

The oracle writes the two conv layers out as explicit tap sums; here they are
checked against torch.nn.functional.conv1d (a library routine with the same
cross-correlation definition) in float64, including causal variants, and
against a brute-force per-output triple loop on a tiny case.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import lte_oracle as O


def _torch_scores(k, v, w1, b1, w2, b2, past1, past2):
    x = torch.cat([k, v], dim=1).T[None]                      # [1, 2D, T]
    k1, k2 = w1.shape[2], w2.shape[1]
    x = F.pad(x, (past1, k1 - 1 - past1))
    u = F.silu(F.conv1d(x, w1, b1))                          # [1, C1, T]
    u = F.pad(u, (past2, k2 - 1 - past2))
    z = F.conv1d(u, w2[None], b2.reshape(1))
    return torch.sigmoid(z)[0, 0]


@pytest.mark.parametrize("past1,past2", [(2, 1), (4, 2), (0, 0), (1, 0)])
def test_cnn_matches_conv1d(past1, past2):
    g = torch.Generator().manual_seed(7)
    T, D, C1 = 40, 8, 6
    k = torch.randn(T, D, generator=g, dtype=torch.float64)
    v = torch.randn(T, D, generator=g, dtype=torch.float64)
    w1 = torch.randn(C1, 2 * D, 5, generator=g, dtype=torch.float64) * 0.3
    b1 = torch.randn(C1, generator=g, dtype=torch.float64) * 0.1
    w2 = torch.randn(C1, 3, generator=g, dtype=torch.float64) * 0.3
    b2 = torch.randn((), generator=g, dtype=torch.float64) * 0.1
    cnn = O.CNN(w1.numpy(), b1.numpy(), w2.numpy(), float(b2), past1, past2)
    r = O.cnn_scores(k.numpy(), v.numpy(), cnn)
    ref = _torch_scores(k, v, w1, b1, w2, b2, past1, past2).numpy()
    F_ = cnn.future
    assert F_ == (4 - past1) + (2 - past2)
    n_scored = T - F_
    assert np.all(np.isnan(r[n_scored:]))
    np.testing.assert_allclose(r[:n_scored], ref[:n_scored], rtol=0, atol=1e-13)


def test_cnn_bruteforce_tiny():
    """Triple loop over (c, ch, tap) for every output; independent of the
    oracle's shifted-matrix formulation."""
    rng = np.random.default_rng(3)
    T, D, C1 = 9, 2, 3
    k = rng.standard_normal((T, D)); v = rng.standard_normal((T, D))
    w1 = rng.standard_normal((C1, 2 * D, 5)); b1 = rng.standard_normal(C1)
    w2 = rng.standard_normal((C1, 3)); b2 = 0.25
    cnn = O.CNN(w1, b1, w2, b2, 2, 1)
    r = O.cnn_scores(k, v, cnn)

    def x(ch, j):
        if j < 0 or j >= T:
            return 0.0
        return k[j, ch] if ch < D else v[j, ch - D]

    def u(c, j):
        if j < 0 or j >= T:
            return 0.0
        z = b1[c]
        for ch in range(2 * D):
            for kk in range(5):
                z += w1[c, ch, kk] * x(ch, j + kk - 2)
        return z / (1 + math.exp(-z))

    for j in range(T - 3):
        z = b2
        for c in range(C1):
            for kk in range(3):
                z += w2[c, kk] * u(c, j + kk - 1)
        assert abs(r[j] - 1 / (1 + math.exp(-z))) < 1e-14


def test_cnn_depends_only_on_receptive_field():
    """r_j reads exactly [j-P, j+F]: perturbing a token outside it leaves r_j
    unchanged, perturbing one inside changes it."""
    rng = np.random.default_rng(5)
    T, D, C1 = 30, 4, 5
    k = rng.standard_normal((T, D)); v = rng.standard_normal((T, D))
    cnn = O.CNN(rng.standard_normal((C1, 2 * D, 5)) * 0.1, rng.standard_normal(C1) * 0.1,
                rng.standard_normal((C1, 3)) * 0.1, 0.1, 2, 1)
    r = O.cnn_scores(k, v, cnn)
    j = 12
    for pos, inside in [(j - 4, False), (j - 3, True), (j + 3, True), (j + 4, False)]:
        k2 = k.copy(); k2[pos] += 1.0
        r2 = O.cnn_scores(k2, v, cnn)
        assert (abs(r2[j] - r[j]) > 1e-12) == inside, pos
    # the v half of the input is read too
    v2 = v.copy(); v2[j + 3] += 1.0
    assert abs(O.cnn_scores(k, v2, cnn)[j] - r[j]) > 1e-12


def test_mask_and_sink():
    r = np.array([0.9, 0.9, 0.4, 0.5, 0.6, np.nan])
    m = O.retention_mask(r, sink=2, tau=0.5)
    assert m.tolist() == [0, 0, 0, 1, 1, 0]
    assert O.fed_mask(np.ones(5, np.uint8), 3).tolist() == [0, 0, 0, 1, 1]
