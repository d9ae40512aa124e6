"""Pins for the oracle's backward through the scoring CNN (no GPU).

``cnn_backward`` writes the chain rule out layer by layer.  It is checked
against torch autograd through ``torch.nn.functional.conv1d`` (float64, the
same zero padding outside the sequence), for causal and centred taps, and
against central finite differences of the oracle's forward on a tiny case.
"""
import numpy as np
import pytest
import torch

from oracle import lte_oracle as O


def _case(seed, n, D, c1, k1, k2, past1, past2, std=0.7):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((n, D))
    v = rng.standard_normal((n, D))
    cnn = O.CNN(rng.standard_normal((c1, 2 * D, k1)) * std, rng.standard_normal(c1) * 0.3,
                rng.standard_normal((c1, k2)) * std, float(rng.standard_normal()) * 0.3, past1, past2)
    dr = rng.standard_normal(n)
    return k, v, cnn, dr


def _torch_forward(k, v, w1, b1, w2, b2, past1, past2):
    n = k.shape[0]
    x = torch.cat([k, v], dim=1).T[None]                       # [1, 2D, n]
    k1, k2 = w1.shape[2], w2.shape[1]
    xp = torch.nn.functional.pad(x, (past1, k1 - 1 - past1))   # zeros outside [0, n)
    u = torch.nn.functional.silu(torch.nn.functional.conv1d(xp, w1, b1))      # [1, C1, n]
    up = torch.nn.functional.pad(u, (past2, k2 - 1 - past2))
    z = torch.nn.functional.conv1d(up, w2[None], b2.reshape(1))[0, 0]
    return torch.sigmoid(z)


@pytest.mark.parametrize("cfg", [
    # n, D, c1, k1, k2, past1, past2, n_scored
    (40, 3, 4, 5, 3, 2, 1, 37),          # the paper's centred taps
    (33, 2, 3, 5, 3, 4, 2, 33),          # causal taps: every token scored
    (25, 4, 5, 3, 2, 0, 0, 22),          # future-only taps
    (12, 2, 2, 1, 1, 0, 0, 12),          # 1 x 1 kernels
])
def test_cnn_backward_vs_autograd(cfg):
    n, D, c1, k1, k2, past1, past2, n_scored = cfg
    k, v, cnn, dr = _case(sum(cfg), n, D, c1, k1, k2, past1, past2)
    got = O.cnn_backward(k, v, cnn, dr, n_scored)
    tk, tv = (torch.tensor(x, requires_grad=True) for x in (k, v))
    tw1, tb1, tw2 = (torch.tensor(np.asarray(x, np.float64), requires_grad=True)
                     for x in (cnn.w1, cnn.b1, cnn.w2))
    tb2 = torch.tensor(cnn.b2, dtype=torch.float64, requires_grad=True)
    r = _torch_forward(tk, tv, tw1, tb1, tw2, tb2, past1, past2)
    np.testing.assert_allclose(r.detach().numpy()[:n - cnn.future],
                               O.cnn_scores(k, v, cnn)[:n - cnn.future], atol=1e-13, rtol=0)
    (r[:n_scored] * torch.tensor(dr[:n_scored])).sum().backward()
    for g, t in zip(got, (tk, tv, tw1, tb1, tw2, tb2)):
        np.testing.assert_allclose(np.asarray(g), t.grad.numpy(), atol=1e-12, rtol=0)


def test_cnn_backward_vs_finite_differences():
    n, D, c1, k1, k2, past1, past2 = 9, 2, 2, 3, 3, 1, 1
    k, v, cnn, dr = _case(3, n, D, c1, k1, k2, past1, past2)
    n_scored = n - cnn.future
    dk, dv, dw1, db1, dw2, db2 = O.cnn_backward(k, v, cnn, dr, n_scored)

    def loss(k_, v_, w1_):
        c = O.CNN(w1_, cnn.b1, cnn.w2, cnn.b2, past1, past2)
        return float((O.cnn_scores(k_, v_, c)[:n_scored] * dr[:n_scored]).sum())

    h = 1e-6
    for which, g in ((0, dk), (1, dv), (2, dw1)):
        base = [k, v, np.asarray(cnn.w1, np.float64)][which]
        num = np.zeros_like(base)
        for i in np.ndindex(base.shape):
            args = [k, v, np.asarray(cnn.w1, np.float64)]
            xp, xm = base.copy(), base.copy()
            xp[i] += h
            xm[i] -= h
            args[which] = xp
            lp = loss(*args)
            args[which] = xm
            num[i] = (lp - loss(*args)) / (2 * h)
        np.testing.assert_allclose(g, num, atol=1e-7, rtol=0)
