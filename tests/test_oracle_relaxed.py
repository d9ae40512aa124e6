"""Pins for the oracle's relaxed-retention attention (no GPU).

Reading (the pages give no gradient rule for the keep decision): the hard
attended sets stay as they are, and every retained-segment key j of row t
enters the softmax with weight r_j (its logit gains log r_j).  The oracle's
``prefill_relaxed_unit`` / ``prefill_relaxed_backward_unit`` are checked here
against computations that share none of their arithmetic:

* weight as multiplicity: with integer r_j, the relaxed row equals plain
  softmax attention (``attend``) over the key list in which retained key j
  appears r_j times;
* r = 1 reduces to the hard prefill (``prefill_unit``), and cap 0 leaves r
  with no gradient;
* torch autograd (float64) through a dense masked softmax whose bias matrix
  carries log r on the (row, key) pairs of the brute-force retained
  membership, for all three cap policies -- dq, dk, dv and dr;
* central finite differences of the relaxed forward in r.
"""
import math

import numpy as np
import pytest
import torch

from oracle import lte_oracle as O
from tests.test_oracle_sets import brute_member, brute_member_first, brute_member_lowest


def _case(seed, T, G, D, s, w, p_keep):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, G, D))
    k = rng.standard_normal((T, D))
    v = rng.standard_normal((T, D))
    do = rng.standard_normal((T, G, D))
    r = 0.3 + 0.7 * rng.random(T)                      # retention scores in (0.3, 1)
    m = (rng.random(T) < p_keep).astype(np.uint8)
    m[:s] = 0
    return q, k, v, do, r, m


def _retained_member(j, t, m, r, s, w, C, policy):
    """j in Ret_t by the brute-force membership rules (out of the window and
    the sink, and a survivor of the cap)."""
    if j < s or j > t - w:
        return False
    if policy == O.CAP_RECENT:
        return brute_member(j, t, m, s, w, C)
    if policy == O.CAP_FIRST:
        return brute_member_first(j, t, m, s, w, C)
    return brute_member_lowest(j, t, m, r, s, w, C)


def _member(j, t, m, r, s, w, C, policy):
    if j > t:
        return False
    return j < s or j > t - w or _retained_member(j, t, m, r, s, w, C, policy)


def test_integer_weight_is_multiplicity():
    """r_j = n_j (an integer) on a retained key = that key listed n_j times."""
    T, G, D, s, w, C = 40, 2, 6, 2, 5, 100
    q, k, v, _, _, m = _case(7, T, G, D, s, w, 0.5)
    rng = np.random.default_rng(8)
    r = rng.integers(1, 4, T).astype(np.float64)
    scale = 0.5
    o, lse = O.prefill_relaxed_unit(q[:, :, :], k, v, m, s, w, C, scale, r)
    for t in range(T):
        keys = []
        for j in range(t + 1):
            if _member(j, t, m, r, s, w, C, O.CAP_RECENT):
                reps = int(r[j]) if _retained_member(j, t, m, r, s, w, C, O.CAP_RECENT) else 1
                keys += [j] * reps
        o_ref, lse_ref = O.attend(q[t], k[keys], v[keys], scale)
        np.testing.assert_allclose(o[t], o_ref, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse[t], lse_ref, atol=1e-12, rtol=0)


def test_unit_weights_reduce_to_hard_attention():
    T, G, D, s, w, C = 50, 3, 4, 3, 6, 4
    q, k, v, do, _, m = _case(3, T, G, D, s, w, 0.6)
    ones = np.ones(T)
    o, lse = O.prefill_relaxed_unit(q, k, v, m, s, w, C, 0.7, ones)
    o_h, lse_h, _ = O.prefill_unit(q, k, v, m, s, w, C, 0.7)
    np.testing.assert_allclose(o, o_h, atol=1e-13, rtol=0)
    np.testing.assert_allclose(lse, lse_h, atol=1e-13, rtol=0)
    dq, dk, dv, _ = O.prefill_relaxed_backward_unit(q, k, v, m, s, w, C, 0.7, do, ones)
    hq, hk, hv = O.prefill_backward_unit(q, k, v, m, s, w, C, 0.7, do)
    for a, b in ((dq, hq), (dk, hk), (dv, hv)):
        np.testing.assert_allclose(a, b, atol=1e-12, rtol=0)


def test_cap_zero_gives_no_score_gradient():
    T, G, D, s, w = 30, 2, 4, 2, 4
    q, k, v, do, r, m = _case(5, T, G, D, s, w, 0.8)
    _, _, _, dr = O.prefill_relaxed_backward_unit(q, k, v, m, s, w, 0, 0.5, do, r)
    assert np.all(dr == 0.0)


def _autograd(q, k, v, do, r, m, s, w, C, scale, policy):
    T = k.shape[0]
    member = np.zeros((T, T), dtype=bool)
    retained = np.zeros((T, T), dtype=bool)
    for t in range(T):
        for j in range(T):
            member[t, j] = _member(j, t, m, r, s, w, C, policy)
            retained[t, j] = j <= t and _retained_member(j, t, m, r, s, w, C, policy)
    qt, kt, vt, rt = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                      for x in (q, k, v, r))
    logits = scale * torch.einsum("tgd,jd->tgj", qt, kt)
    bias = torch.where(torch.tensor(retained), torch.log(rt)[None, :], torch.zeros(T, T,
                                                                                   dtype=torch.float64))
    logits = (logits + bias[:, None, :]).masked_fill(~torch.tensor(member)[:, None, :],
                                                     float("-inf"))
    o = torch.einsum("tgj,jd->tgd", torch.softmax(logits, dim=-1), vt)
    (o * torch.tensor(do)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy(), rt.grad.numpy()


@pytest.mark.parametrize("policy", [O.CAP_RECENT, O.CAP_FIRST, O.CAP_LOWEST])
@pytest.mark.parametrize("seed", range(3))
def test_relaxed_backward_vs_autograd(seed, policy):
    rng = np.random.default_rng(2000 + seed)
    T = int(rng.integers(10, 60))
    s, w = int(rng.integers(0, 4)), int(rng.integers(1, 10))
    C = int(rng.choice([1, 3, 7, 100]))
    q, k, v, do, r, m = _case(seed, T, 2, 5, s, w, float(rng.choice([0.3, 0.7])))
    scale = 0.4
    dq, dk, dv, dr = O.prefill_relaxed_backward_unit(q, k, v, m, s, w, C, scale, do, r, policy)
    aq, ak, av, ar = _autograd(q, k, v, do, r, m, s, w, C, scale, policy)
    for a, b in ((dq, aq), (dk, ak), (dv, av), (dr, ar)):
        np.testing.assert_allclose(a, b, atol=1e-11, rtol=0)


def test_relaxed_score_gradient_vs_finite_differences():
    T, G, D, s, w, C = 36, 2, 4, 2, 5, 6
    q, k, v, do, r, m = _case(11, T, G, D, s, w, 0.6)
    scale = 0.6
    _, _, _, dr = O.prefill_relaxed_backward_unit(q, k, v, m, s, w, C, scale, do, r)

    def loss(rr):
        o, _ = O.prefill_relaxed_unit(q, k, v, m, s, w, C, scale, rr)
        return float((o * do).sum())

    eps = 1e-6
    for j in range(T):
        e = np.zeros(T)
        e[j] = eps
        num = (loss(r + e) - loss(r - e)) / (2 * eps)
        assert math.isclose(num, dr[j], rel_tol=1e-6, abs_tol=1e-8), (j, num, dr[j])
    assert np.abs(dr).max() > 1e-3                   # retained keys do receive a gradient


def test_relaxed_stored_output_equal_to_exact_is_a_no_op():
    T, G, D, s, w, C = 40, 2, 4, 2, 5, 6
    q, k, v, do, r, m = _case(13, T, G, D, s, w, 0.6)
    o, _ = O.prefill_relaxed_unit(q, k, v, m, s, w, C, 0.5, r)
    a = O.prefill_relaxed_backward_unit(q, k, v, m, s, w, C, 0.5, do, r, o_out=o)
    b = O.prefill_relaxed_backward_unit(q, k, v, m, s, w, C, 0.5, do, r)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, atol=1e-13, rtol=0)
