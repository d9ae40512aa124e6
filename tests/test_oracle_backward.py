"""Pins for the oracle's backward of the prefill attention (no GPU).

``prefill_backward_unit`` writes the softmax-attention gradients out by hand
for fixed attended sets.  Here it is checked against two computations that
share none of that arithmetic:

* torch autograd (float64, CPU) through a dense masked softmax whose mask is
  the attended-set membership, for all three cap policies;
* central finite differences of the oracle's forward (``prefill_unit``), on
  tiny inputs.
"""
import numpy as np
import pytest
import torch

from oracle import lte_oracle as O


def _case(seed, T, G, D, s, w, C, p_keep):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, G, D))
    k = rng.standard_normal((T, D))
    v = rng.standard_normal((T, D))
    do = rng.standard_normal((T, G, D))
    r = rng.integers(0, 6, T) / 6.0                    # frequent equal scores
    m = O.retention_mask(r, s, 1.0 - p_keep)
    return q, k, v, do, r, m


def _autograd(q, k, v, do, m, s, w, C, scale, policy, r):
    T = k.shape[0]
    member = np.zeros((T, T), dtype=bool)
    for t in range(T):
        member[t, O.attended_set(t, m, s, w, C, policy, r)] = True
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    logits = scale * torch.einsum("tgd,jd->tgj", qt, kt)
    logits = logits.masked_fill(~torch.tensor(member)[:, None, :], float("-inf"))
    o = torch.einsum("tgj,jd->tgd", torch.softmax(logits, dim=-1), vt)
    (o * torch.tensor(do)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("policy", [O.CAP_RECENT, O.CAP_FIRST, O.CAP_LOWEST])
@pytest.mark.parametrize("seed", range(4))
def test_backward_vs_autograd(seed, policy):
    rng = np.random.default_rng(1000 + seed)
    T = int(rng.integers(2, 60))
    s, w = int(rng.integers(0, 4)), int(rng.integers(1, 12))
    C = int(rng.choice([0, 1, 3, 7, 100]))
    q, k, v, do, r, m = _case(seed, T, 2, 5, s, w, C, float(rng.choice([0.3, 0.7])))
    scale = 0.4
    dq, dk, dv = O.prefill_backward_unit(q, k, v, m, s, w, C, scale, do, policy, r)
    aq, ak, av = _autograd(q, k, v, do, m, s, w, C, scale, policy, r)
    np.testing.assert_allclose(dq, aq, atol=1e-11, rtol=0)
    np.testing.assert_allclose(dk, ak, atol=1e-11, rtol=0)
    np.testing.assert_allclose(dv, av, atol=1e-11, rtol=0)


def test_backward_vs_finite_differences():
    """dL/dx for every entry of q, k and v, L = sum <do, o>, by central
    differences of the oracle's forward."""
    T, G, D, s, w, C, scale = 14, 2, 3, 2, 4, 2, 0.7
    q, k, v, do, r, m = _case(7, T, G, D, s, w, C, 0.6)
    dq, dk, dv = O.prefill_backward_unit(q, k, v, m, s, w, C, scale, do)

    def loss(q_, k_, v_):
        o, _, _ = O.prefill_unit(q_, k_, v_, m, s, w, C, scale)
        return float((o * do).sum())

    h = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for i in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[i] += h
            xm[i] -= h
            args = [q, k, v]
            idx = 0 if x is q else (1 if x is k else 2)
            args[idx] = xp
            lp = loss(*args)
            args[idx] = xm
            num[i] = (lp - loss(*args)) / (2 * h)
        np.testing.assert_allclose(g, num, atol=1e-7, rtol=0)


def test_backward_full_window_is_causal_attention():
    """w >= T: the sets are the causal prefix; the gradients are those of
    torch's causal SDPA (autograd, float64)."""
    T, G, D = 30, 3, 8
    q, k, v, do, r, m = _case(3, T, G, D, 2, T, 5, 0.5)
    scale = 1 / np.sqrt(D)
    dq, dk, dv = O.prefill_backward_unit(q, k, v, m, 2, T, 5, scale, do)
    qt = torch.tensor(q.transpose(1, 0, 2), requires_grad=True)            # [G, T, D]
    kt = torch.tensor(k[None].repeat(G, 0), requires_grad=True)
    vt = torch.tensor(v[None].repeat(G, 0), requires_grad=True)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    (o * torch.tensor(do.transpose(1, 0, 2))).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy().transpose(1, 0, 2), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dk, kt.grad.numpy().sum(0), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dv, vt.grad.numpy().sum(0), atol=1e-11, rtol=0)


def test_batched_backward_splits_heads():
    """The batch wrapper gives each KV head the sum over its query heads (GQA)
    and equals the per-unit function unit by unit."""
    rng = np.random.default_rng(11)
    B, T, Hq, Hkv, D, s, w, C = 2, 20, 4, 2, 3, 1, 5, 3
    q = rng.standard_normal((B, T, Hq, D))
    do = rng.standard_normal((B, T, Hq, D))
    k = rng.standard_normal((B, T, Hkv, D))
    v = rng.standard_normal((B, T, Hkv, D))
    masks = (rng.random((B, Hkv, T)) < 0.5).astype(np.uint8)
    dq, dk, dv = O.prefill_backward(q, k, v, masks, s, w, C, do, 0.5)
    for b in range(B):
        for h in range(Hkv):
            gq, gk, gv = O.prefill_backward_unit(q[b, :, 2 * h:2 * h + 2], k[b, :, h], v[b, :, h],
                                                 masks[b, h], s, w, C, 0.5,
                                                 do[b, :, 2 * h:2 * h + 2])
            np.testing.assert_array_equal(dq[b, :, 2 * h:2 * h + 2], gq)
            np.testing.assert_array_equal(dk[b, :, h], gk)
            np.testing.assert_array_equal(dv[b, :, h], gv)


def test_stored_output_for_delta_vs_autograd():
    """With o_out (the forward output as stored, here rounded to bf16) the
    backward uses D_t = <do_t, o_out_t>.  That is the exact gradient of
    L + sum_t c_t lse_t with the constants c_t = <do_t, o_t - o_out_t> (the
    lse term adds c_t P to the logits' gradient): checked with torch autograd
    for dq, dk and dv, and o_out = o reproduces the plain backward."""
    T, G, D, s, w, C = 48, 2, 8, 2, 7, 5
    q, k, v, do, r, m = _case(21, T, G, D, s, w, C, 0.5)
    scale = 0.45
    o, _, _ = O.prefill_unit(q, k, v, m, s, w, C, scale)
    o_st = torch.tensor(o).to(torch.bfloat16).double().numpy()
    dq, dk, dv = O.prefill_backward_unit(q, k, v, m, s, w, C, scale, do, o_out=o_st)
    member = np.zeros((T, T), dtype=bool)
    for t in range(T):
        member[t, O.attended_set(t, m, s, w, C)] = True
    c = torch.tensor((do * (o - o_st)).sum(-1))                  # [T, G], constants
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    logits = (scale * torch.einsum("tgd,jd->tgj", qt, kt)).masked_fill(
        ~torch.tensor(member)[:, None, :], float("-inf"))
    ot = torch.einsum("tgj,jd->tgd", torch.softmax(logits, dim=-1), vt)
    loss = (ot * torch.tensor(do)).sum() + (c * torch.logsumexp(logits, dim=-1)).sum()
    loss.backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-11, rtol=0)
    assert np.abs(dq - O.prefill_backward_unit(q, k, v, m, s, w, C, scale, do)[0]).max() > 0
    same = O.prefill_backward_unit(q, k, v, m, s, w, C, scale, do, o_out=o)
    for a, b in zip(same, O.prefill_backward_unit(q, k, v, m, s, w, C, scale, do)):
        np.testing.assert_allclose(a, b, atol=1e-13, rtol=0)
