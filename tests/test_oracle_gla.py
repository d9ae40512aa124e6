"""Pins for the gated linear-attention oracle (no GPU).

The oracle runs the state recurrence token by token.  Here it is checked
against the unrolled closed form o_t = sum_{j<=t} v_j ((k_j * prod_{i=j+1..t} a_i) . q_t)
built from explicit cumulative products, and against plain causal linear
attention tril(Q K^T) V when every gate is 1.
"""
import numpy as np

from oracle import gla_oracle as GO


def test_unrolled_closed_form():
    rng = np.random.default_rng(0)
    T, dk, dv = 23, 5, 4
    q = rng.standard_normal((T, dk)); k = rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv)); a = rng.uniform(0.3, 1.0, (T, dk))
    o, S = GO.gla_recurrent(q, k, v, a)
    ref = np.zeros((T, dv))
    for t in range(T):
        for j in range(t + 1):
            decay = np.prod(a[j + 1:t + 1], axis=0) if j < t else np.ones(dk)
            ref[t] += v[j] * np.dot(k[j] * decay, q[t])
    np.testing.assert_allclose(o, ref, atol=1e-12, rtol=0)
    S_ref = sum(np.outer(v[j], k[j] * np.prod(a[j + 1:], axis=0)) for j in range(T))
    np.testing.assert_allclose(S, S_ref, atol=1e-12, rtol=0)


def test_unit_gates_is_causal_linear_attention():
    rng = np.random.default_rng(1)
    T, dk, dv = 17, 6, 3
    q = rng.standard_normal((T, dk)); k = rng.standard_normal((T, dk)); v = rng.standard_normal((T, dv))
    o, _ = GO.gla_recurrent(q, k, v, np.ones((T, dk)))
    np.testing.assert_allclose(o, np.tril(q @ k.T) @ v, atol=1e-12, rtol=0)


def test_batched_and_initial_state():
    rng = np.random.default_rng(2)
    B, T, H, dk, dv = 2, 9, 2, 3, 3
    q, k, a = (rng.standard_normal((B, T, H, dk)) for _ in range(3))
    a = 1 / (1 + np.exp(-a))
    v = rng.standard_normal((B, T, H, dv))
    o, S = GO.gla(q, k, v, a)
    # splitting the sequence and carrying the state gives the same result
    o1, S1 = GO.gla(q[:, :4], k[:, :4], v[:, :4], a[:, :4])
    o2, S2 = GO.gla(q[:, 4:], k[:, 4:], v[:, 4:], a[:, 4:], S0=S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], 1), o, atol=1e-12)
    np.testing.assert_allclose(S2, S, atol=1e-12)
