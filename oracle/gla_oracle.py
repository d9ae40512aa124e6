"""Plain CPU oracle for the gated linear-attention layer of the laLTE hybrid.

TEST INFRASTRUCTURE ONLY (same rules as ``oracle/lte_oracle.py``: only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
use it; the GPU library shares no code with it).

Source: "Sparse Linear Attention: Viewing SWA from the Perspective of Linear
Attention", section "Background: Linear attention" (the state equation):
the state S_t (d_v x d_k) is decayed by A_t, then the outer product of the
value and key is added, and the output is the state read by the query.
The hybrid that interleaves this layer with LTE is the one of "Alleviating
Forgetfulness of Linear Attention by Hybrid Sparse Attention and
Contextualized Learnable Token Eviction" (TL;DR, Abstract).

Reading: A_t = diag(a_t) with a_t in (0, 1)^{d_k} (a gated/diagonal decay
acting on the key dimension), S_0 = 0, float64 throughout.
"""
from __future__ import annotations

import numpy as np


def gla_recurrent(q, k, v, a, S0=None):
    """Token-by-token recurrence for one (batch element, head).

    q, k [T, dk], v [T, dv], a [T, dk].
    S_t = S_{t-1} diag(a_t) + v_t k_t^T ;  o_t = S_t q_t.
    Returns (o [T, dv], S_T [dv, dk]).
    """
    q, k, v, a = (np.asarray(x, dtype=np.float64) for x in (q, k, v, a))
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    for t in range(T):
        S = S * a[t][None, :] + np.outer(v[t], k[t])
        o[t] = S @ q[t]
    return o, S


def gla(q, k, v, a, S0=None):
    """Batched recurrence: q, k, a [B, T, H, dk], v [B, T, H, dv].
    Returns o [B, T, H, dv] and final states [B, H, dv, dk]."""
    B, T, H, dk = np.shape(q)
    dv = np.shape(v)[3]
    o = np.zeros((B, T, H, dv))
    S = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            s0 = None if S0 is None else S0[b, h]
            o[b, :, h], S[b, h] = gla_recurrent(q[b, :, h], k[b, :, h], v[b, :, h],
                                                a[b, :, h], s0)
    return o, S
