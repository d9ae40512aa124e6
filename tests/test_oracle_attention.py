"""Pins for the oracle's sparse attention (no GPU).

Special cases reduce to textbook causal attention, checked against
torch.nn.functional.scaled_dot_product_attention in float64; the general
case is checked against the same library routine given an explicit boolean
mask built from the brute-force membership rule; lse against logsumexp.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import lte_oracle as O
from tests.test_oracle_sets import brute_member


def _rand(B, T, Hq, Hkv, D, seed, qscale=1.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, T, Hq, D, generator=g, dtype=torch.float64) * qscale
    k = torch.randn(B, T, Hkv, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, T, Hkv, D, generator=g, dtype=torch.float64)
    return q, k, v


def _sdpa(q, k, v, allowed, scale):
    """allowed [B,Hkv,T,T] bool; GQA by repeating KV heads."""
    B, T, Hq, D = q.shape
    G = Hq // k.shape[2]
    qh = q.permute(0, 2, 1, 3)
    kh = k.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    vh = v.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    am = allowed.repeat_interleave(G, dim=1)
    o = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=am, scale=scale)
    logits = (qh @ kh.transpose(-1, -2)) * scale
    lse = torch.logsumexp(logits.masked_fill(~am, -math.inf), dim=-1)
    return o.permute(0, 2, 1, 3).numpy(), lse.numpy()


@pytest.mark.parametrize("case", ["window_covers_all", "retain_all"])
def test_reduces_to_causal_sdpa(case):
    B, T, Hq, Hkv, D, s = 2, 37, 4, 2, 8, 3
    q, k, v = _rand(B, T, Hq, Hkv, D, 1)
    rng = np.random.default_rng(0)
    if case == "window_covers_all":
        w, C = T, 5
        masks = (rng.random((B, Hkv, T)) < 0.5).astype(np.uint8)
    else:
        w, C = 6, T
        masks = np.ones((B, Hkv, T), np.uint8)
    masks = np.stack([[O.fed_mask(masks[b, h], s) for h in range(Hkv)] for b in range(B)])
    scale = 1 / math.sqrt(D)
    o, lse, count = O.prefill(q.numpy(), k.numpy(), v.numpy(), masks, s, w, C, scale)
    ref = F.scaled_dot_product_attention(
        q.permute(0, 2, 1, 3), k.permute(0, 2, 1, 3).repeat_interleave(2, 1),
        v.permute(0, 2, 1, 3).repeat_interleave(2, 1), is_causal=True, scale=scale)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), atol=1e-12, rtol=0)
    np.testing.assert_array_equal(count, np.broadcast_to(np.arange(1, T + 1), count.shape))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_general_vs_masked_sdpa(seed):
    rng = np.random.default_rng(seed)
    B, T, Hq, Hkv, D = 1, 45, 6, 3, 16
    s, w, C = int(rng.integers(0, 4)), int(rng.integers(2, 12)), int(rng.integers(0, 6))
    q, k, v = _rand(B, T, Hq, Hkv, D, seed, qscale=3.0)   # peaked softmax
    masks = np.stack([[O.fed_mask((rng.random(T) < 0.4).astype(np.uint8), s)
                       for _ in range(Hkv)] for _ in range(B)])
    scale = 1 / math.sqrt(D)
    o, lse, count = O.prefill(q.numpy(), k.numpy(), v.numpy(), masks, s, w, C, scale)
    allowed = torch.zeros(B, Hkv, T, T, dtype=torch.bool)
    for b in range(B):
        for h in range(Hkv):
            for t in range(T):
                for j in range(T):
                    allowed[b, h, t, j] = brute_member(j, t, masks[b, h], s, w, C)
    ro, rl = _sdpa(q, k, v, allowed, scale)
    np.testing.assert_allclose(o, ro, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, rl, atol=1e-12, rtol=0)
    np.testing.assert_array_equal(count, allowed.sum(-1).numpy())


def test_attend_extreme_logits():
    """Max subtraction keeps huge logits finite; one dominant key wins."""
    q = np.array([[1000.0, 0.0]])
    K = np.array([[1.0, 0.0], [0.0, 1.0], [-1.0, 0.0]])
    V = np.array([[1.0], [2.0], [3.0]])
    o, lse = O.attend(q, K, V, 1.0)
    assert abs(o[0, 0] - 1.0) < 1e-12 and abs(lse[0] - 1000.0) < 1e-9
