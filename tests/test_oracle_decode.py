"""Pins for the oracle's decode cache simulation (no GPU).

The simulation holds the inference cache slot by slot (window ring, sink
slots, retained ring under each cap policy, scores computed from the
window in deferred batches).  It is an independent formulation of the prefill set formula, so
the two are checked against each other: every decode output equals the
prefill row of the concatenated sequence, for several scoring batch sizes.
"""
import math

import numpy as np
import pytest

from oracle import lte_oracle as O


def _setup(seed, T=90, D=6, G=2, C1=4):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, G, D)) * 2
    k = rng.standard_normal((T, D))
    v = rng.standard_normal((T, D))
    cnn = O.CNN(rng.standard_normal((C1, 2 * D, 5)) * 0.6, rng.standard_normal(C1) * 0.1,
                rng.standard_normal((C1, 3)) * 0.6, 0.0, 2, 1)
    return q, k, v, cnn


@pytest.mark.parametrize("seed,s,w,C,T0", [(0, 2, 12, 4, 20), (1, 4, 16, 3, 8),
                                          (2, 0, 9, 5, 30), (3, 3, 10, 0, 15),
                                          (4, 2, 7, 100, 1)])
@pytest.mark.parametrize("score_batch", [1, 3])
@pytest.mark.parametrize("policy", [O.CAP_RECENT, O.CAP_FIRST, O.CAP_LOWEST])
def test_decode_equals_prefill(seed, s, w, C, T0, score_batch, policy):
    q, k, v, cnn = _setup(seed)
    T = k.shape[0]
    tau = 0.5
    scale = 1 / math.sqrt(k.shape[1])
    if w - cnn.past - cnn.future < score_batch:
        pytest.skip("batch larger than the window allows")
    o_d, lse_d, sets, rets, _ = O.decode_unit(q, k, v, T0, s, w, C, tau, cnn, score_batch, scale,
                                              policy=policy)
    r = O.cnn_scores(k, v, cnn)
    m = O.retention_mask(r, s, tau)
    o_p, lse_p, _ = O.prefill_unit(q, k, v, m, s, w, C, scale, policy=policy, r=r)
    for i, t in enumerate(range(T0, T)):
        assert sets[i] == O.attended_set(t, m, s, w, C, policy, r), t
        np.testing.assert_allclose(o_d[i], o_p[t], atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse_d[i], lse_p[t], atol=1e-12, rtol=0)
        ret = [j for j in O.attended_set(t, m, s, w, C, policy, r) if s <= j <= t - w]
        assert rets[i] == ret


def test_scoring_batch_invariance():
    q, k, v, cnn = _setup(9, T=120)
    s, w, C, tau = 4, 20, 6, 0.5
    outs = []
    for D_s in (1, 7, 13):
        o, _, sets, rets, cache = O.decode_unit(q, k, v, 40, s, w, C, tau, cnn, D_s, 0.3)
        outs.append((o, sets, rets))
    for o, sets, rets in outs[1:]:
        np.testing.assert_array_equal(o, outs[0][0])
        assert sets == outs[0][1] and rets == outs[0][2]


@pytest.mark.parametrize("policy", [O.CAP_RECENT, O.CAP_FIRST, O.CAP_LOWEST])
def test_cache_after_prompt_matches_simulation(policy):
    q, k, v, cnn = _setup(5, T=70)
    s, w, C, tau = 3, 11, 4, 0.5
    r = O.cnn_scores(k, v, cnn)
    m = O.retention_mask(r, s, tau)
    for T0 in (1, 5, 11, 12, 20, 47, 70):
        *_, cache = O.decode_unit(q[:T0], k[:T0], v[:T0], T0, s, w, C, tau, cnn, 1, 0.3,
                                  policy=policy)
        st = O.cache_after_prompt(k, v, m, T0, s, w, C, policy, r)
        np.testing.assert_array_equal(st["win_pos"], cache.win_pos)
        np.testing.assert_array_equal(st["sink_pos"], cache.sink_pos)
        if policy == O.CAP_LOWEST:      # replacements land in the dropped token's slot
            assert sorted(st["ret_pos"]) == sorted(cache.ret_pos)
        else:
            np.testing.assert_array_equal(st["ret_pos"], cache.ret_pos)
        assert st["ret_total"] == cache.ret_total


def test_fed_mask_decode():
    rng = np.random.default_rng(1)
    T, D = 60, 4
    q = rng.standard_normal((T, 1, D)); k = rng.standard_normal((T, D)); v = rng.standard_normal((T, D))
    m = O.fed_mask((rng.random(T) < 0.5).astype(np.uint8), 2)
    o_d, _, sets, _, _ = O.decode_unit(q, k, v, 10, 2, 8, 3, 0.5, None, 1, 0.5, fed=m)
    for i, t in enumerate(range(10, T)):
        assert sets[i] == O.attended_set(t, m, 2, 8, 3)
