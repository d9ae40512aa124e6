"""Pins for the oracle's eviction, compaction and attended sets (no GPU).

The oracle states S_t as a union of sink, window and the C most recent
retained tokens.  Here it is checked against a differently phrased
membership rule (a token j <= t-w survives iff fewer than C retained tokens
left the window after it), against closed forms for the degenerate settings,
and against numpy's cumsum for the prefix counts.
"""
import json
import os

import numpy as np
import pytest

from oracle import lte_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def brute_member(j, t, m, s, w, C):
    if j > t or j < 0:
        return False
    if j < s or j > t - w:
        return True
    if not m[j]:
        return False
    newer = sum(1 for i in range(j + 1, t - w + 1) if i >= s and m[i])
    return newer < C


def brute_member_first(j, t, m, s, w, C):
    """Policy "first": a retained token that left the window survives iff
    fewer than C retained tokens left the window before it."""
    if j > t or j < 0:
        return False
    if j < s or j > t - w:
        return True
    if not m[j]:
        return False
    older = sum(1 for i in range(s, j) if m[i])
    return older < C


def brute_member_lowest(j, t, m, r, s, w, C):
    """Policy "lowest": a retained token that left the window survives iff
    fewer than C of the retained tokens that left the window by row t beat
    it (a higher score, or an equal score and a later position)."""
    if j > t or j < 0:
        return False
    if j < s or j > t - w:
        return True
    if not m[j]:
        return False
    better = sum(1 for i in range(s, t - w + 1)
                 if m[i] and i != j and (r[i] > r[j] or (r[i] == r[j] and i > j)))
    return better < C


def arrivals_lowest(order, r, C):
    """The segment after the tokens of `order` arrive one at a time: each is
    appended and, past C entries, the entry with the lowest (score, position)
    is removed (which may be the newcomer)."""
    held = []
    for j in order:
        held.append(j)
        if len(held) > C:
            held.remove(min(held, key=lambda i: (r[i], i)))
    return sorted(held)


@pytest.mark.parametrize("seed", range(6))
def test_attended_set_vs_bruteforce(seed):
    rng = np.random.default_rng(seed)
    for _ in range(25):
        T = int(rng.integers(1, 48))
        s = int(rng.integers(0, 5))
        w = int(rng.integers(1, 14))
        C = int(rng.choice([0, 1, 2, 3, 8, 100]))
        p = float(rng.choice([0.0, 0.3, 0.7, 1.0]))
        m = O.fed_mask((rng.random(T) < p).astype(np.uint8), s)
        for t in range(T):
            S = O.attended_set(t, m, s, w, C)
            ref = [j for j in range(T) if brute_member(j, t, m, s, w, C)]
            assert S == ref, (T, s, w, C, t)


@pytest.mark.parametrize("seed", range(4))
def test_attended_set_first_policy_vs_bruteforce(seed):
    rng = np.random.default_rng(100 + seed)
    for _ in range(25):
        T = int(rng.integers(1, 48))
        s = int(rng.integers(0, 5))
        w = int(rng.integers(1, 14))
        C = int(rng.choice([0, 1, 2, 3, 8, 100]))
        p = float(rng.choice([0.0, 0.3, 0.7, 1.0]))
        m = O.fed_mask((rng.random(T) < p).astype(np.uint8), s)
        for t in range(T):
            S = O.attended_set(t, m, s, w, C, O.CAP_FIRST)
            ref = [j for j in range(T) if brute_member_first(j, t, m, s, w, C)]
            assert S == ref, (T, s, w, C, t)
            if C >= T:                       # the cap never binds: both policies agree
                assert S == O.attended_set(t, m, s, w, C, O.CAP_RECENT)


def test_first_policy_closed_forms():
    """r == 1: the first C tokens past the sink stay for good; the count
    formula min(C, cnt[t-w]) is the same as for the most recent C."""
    T, s, w, C = 120, 3, 10, 7
    ones = O.fed_mask(np.ones(T, np.uint8), s)
    _, _, cnt = O.compact(ones)
    for t in range(T):
        S = O.attended_set(t, ones, s, w, C, O.CAP_FIRST)
        n = cnt[t - w] if t - w >= 0 else 0
        ret = [j for j in S if s <= j <= t - w]
        assert ret == list(range(s, s + min(C, n)))
        assert len(S) == min(t + 1, w) + len([j for j in range(s) if j <= t - w]) + min(C, n)


@pytest.mark.parametrize("seed", range(4))
def test_attended_set_lowest_policy_vs_bruteforce(seed):
    """Scores drawn from a few levels, so that equal scores occur often."""
    rng = np.random.default_rng(200 + seed)
    for _ in range(25):
        T = int(rng.integers(1, 48))
        s = int(rng.integers(0, 5))
        w = int(rng.integers(1, 14))
        C = int(rng.choice([0, 1, 2, 3, 8, 100]))
        r = rng.integers(0, 5, T) / 4.0
        m = O.retention_mask(r, s, float(rng.choice([0.0, 0.25, 0.5])))
        for t in range(T):
            S = O.attended_set(t, m, s, w, C, O.CAP_LOWEST, r)
            ref = [j for j in range(T) if brute_member_lowest(j, t, m, r, s, w, C)]
            assert S == ref, (T, s, w, C, t)
            if C >= T:                       # the cap never binds: all policies agree
                assert S == O.attended_set(t, m, s, w, C, O.CAP_RECENT)


@pytest.mark.parametrize("seed", range(4))
def test_lowest_top_scores_equal_arrivals(seed):
    """The closed form (the C best of all arrivals) equals the segment built
    arrival by arrival with a drop of the lowest (score, position)."""
    rng = np.random.default_rng(300 + seed)
    for _ in range(40):
        n = int(rng.integers(0, 60))
        C = int(rng.integers(1, 12))
        r = rng.integers(0, int(rng.choice([3, 50])), n) / 7.0
        order = list(range(n))
        for k in range(n + 1):
            assert sorted(O.top_by_score(order[:k], r, C)) == arrivals_lowest(order[:k], r, C)


def test_lowest_policy_closed_forms():
    """Scores rising with position: the lowest is always the oldest, so the
    segment is the C most recent (policy "recent"); falling scores: the
    newcomer is always the lowest, so the first C stay (policy "first")."""
    T, s, w, C = 110, 3, 9, 6
    ones = O.fed_mask(np.ones(T, np.uint8), s)
    up = np.linspace(0.1, 0.9, T)
    down = up[::-1].copy()
    for t in range(T):
        assert (O.attended_set(t, ones, s, w, C, O.CAP_LOWEST, up) ==
                O.attended_set(t, ones, s, w, C, O.CAP_RECENT))
        assert (O.attended_set(t, ones, s, w, C, O.CAP_LOWEST, down) ==
                O.attended_set(t, ones, s, w, C, O.CAP_FIRST))
    # equal scores everywhere: ties go against the older token, as in "recent"
    flat = np.full(T, 0.5)
    for t in range(T):
        assert (O.attended_set(t, ones, s, w, C, O.CAP_LOWEST, flat) ==
                O.attended_set(t, ones, s, w, C, O.CAP_RECENT))


def test_closed_forms():
    rng = np.random.default_rng(11)
    T, s, w = 200, 4, 16
    m_rand = O.fed_mask((rng.random(T) < 0.4).astype(np.uint8), s)
    zeros = np.zeros(T, np.uint8)
    ones = O.fed_mask(np.ones(T, np.uint8), s)
    for t in range(T):
        # w >= T: full causal attention
        assert len(O.attended_set(t, m_rand, s, T, 7)) == t + 1
        # r == 0: sink + window
        n0 = min(t + 1, w) + len([j for j in range(s) if j <= t - w])
        assert len(O.attended_set(t, zeros, s, w, 50)) == n0
        # C == 0: sink + window for any r
        assert len(O.attended_set(t, m_rand, s, w, 0)) == n0
        # r == 1 with C >= T: full causal attention
        assert O.attended_set(t, ones, s, w, T) == list(range(t + 1))
        # with the cap binding, exactly min(C, #retained) extra keys
        nret = int(sum(ones[s:max(s, t - w + 1)]))
        assert len(O.attended_set(t, ones, s, w, 10)) == n0 + min(10, nret)


def test_compact_vs_cumsum():
    rng = np.random.default_rng(2)
    m = (rng.random(300) < 0.2).astype(np.uint8)
    idx, n, cnt = O.compact(m)
    assert n == int(m.sum())
    np.testing.assert_array_equal(idx, np.flatnonzero(m))
    np.testing.assert_array_equal(cnt, np.cumsum(m))


def test_prefill_count_formula():
    """Row count from the compaction arrays (the form a kernel uses):
    |S_t| = min(t+1,w) + #sinks out of window + min(C, cnt[t-w])."""
    rng = np.random.default_rng(4)
    T, s, w, C = 300, 4, 32, 9
    m = O.fed_mask((rng.random(T) < 0.3).astype(np.uint8), s)
    _, _, cnt = O.compact(m)
    for t in range(T):
        n = cnt[t - w] if t - w >= 0 else 0
        expect = min(t + 1, w) + len([j for j in range(s) if j <= t - w]) + min(C, n)
        assert len(O.attended_set(t, m, s, w, C)) == expect


def test_golden_fig2_setting():
    """Fig. 2 of the LTE paper draws s=2, w=12; the fixture holds a mask and
    the attended sets for that setting, written by tests/golden/make_golden.py
    from the oracle and checked here against the brute-force rule too."""
    with open(os.path.join(GOLDEN, "fig2_sets.json")) as f:
        gold = json.load(f)
    s, w, C = gold["sink"], gold["window"], gold["cap"]
    m = np.array(gold["mask"], np.uint8)
    for t, S in enumerate(gold["sets"]):
        assert O.attended_set(t, m, s, w, C) == S
        assert S == [j for j in range(len(m)) if brute_member(j, t, m, s, w, C)]


def test_worked_example_sets_by_hand():
    """A hand-derived example (tests/golden/worked_example_sets.json, with its
    derivation): s = 1, w = 3, C = 2 over ten tokens, for all three cap
    policies.  The expected sets were worked out from the LTE paper's Fig. 2
    caption (sinks, window, at most C retained KVs per head), not by the oracle,
    so this pins the oracle's set logic independently of its own code."""
    with open(os.path.join(GOLDEN, "worked_example_sets.json")) as f:
        gold = json.load(f)
    s, w, C = gold["sink"], gold["window"], gold["cap"]
    m = O.fed_mask(np.array(gold["mask"], np.uint8), s)
    r = np.array(gold["scores"], np.float64)
    for policy, sets in gold["sets"].items():
        for t, expect in enumerate(sets):
            got = O.attended_set(t, m, s, w, C, policy, r if policy == O.CAP_LOWEST else None)
            assert got == expect, f"{policy} t={t}: {got} != {expect}"
