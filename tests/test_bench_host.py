"""Host-side pieces of bench.py that its reported figures rest on (CPU only).

`attended_pairs` gives |S_t| for every (b, KV head, row t) from a fed mask;
the headline roofline's attended FLOPs are 4 * D * G times its sum, so it is
checked here against the oracle's attended sets, row by row."""
import importlib.util
import os

import numpy as np
import pytest

from oracle import lte_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("T,sink,window,cap,p", [
    (40, 4, 8, 3, 0.3),      # the cap binds
    (40, 4, 8, 64, 0.5),     # the cap never binds
    (33, 0, 5, 2, 0.7),      # no sinks
    (25, 6, 30, 4, 0.5),     # the window covers every row
    (30, 4, 1, 0, 0.5),      # window of one, no retained segment
    (50, 3, 7, 5, 1.0),      # every token retained
    (50, 3, 7, 5, 0.0),      # none retained
])
def test_attended_pairs_equals_oracle_set_sizes(bench, T, sink, window, cap, p):
    rng = np.random.default_rng(T * 1000 + sink * 100 + window * 10 + cap)
    B, H = 2, 3
    mask = (rng.random((B, H, T)) < p).astype(np.uint8)
    got = bench.attended_pairs(mask, sink, window, cap)
    assert got.shape == (B, H, T)
    for b in range(B):
        for h in range(H):
            m = O.fed_mask(mask[b, h], sink)
            want = [len(O.attended_set(t, m, sink, window, cap)) for t in range(T)]
            np.testing.assert_array_equal(got[b, h], want)


def test_attended_pairs_full_causal_when_everything_is_kept(bench):
    """Every token retained and C >= T: |S_t| = t + 1, the causal count."""
    T = 64
    mask = np.ones((1, 2, T), np.uint8)
    got = bench.attended_pairs(mask, 4, 16, T)
    np.testing.assert_array_equal(got[0, 0], np.arange(1, T + 1))


def test_clock_summary_reads_nvidia_smi_rows(bench):
    """The clocks object of the bench line: median SM clock under load, the
    highest max clock seen, and only reasons reported Active."""
    c = bench.Clocks(0)
    c.out = "\n".join([
        "0, 1965, 1965, 701.2, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 998.0, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 900.5, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 0, Not Active, Not Active, Not Active, Not Active",
    ])
    s = c.summary()
    assert s == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    c.out = ""
    assert c.summary()["samples"] == 0
