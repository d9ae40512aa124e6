"""Parity at the full workload sizes, in the launch configuration the bench
times, on sampled (batch, KV head, row) outputs that the oracle computes one
by one.

* prefill workload: B=32, T=4096, Hq=16, Hkv=4, D=128, s=4, w=512, C=512,
  retention mask Bernoulli(0.1) fed;
* long-context sweep: B=4, T=16384, w=1024, C in {0, 1024, 4096, 16384} x
  per-head retention rates ~ U[0, 2*rate] clipped, rate in {0, 5, 25, 100} %
  (rate 100 % with C = 16384 is full causal attention).
Rows are sampled at the window / sink / cap boundaries, the ragged end, and
uniformly in between."""
import numpy as np
import pytest
import torch

import lte_inputs as LI
from tests.gpu_util import assert_attention_close, f64, fed_masks, oracle_rows, scale_of

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def layer():
    from learnable_kv_token_b200 import layer
    return layer


def _rows(T, window, sink, rng, n_random=16):
    edges = [0, 1, sink, window - 1, window, window + sink - 1, window + sink, window + sink + 1,
             2 * window, T // 2, T - 2, T - 1]
    rows = sorted(set([r for r in edges if 0 <= r < T] + rng.integers(0, T, n_random).tolist()))
    return rows


def _check(q, k, v, mask, out, units, sink, window, cap, rng, dtype=torch.bfloat16):
    T, Hq, Hkv, D = q.shape[1], q.shape[2], k.shape[2], q.shape[3]
    G = Hq // Hkv
    masks = fed_masks(mask, sink)
    for b, h in units:
        rows = _rows(T, window, sink, rng)
        o_ref, lse_ref, _ = oracle_rows(q, k, v, masks, b, h, rows, sink, window, cap, scale_of(D))
        o_g = f64(out.o[b, rows, h * G:(h + 1) * G])
        lse_g = f64(out.lse[b, h * G:(h + 1) * G][:, rows]).T
        assert_attention_close(o_g, lse_g, o_ref, lse_ref, dtype, f"unit {b},{h}")


def test_prefill_workload_sampled(layer):
    wl = LI.WORKLOADS["prefill"]
    inp = LI.lte_inputs(wl, T=wl.T)
    q, k, v, mask = inp["q"], inp["k"], inp["v"], inp["mask"]
    p = layer.LayerParams(sink=wl.sink, window=wl.window, cap=wl.cap)
    out = layer.prefill(q.cuda(), k.cuda(), v.cuda(), p, mask=mask.cuda())
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    _check(q, k, v, mask, out, [(0, 0), (13, 1), (31, 3)], wl.sink, wl.window, wl.cap, rng)


@pytest.fixture(scope="module")
def sweep_inputs():
    wl = LI.WORKLOADS["sweep"]
    g = LI.generator(wl.seed)
    q, k, v = LI.qkv(wl.B, wl.T, wl.Hq, wl.Hkv, wl.D, wl.dtype, g)
    return wl, q, k, v, (q.cuda(), k.cuda(), v.cuda())


@pytest.mark.parametrize("cap", LI.SWEEP_CAPS)
@pytest.mark.parametrize("rate", LI.SWEEP_RATES)
def test_sweep_sampled(layer, sweep_inputs, cap, rate):
    wl, q, k, v, (qd, kd, vd) = sweep_inputs
    mask = LI.rate_mask(wl.B, wl.Hkv, wl.T, rate, LI.generator(1000 + cap + int(rate * 100)))
    p = layer.LayerParams(sink=wl.sink, window=wl.window, cap=cap)
    out = layer.prefill(qd, kd, vd, p, mask=mask.cuda())
    torch.cuda.synchronize()
    rng = np.random.default_rng(cap + int(rate * 1000))
    _check(q, k, v, mask, out, [(0, 0), (3, 3)], wl.sink, wl.window, cap, rng)
