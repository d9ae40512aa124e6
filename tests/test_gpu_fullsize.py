"""Parity at the full workload sizes, in the launch configuration the bench
times, on sampled (batch, KV head, row) outputs that the oracle computes one
by one.

* prefill workload: B=32, T=4096, Hq=16, Hkv=4, D=128, s=4, w=512, C=512,
  retention mask Bernoulli(0.1) fed;
* long-context sweep: B=4, T=16384, w=1024, C in {0, 1024, 4096, 16384} x
  per-head retention rates ~ U[0, 2*rate] clipped, rate in {0, 5, 25, 100} %
  (rate 100 % with C = 16384 is full causal attention);
* laLTE hybrid pair: B=32 x 4096-token prompts, the CNN scored live (sampled
  units against the oracle's scores), and the gated linear-attention layer
  (16 heads, dk = dv = 128) through prefill and 256 decode steps (sampled
  heads against the oracle's recurrence).
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


# --------------------------------------------------------------------------- laLTE hybrid pair
def test_hybrid_scores_sampled():
    """lte_score at the hybrid workload's size (B=32, 4096-token prompts, Hkv=4,
    D=128, the CNN live): sampled units against the oracle's scores, masks exact
    off the band around tau."""
    from learnable_kv_token_b200 import lte as L
    from oracle import lte_oracle as O
    from tests.gpu_util import MASK_BAND, R_TOL, oracle_cnn
    wl = LI.WORKLOADS["hybrid"]
    inp = LI.lte_inputs(wl, T=wl.T)
    k, v, cnn = inp["k"], inp["v"], inp["cnn"]
    B, T, Hkv = wl.B, wl.T, wl.Hkv
    dims = L.make_dims(B, T, wl.Hq, Hkv, wl.D, wl.sink, wl.window, wl.cap, wl.tau, scale_of(wl.D),
                       wl.dtype)
    c, _keep = L.make_cnn(*(x.cuda() for x in cnn), wl.past1, wl.past2)
    n = T - 3
    r = torch.full((B, Hkv, T), float("nan"), device="cuda")
    m = torch.zeros(B, Hkv, T, dtype=torch.uint8, device="cuda")
    L.lte_score(dims, c, k.cuda(), v.cuda(), 0, n, r, m)
    torch.cuda.synchronize()
    assert torch.isfinite(r[..., :n]).all()
    for b, h in [(0, 0), (7, 2), (19, 1), (31, 3)]:
        ro = O.cnn_scores(f64(k[b, :, h]), f64(v[b, :, h]), oracle_cnn(cnn, h, wl.past1, wl.past2))
        np.testing.assert_allclose(f64(r[b, h])[:n], ro[:n], atol=R_TOL, rtol=0)
        clear = np.abs(ro[:n] - wl.tau) > MASK_BAND
        np.testing.assert_array_equal(m[b, h].cpu().numpy()[:n][clear],
                                      O.retention_mask(ro, wl.sink, wl.tau)[:n][clear])


def test_hybrid_gla_sampled():
    """The gated linear-attention layer of the pair at full size: prefill of
    B=32 x 4096 tokens x 16 heads (dk = dv = 128), then 256 decode steps; sampled
    heads against the oracle's token-by-token recurrence (outputs of every token
    and the final state, max-abs error relative to max |reference| <= 1e-2)."""
    from learnable_kv_token_b200 import lte as L
    from oracle import gla_oracle as GO
    wl = LI.WORKLOADS["hybrid"]
    B, T, H, dk, steps = wl.B, wl.T, 16, 128, wl.decode_steps
    q, k, v, a = LI.gla_inputs(B, T + steps, H, dk, dk, LI.generator(wl.seed + 1000))
    qd, kd, vd, ad = (x.cuda() for x in (q, k, v, a))
    o = torch.empty(B, T, H, dk, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(B, H, dk, dk, dtype=torch.float32, device="cuda")
    L.lte_gla_prefill(qd[:, :T].contiguous(), kd[:, :T].contiguous(), vd[:, :T].contiguous(),
                      ad[:, :T].contiguous(), o, st)
    od = torch.empty(steps, B, H, dk, dtype=torch.bfloat16, device="cuda")
    for t in range(steps):
        L.lte_gla_decode_step(qd[:, T + t].contiguous(), kd[:, T + t].contiguous(),
                              vd[:, T + t].contiguous(), ad[:, T + t].contiguous(), od[t], st)
    torch.cuda.synchronize()

    def rel(got, ref):
        return float(np.abs(got - ref).max() / np.abs(ref).max())

    for b, h in [(0, 0), (17, 9), (31, 15)]:
        o_ref, S_ref = GO.gla_recurrent(f64(q[b, :, h]), f64(k[b, :, h]), f64(v[b, :, h]),
                                        f64(a[b, :, h]))
        assert rel(f64(o[b, :, h]), o_ref[:T]) <= 1e-2, (b, h)
        assert rel(f64(od[:, b, h]), o_ref[T:]) <= 1e-2, (b, h)
        assert rel(f64(st[b, h]), S_ref) <= 1e-2, (b, h)


# --------------------------------------------------------------------------- attention backward
def test_backward_bench_shape_sampled(layer):
    """lte_sparse_attn_backward at the bench's shape -- B=32, T=4096, Hq=16 /
    Hkv=4, D=128, s=4, w=512, C=512, a fed Bernoulli(0.5) retention mask, so the
    cap binds from t ~ 1500 on and a retained slot is attended from ~1000 rows
    (the column pass's multi-CTA atomics at full depth) -- against the oracle's
    prefill_backward_unit for two whole units: every element of dq, dk and dv
    within 2e-2 of its row's largest reference entry (D_t from the oracle's own
    o rounded to bf16, the forward's stored output)."""
    from oracle import lte_oracle as O
    from tests.gpu_util import assert_grad_close, bf16_round, dq_delta_allowance
    B, T, Hq, Hkv, D, sink, window, cap = 32, 4096, 16, 4, 128, 4, 512, 512
    G = Hq // Hkv
    g = LI.generator(4242)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, torch.bfloat16, g)
    do = LI.normal((B, T, Hq, D), 1.0, torch.bfloat16, g)
    mask = LI.bernoulli_mask(B, Hkv, T, 0.5, g)
    p = layer.LayerParams(sink=sink, window=window, cap=cap)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    out = layer.prefill(qd, kd, vd, p, mask=mask.cuda())
    dq, dk, dv = layer.backward(qd, kd, vd, out, dod, p, check_errors=True)
    torch.cuda.synchronize()
    masks = fed_masks(mask, sink)
    for b, h in [(0, 0), (31, 3)]:
        o_ref, _, _ = O.prefill_unit(f64(q[b, :, h * G:(h + 1) * G]), f64(k[b, :, h]),
                                     f64(v[b, :, h]), masks[b, h], sink, window, cap, scale_of(D))
        rq, rk, rv = O.prefill_backward_unit(f64(q[b, :, h * G:(h + 1) * G]), f64(k[b, :, h]),
                                             f64(v[b, :, h]), masks[b, h], sink, window, cap,
                                             scale_of(D), f64(do[b, :, h * G:(h + 1) * G]),
                                             o_out=bf16_round(o_ref))
        pk, _, _ = O.prefill_unit(f64(q[b, :, h * G:(h + 1) * G]), f64(k[b, :, h]),
                                  f64(k[b, :, h]), masks[b, h], sink, window, cap, scale_of(D))
        assert_grad_close(f64(dq[b, :, h * G:(h + 1) * G]), rq, f"dq unit {b},{h}",
                          dq_delta_allowance(f64(do[b, :, h * G:(h + 1) * G]), o_ref, pk, scale_of(D)))
        assert_grad_close(f64(dk[b, :, h]), rk, f"dk unit {b},{h}")
        assert_grad_close(f64(dv[b, :, h]), rv, f"dv unit {b},{h}")
