"""GPU parity of lte_sparse_attn_backward (gradients of the prefill attention
for fixed attended sets) against the oracle's prefill_backward, through the
C ABI, on seeded inputs spanning several tiles with ragged tails, all three cap
policies, GQA group sizes 1 to 16 and head dims 64 and 128.

Tolerance.  The oracle works in float64 on the same bf16 inputs.  The kernels
round P and dS to bf16 (relative 2^-9 each) before the products that use
them, so every term of a gradient sum carries a relative error of about
2^-8.  D_t = <dO_t, o_t> is taken, as the call's contract states, from the
forward output as stored (bf16); the oracle is given its own o rounded to
bf16 for D_t, and dq gets an allowance for the forward output's own error
in D_t (tests/gpu_util.dq_delta_allowance: it matters only on rows with few
keys, where dq is a near-cancelling sum).  Every element must lie
within 2e-2 of its row's largest reference entry (a row: one position of dk
or dv, one (position, head) of dq), so a missing or doubled contribution to
any one position fails; the relative Frobenius error of each tensor must also
stay below 1e-2."""
import numpy as np
import pytest
import torch

import lte_inputs as LI
from oracle import lte_oracle as O
from tests.gpu_util import (assert_grad_close, bf16_round, dq_delta_allowance, f64, fed_masks,
                            scale_of)

pytestmark = pytest.mark.gpu

REL_FRO = 1e-2


@pytest.fixture(scope="module")
def layer():
    from learnable_kv_token_b200 import layer
    return layer


def _close(g, ref, what, extra=None):
    g, ref = np.asarray(g, np.float64), np.asarray(ref, np.float64)
    fro = np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)
    assert fro <= REL_FRO, f"{what}: relative Frobenius {fro:.2e}"
    mx = assert_grad_close(g, ref, what, extra)
    return fro, mx


CASES = [
    # B, T, Hq, Hkv, D, sink, window, cap, policy, retention source
    (2, 700, 8, 2, 128, 4, 128, 24, "recent", 0.3),
    (1, 333, 4, 1, 64, 2, 37, 5, "first", 0.5),
    (1, 500, 16, 4, 128, 4, 64, 40, "lowest", 8),       # grid scores with 8 levels (ties)
    (1, 300, 8, 8, 128, 0, 16, 3, "recent", 0.7),       # G = 1, no sink
    (1, 260, 16, 1, 64, 5, 50, 0, "recent", 0.6),       # G = 16, cap 0
    (1, 200, 4, 2, 128, 3, 400, 10, "recent", 0.5),     # window longer than the sequence
    (1, 300, 16, 1, 128, 4, 48, 12, "recent", 0.5),     # G = 16 on the tcgen05 kernels
    (1, 260, 16, 2, 128, 2, 40, 9, "first", 0.4),       # G = 8
    (2, 190, 4, 2, 128, 1, 30, 6, "lowest", 16),        # G = 2, lowest-score policy
    # long enough that a column tile's attending rows exceed one work item of the
    # tcgen05 column pass (several CTAs add into the same slots) under each policy
    (1, 2048, 8, 2, 128, 4, 256, 48, "first", 0.5),
    (1, 2048, 8, 2, 128, 4, 256, 48, "lowest", 8),
]
POLICY = {"recent": (0, O.CAP_RECENT), "first": (1, O.CAP_FIRST), "lowest": (2, O.CAP_LOWEST)}


@pytest.mark.parametrize("case", CASES)
def test_backward_vs_oracle(layer, case):
    B, T, Hq, Hkv, D, sink, window, cap, policy, src = case
    code, opol = POLICY[policy]
    g = LI.generator(900 + T + D)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, torch.bfloat16, g)
    do = LI.normal((B, T, Hq, D), 1.0, torch.bfloat16, g)
    p = layer.LayerParams(sink=sink, window=window, cap=cap, tau=0.5, cap_policy=code)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    if policy == "lowest":
        r = LI.grid_scores(B, Hkv, T, src, g)
        out = layer.prefill(qd, kd, vd, p, scores=r.cuda())
        masks = np.stack([[O.retention_mask(f64(r[b, h]), sink, 0.5) for h in range(Hkv)]
                          for b in range(B)])
        r64 = f64(r)
    else:
        mask = LI.bernoulli_mask(B, Hkv, T, src, g)
        out = layer.prefill(qd, kd, vd, p, mask=mask.cuda())
        masks, r64 = fed_masks(mask, sink), None
    dq, dk, dv = layer.backward(qd, kd, vd, out, dod, p, check_errors=True)
    torch.cuda.synchronize()
    # D_t comes from the forward's stored output: the oracle's o rounded to bf16
    o_ref, _, _ = O.prefill(f64(q), f64(k), f64(v), masks, sink, window, cap, scale_of(D), opol, r64)
    pk, _, _ = O.prefill(f64(q), f64(k), f64(k), masks, sink, window, cap, scale_of(D), opol, r64)
    rq, rk, rv = O.prefill_backward(f64(q), f64(k), f64(v), masks, sink, window, cap, f64(do),
                                    scale_of(D), opol, r64, o_out=bf16_round(o_ref))
    extra = {"dq": dq_delta_allowance(f64(do), o_ref, pk, scale_of(D)), "dk": None, "dv": None}
    for name, a, b in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        fro, mx = _close(f64(a), b, f"{name} {case}", extra[name])
        print(f"{name}: relative Frobenius {fro:.2e}, worst element / row max {mx:.2e}")


def test_backward_gradient_check_direction(layer):
    """The directional derivative of L = sum <dO, o> along a random direction
    e of q, by central differences of the oracle's float64 forward, agrees
    with <dq, e> from the GPU backward: a check that uses no backward formula."""
    B, T, Hq, Hkv, D, sink, window, cap = 1, 256, 4, 1, 128, 2, 32, 6
    g = LI.generator(77)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, torch.bfloat16, g)
    do = LI.normal((B, T, Hq, D), 1.0, torch.bfloat16, g)
    mask = LI.bernoulli_mask(B, Hkv, T, 0.4, g)
    p = layer.LayerParams(sink=sink, window=window, cap=cap)
    qd, kd, vd, dod, md = (x.cuda() for x in (q, k, v, do, mask))
    out = layer.prefill(qd, kd, vd, p, mask=md)
    dq, _, _ = layer.backward(qd, kd, vd, out, dod, p, check_errors=True)
    # the oracle's forward in float64 along q + eps * e, e a random direction
    e = LI.normal((B, T, Hq, D), 1.0, torch.float32, g)
    masks = fed_masks(mask, sink)
    eps = 1e-4

    def loss(qq):
        o, _, _ = O.prefill(qq, f64(k), f64(v), masks, sink, window, cap, scale_of(D))
        return float((o * f64(do)).sum())

    num = (loss(f64(q) + eps * f64(e)) - loss(f64(q) - eps * f64(e))) / (2 * eps)
    ana = float((f64(dq) * f64(e)).sum())
    assert abs(num - ana) <= 1e-2 * abs(num) + 1e-6, (num, ana)
