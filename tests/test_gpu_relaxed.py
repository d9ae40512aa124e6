"""GPU parity of the relaxed-retention training path against the oracle
(``prefill_relaxed_unit``, ``prefill_relaxed_backward_unit``), through the C
ABI: lte_sparse_attn_prefill_relaxed (o, lse) and
lte_sparse_attn_backward_relaxed (dq, dk, dv and dL/dr), all three cap
policies, GQA groups 1 to 16, several tiles and ragged tails.

Reading (the pages give no gradient rule for the keep decision): the hard
attended sets stay, and every retained-segment key j enters the softmax with
weight r_j.  Tolerances as for the hard kernels: the attention gates for o
and lse; dq, dk, dv element by element within 2e-2 of their row's largest
reference entry; dr (a sum over the rows that attend a key through the
retained segment, of bf16-rounded products) within 1e-2 of the unit's
largest |dr| at every position, and relative Frobenius 1e-2.  As for the hard
backward, D_t comes from the stored (bf16) forward output: the oracle gets
its own o rounded to bf16 for it."""
import numpy as np
import pytest
import torch

import lte_inputs as LI
from oracle import lte_oracle as O
from tests.gpu_util import (assert_attention_close, assert_grad_close, bf16_round,
                            dq_delta_allowance, f64, scale_of)

pytestmark = pytest.mark.gpu

POLICY = {"recent": (0, O.CAP_RECENT), "first": (1, O.CAP_FIRST), "lowest": (2, O.CAP_LOWEST)}
CASES = [
    # B, T, Hq, Hkv, sink, window, cap, policy, score levels (0: uniform)
    (2, 700, 8, 2, 4, 128, 24, "recent", 0),
    (1, 500, 16, 4, 4, 64, 40, "lowest", 8),
    (1, 300, 8, 8, 0, 16, 3, "first", 0),
    (1, 260, 16, 1, 2, 40, 9, "recent", 16),
    # the first C retained slots are attended by every later row: their rows span
    # several column work items, whose dK, dV and dL/dr adds meet in the same slots
    (1, 2048, 8, 2, 4, 256, 48, "first", 0),
]


@pytest.fixture(scope="module")
def layer():
    from learnable_kv_token_b200 import layer
    return layer


def _setup(layer, case, seed):
    B, T, Hq, Hkv, s, w, C, policy, levels = case
    code, opol = POLICY[policy]
    D = 128
    g = LI.generator(seed)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, torch.bfloat16, g)
    do = LI.normal((B, T, Hq, D), 1.0, torch.bfloat16, g)
    r = (LI.grid_scores(B, Hkv, T, levels, g) if levels else
         torch.rand(B, Hkv, T, generator=g, dtype=torch.float32))
    p = layer.LayerParams(sink=s, window=w, cap=C, tau=0.5, cap_policy=code)
    qd, kd, vd, dod, rd = (x.cuda() for x in (q, k, v, do, r))
    out = layer.prefill(qd, kd, vd, p, scores=rd)
    return dict(q=q, k=k, v=v, do=do, r=r, p=p, qd=qd, kd=kd, vd=vd, dod=dod, rd=rd, out=out,
                opol=opol, G=Hq // Hkv, D=D)


@pytest.mark.parametrize("case", CASES)
def test_relaxed_forward_and_backward_vs_oracle(layer, case):
    B, T, Hq, Hkv, s, w, C, policy, levels = case
    c = _setup(layer, case, 3100 + T)
    o, lse, ws = layer.prefill_relaxed(c["qd"], c["kd"], c["vd"], c["out"], c["rd"], c["p"])
    dq, dk, dv, dr = layer.backward_relaxed(c["qd"], c["kd"], c["vd"], c["out"], c["rd"], o, lse,
                                            c["dod"], c["p"], ws, check_errors=True)
    torch.cuda.synchronize()
    G, D = c["G"], c["D"]
    for b in range(B):
        for h in range(Hkv):
            r64 = f64(c["r"][b, h])
            m = O.retention_mask(r64, s, 0.5)
            sl = slice(h * G, (h + 1) * G)
            o_ref, lse_ref = O.prefill_relaxed_unit(f64(c["q"][b, :, sl]), f64(c["k"][b, :, h]),
                                                    f64(c["v"][b, :, h]), m, s, w, C, scale_of(D),
                                                    r64, policy=c["opol"])
            assert_attention_close(f64(o[b, :, sl]), f64(lse[b, sl]).T, o_ref, lse_ref,
                                   torch.bfloat16, f"forward {case} unit {b},{h}")
            rq, rk, rv, rr = O.prefill_relaxed_backward_unit(
                f64(c["q"][b, :, sl]), f64(c["k"][b, :, h]), f64(c["v"][b, :, h]), m, s, w, C,
                scale_of(D), f64(c["do"][b, :, sl]), r64, policy=c["opol"],
                o_out=bf16_round(o_ref))
            pk, _ = O.prefill_relaxed_unit(f64(c["q"][b, :, sl]), f64(c["k"][b, :, h]),
                                           f64(c["k"][b, :, h]), m, s, w, C, scale_of(D), r64,
                                           policy=c["opol"])
            assert_grad_close(f64(dq[b, :, sl]), rq, f"dq {case} unit {b},{h}",
                              dq_delta_allowance(f64(c["do"][b, :, sl]), o_ref, pk, scale_of(D)))
            assert_grad_close(f64(dk[b, :, h]), rk, f"dk {case} unit {b},{h}")
            assert_grad_close(f64(dv[b, :, h]), rv, f"dv {case} unit {b},{h}")
            g_dr = f64(dr[b, h])
            scale = np.abs(rr).max()
            assert scale > 0 or C == 0
            assert np.abs(g_dr - rr).max() <= 1e-2 * scale + 1e-6, \
                f"dr {case} unit {b},{h}: {np.abs(g_dr - rr).max():.3g} vs {scale:.3g}"
            assert np.linalg.norm(g_dr - rr) <= 1e-2 * np.linalg.norm(rr) + 1e-6
            assert np.all(g_dr[rr == 0] == 0)            # only retained-segment keys get dL/dr


def test_relaxed_unit_weights_equal_hard(layer):
    """r = 1 on every retained token: the relaxed calls equal the hard ones
    (bit-identical o and lse -- the log weights are exactly 0 -- and dq, dk,
    dv within atomics' rounding), while dL/dr is still produced."""
    case = (1, 400, 8, 2, 4, 64, 16, "recent", 0)
    c = _setup(layer, case, 77)
    ones = torch.ones_like(c["rd"])
    o, lse, ws = layer.prefill_relaxed(c["qd"], c["kd"], c["vd"], c["out"], ones, c["p"])
    torch.cuda.synchronize()
    assert torch.equal(o, c["out"].o) and torch.equal(lse, c["out"].lse)
    dq, dk, dv, dr = layer.backward_relaxed(c["qd"], c["kd"], c["vd"], c["out"], ones, o, lse,
                                            c["dod"], c["p"], ws, check_errors=True)
    hq, hk, hv = layer.backward(c["qd"], c["kd"], c["vd"], c["out"], c["dod"], c["p"],
                                check_errors=True)
    torch.cuda.synchronize()
    assert torch.equal(dq, hq)
    for a, b in ((dk, hk), (dv, hv)):
        assert (a - b).abs().max().item() <= 1e-5 * b.abs().max().item()
    assert dr.abs().max().item() > 0
