"""GPU parity of the gated linear-attention layer (chunk-wise prefill and the
recurrent decode step) against the oracle's float64 token-by-token
recurrence, on identical seeded inputs.

Tolerance: bf16 operands with fp32 accumulation, measured as max-abs error
relative to max |reference| (<= 1e-2 for bf16, <= 1e-5 for the fp32 decode
arithmetic), on both the outputs and the final state."""
import numpy as np
import pytest
import torch

import lte_inputs as LI
from oracle import gla_oracle as GO

pytestmark = pytest.mark.gpu


def f64(t):
    return t.detach().cpu().double().numpy()


def rel_err(got, ref):
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))


@pytest.fixture(scope="module")
def L():
    from learnable_kv_token_b200 import lte
    return lte


@pytest.mark.parametrize("B,T,H,gates,init", [(2, 256, 3, "sigmoid", False), (1, 192, 2, "ones", False),
                                              (1, 128, 2, "sigmoid", True), (1, 64, 1, "low", False)])
def test_gla_prefill_vs_recurrence(L, B, T, H, gates, init):
    g = LI.generator(T + H)
    q, k, v, a = LI.gla_inputs(B, T, H, 128, 128, g)
    if gates == "ones":
        a = torch.ones_like(a)
    elif gates == "low":          # faster decay: products down to ~sigmoid(0)^32 over a half chunk
        a = torch.sigmoid(torch.randn(a.shape, generator=g) * 0.5)
    S0 = torch.randn(B, H, 128, 128, generator=g) * 0.05 if init else torch.zeros(B, H, 128, 128)
    o = torch.empty_like(q, device="cuda")
    st = S0.clone().cuda()
    L.lte_gla_prefill(q.cuda(), k.cuda(), v.cuda(), a.cuda(), o, st)
    torch.cuda.synchronize()
    o_ref, S_ref = GO.gla(f64(q), f64(k), f64(v), f64(a), S0=f64(S0) if init else None)
    assert rel_err(f64(o), o_ref) <= 1e-2
    assert rel_err(f64(st), S_ref) <= 1e-2


@pytest.mark.parametrize("kind", ["all-0.05", "sparse-zeros", "alternating"])
def test_gla_prefill_any_gate(L, kind):
    """Gates far below the chunk form's range: a = 0.05 everywhere (the product
    of 32 gates is 2e-42), and typical gates with a = 0 or 1e-3 at a few
    (token, channel) entries, and chunks that alternate between the two.  The
    chunks whose gates leave the range run the recurrence token by token; the
    result still matches the float64 recurrence at relative 1e-2, and the
    final state too (the state then flows into the next chunk of either kind)."""
    B, T, H = 2, 320, 2
    g = LI.generator(4000 + len(kind))
    q, k, v, a = LI.gla_inputs(B, T, H, 128, 128, g)
    if kind == "all-0.05":
        a = torch.full_like(a, 0.05)
    elif kind == "sparse-zeros":
        pick = torch.rand(a.shape, generator=g) < 2e-3
        a = torch.where(pick, torch.where(torch.rand(a.shape, generator=g) < 0.5, 0.0, 1e-3), a)
    else:                             # chunks 1, 3 of each sequence at 0.05, the others typical
        for c in (1, 3):
            a[:, 64 * c:64 * (c + 1)] = 0.05
    S0 = torch.randn(B, H, 128, 128, generator=g) * 0.05
    o = torch.empty_like(q, device="cuda")
    st = S0.clone().cuda()
    L.lte_gla_prefill(q.cuda(), k.cuda(), v.cuda(), a.cuda(), o, st)
    torch.cuda.synchronize()
    o_ref, S_ref = GO.gla(f64(q), f64(k), f64(v), f64(a), S0=f64(S0))
    assert np.isfinite(f64(o)).all() and np.isfinite(f64(st)).all()
    assert rel_err(f64(o), o_ref) <= 1e-2
    assert rel_err(f64(st), S_ref) <= 1e-2


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, 1e-2), (torch.float32, 1e-5)])
def test_gla_decode_continues_recurrence(L, dtype, tol):
    B, T0, steps, H = 2, 128, 12, 2
    g = LI.generator(99)
    q, k, v, a = LI.gla_inputs(B, T0 + steps, H, 128, 128, g, dtype=dtype)
    S0 = torch.randn(B, H, 128, 128, generator=g) * 0.05
    st = S0.clone().cuda()
    outs = []
    for t in range(T0, T0 + steps):
        o_t = torch.empty(B, H, 128, dtype=dtype, device="cuda")
        L.lte_gla_decode_step(q[:, t].contiguous().cuda(), k[:, t].contiguous().cuda(),
                              v[:, t].contiguous().cuda(), a[:, t].contiguous().cuda(), o_t, st)
        outs.append(o_t)
    torch.cuda.synchronize()
    o_ref, S_ref = GO.gla(f64(q[:, T0:]), f64(k[:, T0:]), f64(v[:, T0:]), f64(a[:, T0:]), S0=f64(S0))
    got = np.stack([f64(x) for x in outs], axis=1)
    assert rel_err(got, o_ref) <= tol
    assert rel_err(f64(st), S_ref) <= tol


def test_gla_prefill_then_decode(L):
    """Prefill 128 tokens, then decode 8: the outputs continue the single
    recurrence over all 136 tokens."""
    B, T0, steps, H = 1, 128, 8, 2
    g = LI.generator(5)
    q, k, v, a = LI.gla_inputs(B, T0 + steps, H, 128, 128, g)
    st = torch.zeros(B, H, 128, 128, device="cuda")
    o = torch.empty(B, T0, H, 128, dtype=torch.bfloat16, device="cuda")
    L.lte_gla_prefill(q[:, :T0].contiguous().cuda(), k[:, :T0].contiguous().cuda(),
                      v[:, :T0].contiguous().cuda(), a[:, :T0].contiguous().cuda(), o, st)
    outs = []
    for t in range(T0, T0 + steps):
        o_t = torch.empty(B, H, 128, dtype=torch.bfloat16, device="cuda")
        L.lte_gla_decode_step(q[:, t].contiguous().cuda(), k[:, t].contiguous().cuda(),
                              v[:, t].contiguous().cuda(), a[:, t].contiguous().cuda(), o_t, st)
        outs.append(o_t)
    torch.cuda.synchronize()
    o_ref, _ = GO.gla(f64(q), f64(k), f64(v), f64(a))
    assert rel_err(f64(o), o_ref[:, :T0]) <= 1e-2
    assert rel_err(np.stack([f64(x) for x in outs], axis=1), o_ref[:, T0:]) <= 1e-2


def test_gla_rejects_unsupported(L):
    q = torch.zeros(1, 100, 1, 128, dtype=torch.bfloat16, device="cuda")     # T % 64 != 0
    a = torch.ones(1, 100, 1, 128, device="cuda")
    with pytest.raises(L.LteError) as ei:
        L.lte_gla_prefill(q, q, q, a, torch.empty_like(q), torch.zeros(1, 1, 128, 128, device="cuda"))
    assert ei.value.status == 2
