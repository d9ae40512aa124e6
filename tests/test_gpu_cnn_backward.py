"""GPU parity of lte_score_backward (gradients through the scoring CNN given
dL/dr) against the oracle's cnn_backward, through the C ABI, on seeded inputs
with ragged position tiles, centred and causal taps, bf16 and fp32 inputs.

Tolerance.  The kernels compute in fp32 (the oracle in float64 on the same
inputs): each input gradient sums at most 2 x 64 x 9 products and each weight
gradient B x T of them, with unit roundoff 6e-8, so relative errors stay near
1e-6; the bound is 1e-4 of the tensor's norm and 1e-3 of its largest entry."""
import numpy as np
import pytest
import torch

import lte_inputs as LI
from oracle import lte_oracle as O
from tests.gpu_util import f64, oracle_cnn

pytestmark = pytest.mark.gpu


def _close(g, ref, what):
    g, ref = np.asarray(g, np.float64), np.asarray(ref, np.float64)
    fro = np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)
    mx = np.abs(g - ref).max() / max(np.abs(ref).max(), 1e-30)
    assert fro <= 1e-4 and mx <= 1e-3, f"{what}: relative Frobenius {fro:.2e}, max {mx:.2e}"


@pytest.mark.parametrize("cfg", [
    # B, T, Hkv, D, dtype, past1, past2
    (2, 300, 2, 128, torch.bfloat16, 2, 1),      # the paper's centred taps, ragged tiles
    (1, 200, 3, 64, torch.float32, 4, 2),        # causal taps, fp32 inputs
    (2, 64, 1, 128, torch.bfloat16, 0, 0),       # future-only taps, one tile
])
def test_score_backward_vs_oracle(cfg):
    from learnable_kv_token_b200 import lte as L
    B, T, Hkv, D, dtype, past1, past2 = cfg
    g = LI.generator(700 + T + D)
    _, k, v = LI.qkv(B, T, Hkv, Hkv, D, dtype, g)
    cnn = LI.cnn_weights(Hkv, D, 32, 5, 3, g, 0.05)
    dr = LI.normal((B, Hkv, T), 1.0, torch.float32, g)
    dk0 = LI.normal((B, T, Hkv, D), 1.0, torch.float32, g)      # the gradients are added to these
    dv0 = LI.normal((B, T, Hkv, D), 1.0, torch.float32, g)
    dims = L.make_dims(B, T, Hkv, Hkv, D, 4, 64, 16, 0.5, D ** -0.5, dtype)
    cd = tuple(x.cuda() for x in cnn)
    c, _keep = L.make_cnn(*cd, past1, past2)
    F = (5 - 1 - past1) + (3 - 1 - past2)
    n_scored = T - F
    kd, vd, drd = k.cuda(), v.cuda(), dr.cuda()
    dk, dv = dk0.cuda(), dv0.cuda()
    dw1 = torch.empty_like(cd[0]); db1 = torch.empty_like(cd[1])
    dw2 = torch.empty_like(cd[2]); db2 = torch.empty_like(cd[3])
    ws = torch.zeros(L.lte_score_backward_workspace_bytes(dims, c) + 16, dtype=torch.uint8,
                     device="cuda")
    L.lte_score_backward(dims, c, kd, vd, n_scored, drd, dk, dv, dw1, db1, dw2, db2, ws)
    torch.cuda.synchronize()
    assert L.lte_read_device_error(ws) == (0, 0)
    ref = {n: np.zeros(t.shape) for n, t in (("dk", dk), ("dv", dv), ("dw1", dw1), ("db1", db1),
                                               ("dw2", dw2), ("db2", db2))}
    for b in range(B):
        for h in range(Hkv):
            gk, gv, gw1, gb1, gw2, gb2 = O.cnn_backward(
                f64(k[b, :, h]), f64(v[b, :, h]), oracle_cnn(cnn, h, past1, past2),
                f64(dr[b, h]), n_scored)
            ref["dk"][b, :, h] = gk
            ref["dv"][b, :, h] = gv
            ref["dw1"][h] += gw1
            ref["db1"][h] += gb1
            ref["dw2"][h] += gw2
            ref["db2"][h] += gb2
    _close(f64(dk) - f64(dk0), ref["dk"], "dk")
    _close(f64(dv) - f64(dv0), ref["dv"], "dv")
    for n, t in (("dw1", dw1), ("db1", db1), ("dw2", dw2), ("db2", db2)):
        _close(f64(t), ref[n], n)
