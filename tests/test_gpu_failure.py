"""Failure detection on the GPU without a fault: a bounded device wait that
runs out must end in an error status the host reads, and leave the context
usable.  The wait is the library's bounded mbarrier wait (the one the fused
decode step uses); the barrier's only arrival is gated on a device flag that
nothing sets.  No trap, assert, bad address or endless loop is involved."""
import time

import numpy as np
import pytest
import torch

import lte_inputs as LI
from oracle import lte_oracle as O
from tests.gpu_util import assert_attention_close, clean_tau, f64, oracle_cnn, scale_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from learnable_kv_token_b200 import lte
    return lte


def test_wait_runs_out_into_timeout_status(L):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")       # nothing ever sets it to 1
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    L.lte_wait_probe(flag, 1, 200_000_000, ws)                     # 0.2 s limit
    code, where = L.lte_read_device_error(ws)
    elapsed = time.perf_counter() - t0
    assert code == 4 and where == 301, (code, where)               # LTE_ERR_TIMEOUT at the probe
    assert 0.15 < elapsed < 5.0, elapsed                           # it waited, then gave up
    # the context is still usable: a kernel launched afterwards runs normally
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float((x * 2).sum()) == 2 * 1023 * 1024 / 2


def test_wait_completes_when_flag_is_set(L):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    flag = torch.ones(1, dtype=torch.int32, device="cuda")
    L.lte_wait_probe(flag, 1, 1_000_000_000, ws)
    assert L.lte_read_device_error(ws) == (0, 0)


def test_library_still_correct_after_a_timeout(L):
    """After a wait ran out, the library's kernels still produce parity results:
    a small decode run matches the oracle."""
    from learnable_kv_token_b200 import layer
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lte_wait_probe(flag, 7, 50_000_000, ws)
    assert L.lte_read_device_error(ws)[0] == 4
    B, Hq, Hkv, D, s, w, C, T0, steps, Ds = 1, 8, 2, 128, 4, 48, 16, 100, 30, 8
    g = LI.generator(5)
    q, k, v = LI.qkv(B, T0 + steps, Hq, Hkv, D, torch.bfloat16, g)
    cnn = LI.cnn_weights(Hkv, D, 32, 5, 3, g, 0.1)
    r_or = np.stack([O.cnn_scores(f64(k[0, :, h]), f64(v[0, :, h]), oracle_cnn(cnn, h))
                     for h in range(Hkv)])
    tau, margin = clean_tau(r_or)
    assert margin > 1e-5
    p = layer.LayerParams(sink=s, window=w, cap=C, tau=tau)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    cd = tuple(x.cuda() for x in cnn)
    kp, vp = kd[:, :T0].contiguous(), vd[:, :T0].contiguous()
    out = layer.prefill(qd[:, :T0].contiguous(), kp, vp, p, cnn=cd)
    dims = p.dims(B, T0, Hq, Hkv, D, torch.bfloat16)
    cache = layer.DecodeCache(B, Hkv, D, torch.bfloat16, s, w, C)
    cache.init_from_prefill(dims, kp, vp, out, T0)
    dec = layer.Decoder(dims, cd, p.past1, p.past2, cache, Ds)
    o_g, lse_g = [], []
    for t in range(T0, T0 + steps):
        o, lse = dec.step(qd[:, t].contiguous(), kd[:, t].contiguous(), vd[:, t].contiguous())
        o_g.append(o.clone())
        lse_g.append(lse.clone())
    torch.cuda.synchronize()
    assert L.lte_read_device_error(dec.ws) == (0, 0)
    G = Hq // Hkv
    o_g, lse_g = torch.stack(o_g), torch.stack(lse_g)
    for h in range(Hkv):
        o_ref, lse_ref, _, _, _ = O.decode_unit(f64(q[0, :, h * G:(h + 1) * G]), f64(k[0, :, h]),
                                                f64(v[0, :, h]), T0, s, w, C, tau, oracle_cnn(cnn, h),
                                                Ds, scale_of(D))
        assert_attention_close(f64(o_g[:, 0, h * G:(h + 1) * G]), f64(lse_g[:, 0, h * G:(h + 1) * G]),
                               o_ref, lse_ref, torch.bfloat16, f"unit 0,{h}")
