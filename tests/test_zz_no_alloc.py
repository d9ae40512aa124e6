"""The allocation-free decode entry point (lte_decode_step_noalloc).

Some callers cannot allocate device memory -- a host runtime that keeps the
whole GPU in its own pool and gives a plugin only input and output buffers,
or a latency-critical loop that cannot afford the synchronisation a
cudaMalloc may imply.  For them the library keeps the decode step's scratch
in a fixed static device array instead of a caller workspace.  These tests
call that entry point through the C ABI and check it against
lte_decode_step (same kernels, caller workspace) on two calls in a row, on
two caches set up identically, once with one CTA per unit (the fused step)
and once with more units than SMs (the split step, whose partials and
completion counters live inside the static array).  After every call the
error word in the static array is read back through
lte_noalloc_read_device_error.  The file name makes pytest collect it last.
"""
import numpy as np
import pytest
import torch

import lte_inputs as LI

pytestmark = pytest.mark.gpu


def _setup(B, Hkv, T0, seed):
    from learnable_kv_token_b200 import layer, lte as L
    Hq, D, sink, window, cap = 4 * Hkv, 128, 4, 64, 16
    g = LI.generator(seed)
    q, k, v = (x.cuda() for x in LI.qkv(B, T0 + 2, Hq, Hkv, D, torch.bfloat16, g))
    cnn = tuple(x.cuda() for x in LI.cnn_weights(Hkv, D, 32, 5, 3, g, 0.1))
    p = layer.LayerParams(sink=sink, window=window, cap=cap, tau=0.5)
    kp, vp = k[:, :T0].contiguous(), v[:, :T0].contiguous()
    out = layer.prefill(q[:, :T0].contiguous(), kp, vp, p, cnn=cnn)
    dims = p.dims(B, T0, Hq, Hkv, D, torch.bfloat16)
    assert L.lte_workspace_bytes(dims, L.LTE_WS_DECODE) <= 4 << 20
    caches = []
    for _ in range(2):
        c = layer.DecodeCache(B, Hkv, D, torch.bfloat16, sink, window, cap)
        c.init_from_prefill(dims, kp, vp, out, T0)
        caches.append(c)
    c_struct, keep = L.make_cnn(*cnn, p.past1, p.past2)
    return dict(q=q, k=k, v=v, cnn=cnn, p=p, dims=dims, caches=caches, c_struct=c_struct,
                keep=keep, B=B, Hq=Hq, D=D)


@pytest.mark.parametrize("B,Hkv", [(2, 2), (40, 4)], ids=["fused-4units", "split-160units"])
def test_noalloc_decode_matches_workspace_variant(B, Hkv):
    from learnable_kv_token_b200 import layer, lte as L
    T0 = 150
    s = _setup(B, Hkv, T0, 314 + B)
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    if B * Hkv > 100:
        assert B * Hkv > n_sm                       # the split step: more units than SMs
    caches = s["caches"]
    ref = layer.Decoder(s["dims"], s["cnn"], s["p"].past1, s["p"].past2, caches[0], score_batch=4)
    o_na = torch.empty(B, s["Hq"], s["D"], dtype=torch.bfloat16, device="cuda")
    lse_na = torch.empty(B, s["Hq"], dtype=torch.float32, device="cuda")
    for t in (T0, T0 + 1):                                   # two calls in a row
        qt, kt, vt = (x[:, t].contiguous() for x in (s["q"], s["k"], s["v"]))
        o_ref, lse_ref = ref.step(qt, kt, vt)
        L.lte_decode_step_noalloc(s["dims"], s["c_struct"], caches[1].struct, qt, kt, vt, o_na,
                                  lse_na, 4)
        assert L.lte_noalloc_read_device_error() == (0, 0)
        assert ref.device_error() == (0, 0)
        np.testing.assert_allclose(o_na.float().cpu().numpy(), o_ref.float().cpu().numpy(),
                                   atol=2e-2, rtol=0)
        np.testing.assert_allclose(lse_na.cpu().numpy(), lse_ref.cpu().numpy(), atol=1e-4, rtol=0)
        assert torch.equal(caches[1].pos, caches[0].pos)
        assert torch.equal(caches[1].meta[:2], caches[0].meta[:2])


def test_noalloc_reports_device_check_failure():
    """A device-side check that fails inside the allocation-free step lands in
    the static array's error word, where lte_noalloc_read_device_error finds
    it; the next call starts from a clean word.  The failure is made on the
    host: the window slot of the token about to leave is given a wrong
    position tag, which the update's slot check reports (LTE_ERR_DEVICE, site
    201) and treats as a dropped token -- no access leaves the cache."""
    from learnable_kv_token_b200 import lte as L
    B, T0 = 2, 150
    s = _setup(B, 2, T0, 2718)
    c = s["caches"][1]
    w = c.window
    o = torch.empty(B, s["Hq"], s["D"], dtype=torch.bfloat16, device="cuda")
    t = T0                                          # token t - w leaves slot t mod w
    c.pos[1, 0, t % w] = 7 * w + 3                  # not the leaving token's position
    qt, kt, vt = (x[:, t].contiguous() for x in (s["q"], s["k"], s["v"]))
    L.lte_decode_step_noalloc(s["dims"], s["c_struct"], c.struct, qt, kt, vt, o, None, 4)
    assert L.lte_noalloc_read_device_error() == (6, 201)     # LTE_ERR_DEVICE at the slot check
    assert int(c.pos[1, 0, t % w]) == t             # the new token took the slot all the same
    qt, kt, vt = (x[:, t + 1].contiguous() for x in (s["q"], s["k"], s["v"]))
    L.lte_decode_step_noalloc(s["dims"], s["c_struct"], c.struct, qt, kt, vt, o, None, 4)
    assert L.lte_noalloc_read_device_error() == (0, 0)
    assert torch.isfinite(o.float()).all()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from learnable_kv_token_b200 import lte as L
    # 512 units x G = 16 heads x 2 partials per unit x 130 floats ~ 8.5 MB > 4 MiB
    dims = L.make_dims(64, 64, 128, 8, 128, 4, 512, 512, 0.5, 0.088, L.LTE_BF16)
    assert L.lte_workspace_bytes(dims, L.LTE_WS_DECODE) > 4 << 20
    cnn = L.lte_cnn(32, 5, 2, 3, 1, 16, 16, 16, 16)
    cache = L.lte_cache(16, 16, 16, 16, 16, 16)
    p = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(L.LteError) as ei:
        L.lte_decode_step_noalloc(dims, cnn, cache, p, p, p, p, None, 8)
    assert ei.value.status == 5     # LTE_ERR_WORKSPACE
