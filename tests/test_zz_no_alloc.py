"""The allocation-free decode entry point (lte_decode_step_noalloc).

Some callers cannot allocate device memory -- a host runtime that keeps the
whole GPU in its own pool and gives a plugin only input and output buffers,
or a latency-critical loop that cannot afford the synchronisation a
cudaMalloc may imply.  For them the library keeps the decode step's scratch
in a fixed static device array instead of a caller workspace.  This test
calls that entry point through the C ABI and checks it against
lte_decode_step (same kernels, caller workspace) on two calls in a row, on
two caches set up identically.  The file name makes pytest collect it last.
"""
import numpy as np
import pytest
import torch

import lte_inputs as LI

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_variant():
    from learnable_kv_token_b200 import layer, lte as L
    B, Hq, Hkv, D, sink, window, cap, T0 = 2, 8, 2, 128, 4, 64, 16, 150
    g = LI.generator(314)
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
    ref = layer.Decoder(dims, cnn, p.past1, p.past2, caches[0], score_batch=4)
    c_struct, _keep = L.make_cnn(*cnn, p.past1, p.past2)
    o_na = torch.empty(B, Hq, D, dtype=torch.bfloat16, device="cuda")
    lse_na = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    for t in (T0, T0 + 1):                                   # two calls in a row
        qt, kt, vt = (x[:, t].contiguous() for x in (q, k, v))
        o_ref, lse_ref = ref.step(qt, kt, vt)
        L.lte_decode_step_noalloc(dims, c_struct, caches[1].struct, qt, kt, vt, o_na, lse_na, 4)
        torch.cuda.synchronize()
        np.testing.assert_allclose(o_na.float().cpu().numpy(), o_ref.float().cpu().numpy(),
                                   atol=2e-2, rtol=0)
        np.testing.assert_allclose(lse_na.cpu().numpy(), lse_ref.cpu().numpy(), atol=1e-4, rtol=0)
        assert torch.equal(caches[1].pos, caches[0].pos)
        assert torch.equal(caches[1].meta[:2], caches[0].meta[:2])


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
