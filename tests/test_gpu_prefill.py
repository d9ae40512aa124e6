"""GPU parity of the prefill path through the C ABI: scoring CNN, eviction /
compaction, sparse attention, against the CPU oracle on identical seeded
inputs."""
import math

import numpy as np
import pytest
import torch

import lte_inputs as LI
from oracle import lte_oracle as O
from tests.gpu_util import (MASK_BAND, R_TOL, assert_attention_close, clean_tau, f64, fed_masks,
                            oracle_cnn, oracle_rows, scale_of)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from learnable_kv_token_b200 import lte
    return lte


@pytest.fixture(scope="module")
def layer():
    from learnable_kv_token_b200 import layer
    return layer


def _dev(*ts):
    return [t.cuda() for t in ts]


# --------------------------------------------------------------------------- scores
@pytest.mark.parametrize("wl_name,T,dtype", [("tiny", 512, torch.float32),
                                             ("decode", 700, torch.bfloat16)])
def test_score_parity(L, wl_name, T, dtype):
    wl = LI.WORKLOADS[wl_name]
    g = LI.generator(wl.seed)
    _, k, v = LI.qkv(1 if wl_name == "decode" else wl.B, T, wl.Hq, wl.Hkv, wl.D, dtype, g)
    cnn = LI.cnn_weights(wl.Hkv, wl.D, wl.c_hid, wl.k1, wl.k2, g, wl.w_std)
    B = k.shape[0]
    kd, vd = _dev(k, v)
    cd = _dev(*cnn)
    dims = L.make_dims(B, T, wl.Hq, wl.Hkv, wl.D, wl.sink, wl.window, wl.cap, wl.tau, wl.scale, dtype)
    c, _keep = L.make_cnn(*cd, wl.past1, wl.past2)
    F = 3
    r = torch.full((B, wl.Hkv, T), float("nan"), device="cuda")
    m = torch.zeros(B, wl.Hkv, T, dtype=torch.uint8, device="cuda")
    L.lte_score(dims, c, kd, vd, 0, T - F, r, m)
    # split launch: same values bit for bit
    r2 = torch.full_like(r, float("nan"))
    L.lte_score(dims, c, kd, vd, 0, 97, r2)
    L.lte_score(dims, c, kd, vd, 97, T - F, r2)
    torch.cuda.synchronize()
    assert torch.equal(r[..., :T - F], r2[..., :T - F])
    assert torch.isnan(r[..., T - F:]).all()
    band = 0
    for b in range(B):
        for h in range(wl.Hkv):
            ro = O.cnn_scores(f64(k[b, :, h]), f64(v[b, :, h]), oracle_cnn(cnn, h))
            rg = f64(r[b, h])
            np.testing.assert_allclose(rg[:T - F], ro[:T - F], atol=R_TOL, rtol=0)
            mo = O.retention_mask(ro, wl.sink, wl.tau)
            clear = np.abs(ro[:T - F] - wl.tau) > MASK_BAND
            band += int((~clear).sum())
            np.testing.assert_array_equal(m[b, h].cpu().numpy()[:T - F][clear], mo[:T - F][clear])
    print(f"scores within {R_TOL}; {band} tokens in the +-{MASK_BAND} band")


def test_score_causal_variant(L):
    """past1 = k1-1, past2 = k2-1: a CNN that reads the past only."""
    g = LI.generator(11)
    B, T, H, D = 2, 300, 2, 64
    _, k, v = LI.qkv(B, T, H, H, D, torch.float32, g)
    cnn = LI.cnn_weights(H, D, 16, 5, 3, g, 0.05)
    kd, vd = _dev(k, v)
    cd = _dev(*cnn)
    dims = L.make_dims(B, T, H, H, D, 2, 32, 8, 0.5, 0.125, torch.float32)
    c, _k = L.make_cnn(*cd, 4, 2)
    r = torch.full((B, H, T), float("nan"), device="cuda")
    L.lte_score(dims, c, kd, vd, 0, T, r, None)
    for b in range(B):
        for h in range(H):
            ro = O.cnn_scores(f64(k[b, :, h]), f64(v[b, :, h]), oracle_cnn(cnn, h, 4, 2))
            np.testing.assert_allclose(f64(r[b, h]), ro, atol=R_TOL, rtol=0)


@pytest.mark.parametrize("B,T,Hkv,D,c_hid,past1,past2,k1,k2", [
    (3, 1500, 2, 64, 32, 2, 1, 5, 3),     # head dim 64, several sequences and heads
    (2, 1000, 4, 128, 20, 4, 2, 5, 3),    # fewer hidden channels than columns per tap; causal taps
    (1, 40, 1, 128, 32, 2, 1, 5, 3),      # a sequence shorter than one tile (one CTA of the pair idle)
    (2, 700, 2, 128, 32, 4, 1, 8, 3),     # the widest first layer: 256 output columns
    (3, 900, 3, 64, 16, 1, 2, 3, 5),      # a narrow first layer, a wide second, an odd tile count
])
def test_score_tensor_core_shapes(L, B, T, Hkv, D, c_hid, past1, past2, k1, k2):
    """bf16 scores from the tcgen05 scorer, with k and v strided views into one
    packed [B, T, Hkv, 2, D] tensor, against the oracle; a split launch gives
    the same values bit for bit."""
    g = LI.generator(23)
    kv = (torch.randn(B, T, Hkv, 2, D, generator=g) / math.sqrt(D)).to(torch.bfloat16)
    k, v = kv[:, :, :, 0], kv[:, :, :, 1]
    w1, _, w2, _ = LI.cnn_weights(Hkv, D, c_hid, k1, k2, g, 0.05)
    cnn = (w1, 0.1 * torch.randn(Hkv, c_hid, generator=g), w2, 0.1 * torch.randn(Hkv, generator=g))
    kvd = kv.cuda()
    kd, vd = kvd[:, :, :, 0], kvd[:, :, :, 1]
    cd = _dev(*cnn)
    dims = L.make_dims(B, T, Hkv, Hkv, D, 4, 64, 32, 0.5, 1.0 / math.sqrt(D), torch.bfloat16)
    c, _keep = L.make_cnn(*cd, past1, past2)
    F = (k1 - 1 - past1) + (k2 - 1 - past2)
    n = T - F
    r = torch.full((B, Hkv, T), float("nan"), device="cuda")
    m = torch.zeros(B, Hkv, T, dtype=torch.uint8, device="cuda")
    L.lte_score(dims, c, kd, vd, 0, n, r, m)
    cut = min(n, 233)
    r2 = torch.full_like(r, float("nan"))
    L.lte_score(dims, c, kd, vd, 0, cut, r2)
    L.lte_score(dims, c, kd, vd, cut, n, r2)
    torch.cuda.synchronize()
    assert torch.equal(r[..., :n], r2[..., :n])
    assert torch.isnan(r[..., n:]).all()
    for b in range(B):
        for h in range(Hkv):
            ro = O.cnn_scores(f64(k[b, :, h]), f64(v[b, :, h]), oracle_cnn(cnn, h, past1, past2))
            np.testing.assert_allclose(f64(r[b, h])[:n], ro[:n], atol=R_TOL, rtol=0)
            clear = np.abs(ro[:n] - 0.5) > MASK_BAND
            mo = O.retention_mask(ro, 4, 0.5)
            np.testing.assert_array_equal(m[b, h].cpu().numpy()[:n][clear], mo[:n][clear])


# --------------------------------------------------------------------------- compaction
@pytest.mark.parametrize("T,sink,p,n_scored", [(1000, 4, 0.1, 1000), (3001, 0, 0.5, 2990),
                                               (77, 4, 1.0, 77), (64, 2, 0.0, 64), (3, 4, 1.0, 3),
                                               (4100, 7, 0.03, 4000)])
def test_compact_parity(L, T, sink, p, n_scored):
    g = LI.generator(5)
    B, H, D = 2, 3, 128
    _, k, v = LI.qkv(B, T, H, H, D, torch.bfloat16, g)
    mask = LI.bernoulli_mask(B, H, T, p, g)
    kd, vd, md = _dev(k, v, mask)
    dims = L.make_dims(B, T, H, H, D, sink, 16, 8, 0.5, 0.1, torch.bfloat16)
    idx = torch.full((B, H, T), -7, dtype=torch.int32, device="cuda")
    nret = torch.empty(B, H, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, H, T, dtype=torch.int32, device="cuda")
    kc = torch.zeros(B, H, sink + T, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    L.lte_evict_compact(dims, None, md, n_scored, idx, nret, cnt, kd, vd, kc, vc)
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(H):
            m = fed_masks(mask, sink)[b, h].copy()
            m[n_scored:] = 0
            ix, n, cn = O.compact(m)
            assert int(nret[b, h]) == n
            np.testing.assert_array_equal(idx[b, h, :n].cpu().numpy(), ix)
            np.testing.assert_array_equal(cnt[b, h].cpu().numpy(), cn)
            ns = min(sink, T)
            assert torch.equal(kc[b, h, :ns].cpu(), k[b, :ns, h])
            assert torch.equal(kc[b, h, sink:sink + n].cpu(), k[b, ix, h])
            assert torch.equal(vc[b, h, sink:sink + n].cpu(), v[b, ix, h])


def test_compact_from_scores(L):
    """r input path: m_j = j >= s and j < n_scored and r_j >= tau."""
    B, H, T, s, tau = 1, 2, 500, 3, 0.4
    r = torch.rand(B, H, T, generator=LI.generator(3), dtype=torch.float32)
    dims = L.make_dims(B, T, H, H, 64, s, 16, 8, tau, 0.1, torch.float32)
    idx = torch.empty(B, H, T, dtype=torch.int32, device="cuda")
    nret = torch.empty(B, H, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, H, T, dtype=torch.int32, device="cuda")
    L.lte_evict_compact(dims, r.cuda(), None, 480, idx, nret, cnt)
    for h in range(H):
        rr = f64(r[0, h]).copy()
        rr[480:] = np.nan
        ix, n, cn = O.compact(O.retention_mask(rr, s, tau))
        assert int(nret[0, h]) == n
        np.testing.assert_array_equal(idx[0, h, :n].cpu().numpy(), ix)
        np.testing.assert_array_equal(cnt[0, h].cpu().numpy(), cn)


# --------------------------------------------------------------------------- attention
def _run_prefill(layer, q, k, v, mask, sink, window, cap, scale=None, cap_policy=0):
    p = layer.LayerParams(sink=sink, window=window, cap=cap, scale=scale, cap_policy=cap_policy)
    qd, kd, vd, md = _dev(q, k, v, mask)
    out = layer.prefill(qd, kd, vd, p, mask=md)
    torch.cuda.synchronize()
    return out


CASES = [
    # B, T, Hq, Hkv, D, dtype, sink, window, cap, rate
    (1, 512, 4, 4, 64, torch.float32, 4, 64, 32, 0.3),
    (2, 1100, 8, 2, 128, torch.bfloat16, 4, 128, 64, 0.1),
    (1, 777, 16, 4, 128, torch.bfloat16, 4, 100, 500, 0.4),
    (2, 333, 4, 1, 64, torch.bfloat16, 2, 37, 5, 0.5),
    (1, 260, 8, 8, 128, torch.bfloat16, 0, 16, 3, 0.7),
    (1, 300, 16, 2, 64, torch.bfloat16, 5, 50, 0, 0.6),
    (1, 400, 2, 2, 128, torch.float32, 3, 20, 7, 0.5),
]


@pytest.mark.parametrize("case", CASES)
def test_prefill_fed_mask_parity(layer, case):
    B, T, Hq, Hkv, D, dtype, sink, window, cap, rate = case
    g = LI.generator(100 + T)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, dtype, g)
    mask = LI.bernoulli_mask(B, Hkv, T, rate, g)
    out = _run_prefill(layer, q, k, v, mask, sink, window, cap)
    masks = fed_masks(mask, sink)
    G = Hq // Hkv
    rows = list(range(T))
    for b in range(B):
        for h in range(Hkv):
            o_ref, lse_ref, _ = oracle_rows(q, k, v, masks, b, h, rows, sink, window, cap, scale_of(D))
            o_g = f64(out.o[b, :, h * G:(h + 1) * G])
            lse_g = f64(out.lse[b, h * G:(h + 1) * G]).T
            assert_attention_close(o_g, lse_g, o_ref, lse_ref, dtype, f"unit {b},{h}")


FIRST_CASES = [
    # B, T, Hq, Hkv, D, dtype, sink, window, cap, rate: the cap binds early
    (2, 1100, 8, 2, 128, torch.bfloat16, 4, 128, 24, 0.3),     # tcgen05 kernel
    (2, 333, 4, 1, 64, torch.bfloat16, 2, 37, 5, 0.5),         # warp-MMA kernel (head dim 64)
    (1, 400, 2, 2, 128, torch.float32, 3, 20, 7, 0.5),         # fp32 kernel
    (1, 700, 16, 4, 128, torch.bfloat16, 4, 64, 300, 0.2),     # the cap never binds
]


@pytest.mark.parametrize("case", FIRST_CASES)
def test_prefill_cap_first_policy(layer, case):
    """LTE_CAP_FIRST: rows attend to the first C retained tokens instead of the
    C most recent, in every prefill kernel, against the oracle's policy "first"."""
    from learnable_kv_token_b200 import lte as L
    B, T, Hq, Hkv, D, dtype, sink, window, cap, rate = case
    g = LI.generator(300 + T)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, dtype, g)
    mask = LI.bernoulli_mask(B, Hkv, T, rate, g)
    out = _run_prefill(layer, q, k, v, mask, sink, window, cap, cap_policy=L.LTE_CAP_FIRST)
    masks = fed_masks(mask, sink)
    G = Hq // Hkv
    rows = list(range(T))
    for b in range(B):
        for h in range(Hkv):
            o_ref, lse_ref, _ = oracle_rows(q, k, v, masks, b, h, rows, sink, window, cap,
                                            scale_of(D), policy=O.CAP_FIRST)
            o_g = f64(out.o[b, :, h * G:(h + 1) * G])
            lse_g = f64(out.lse[b, h * G:(h + 1) * G]).T
            assert_attention_close(o_g, lse_g, o_ref, lse_ref, dtype, f"unit {b},{h}")


@pytest.mark.parametrize("case", [
    # B, T, Hq, Hkv, D, dtype, sink, window, cap, rate
    (1, 300, 8, 2, 128, torch.bfloat16, 0, 16, 3, 0.7),      # tcgen05 kernel, no sink
    (1, 300, 8, 8, 128, torch.bfloat16, 0, 16, 3, 0.7),      # tcgen05 kernel, G = 1
    (1, 20, 4, 1, 128, torch.bfloat16, 40, 8, 4, 0.5),       # more sink slots than tokens
    (1, 333, 4, 1, 64, torch.bfloat16, 2, 37, 5, 0.5),       # warp-MMA kernel
])
def test_prefill_stale_column_segment(layer, case):
    """The column segment's buffers start as NaN (stale memory): compaction
    writes the rows past the retained ones that a 64-row tile can reach, so the
    output is still finite and equal to the oracle's."""
    B, T, Hq, Hkv, D, dtype, sink, window, cap, rate = case
    g = LI.generator(600 + T)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, dtype, g)
    mask = LI.bernoulli_mask(B, Hkv, T, rate, g)
    p = layer.LayerParams(sink=sink, window=window, cap=cap)
    qd, kd, vd, md = _dev(q, k, v, mask)
    dims = p.dims(B, T, Hq, Hkv, D, dtype)
    bufs = layer.PrefillBuffers(B, T, Hq, Hkv, D, dtype, sink, dims, "cuda", want_r=False)
    bufs.k_col.fill_(float("nan"))
    bufs.v_col.fill_(float("nan"))
    out = layer.prefill(qd, kd, vd, p, mask=md, bufs=bufs)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out.o.float()).all()) and bool(torch.isfinite(out.lse).all())
    masks = fed_masks(mask, sink)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hkv):
            o_ref, lse_ref, _ = oracle_rows(q, k, v, masks, b, h, list(range(T)), sink, window, cap,
                                            scale_of(D))
            assert_attention_close(f64(out.o[b, :, h * G:(h + 1) * G]),
                                   f64(out.lse[b, h * G:(h + 1) * G]).T, o_ref, lse_ref, dtype,
                                   f"unit {b},{h}")


LOWEST_CASES = [
    # B, T, Hq, Hkv, D, dtype, sink, window, cap, score levels (few levels: many equal scores)
    (2, 1100, 8, 2, 128, torch.bfloat16, 4, 128, 24, 1024),   # tcgen05 kernel
    (1, 900, 16, 4, 128, torch.bfloat16, 4, 64, 40, 8),       # tcgen05 kernel, G = 4, ties
    (2, 333, 4, 1, 64, torch.bfloat16, 2, 37, 5, 16),         # warp-MMA kernel (head dim 64)
    (1, 400, 2, 2, 128, torch.float32, 3, 20, 7, 256),        # fp32 kernel
    (1, 700, 16, 4, 128, torch.bfloat16, 4, 64, 300, 64),     # the cap binds late
    (1, 300, 8, 2, 128, torch.bfloat16, 2, 30, 0, 64),        # cap 0
]


def _run_prefill_scores(layer, q, k, v, r, sink, window, cap, cap_policy):
    p = layer.LayerParams(sink=sink, window=window, cap=cap, tau=0.5, cap_policy=cap_policy)
    qd, kd, vd, rd = _dev(q, k, v, r)
    out = layer.prefill(qd, kd, vd, p, scores=rd)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("case", LOWEST_CASES)
def test_prefill_cap_lowest_policy(layer, case):
    """LTE_CAP_LOWEST: each row attends to the C retained tokens with the
    highest (score, position) among those that left the window, in every
    prefill kernel, against the oracle's policy "lowest".  The scores are fed
    (exact in fp32, so both sides rank the same values)."""
    from learnable_kv_token_b200 import lte as L
    B, T, Hq, Hkv, D, dtype, sink, window, cap, levels = case
    g = LI.generator(400 + T)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, dtype, g)
    r = LI.grid_scores(B, Hkv, T, levels, g)
    out = _run_prefill_scores(layer, q, k, v, r, sink, window, cap, L.LTE_CAP_LOWEST)
    masks = np.stack([[O.retention_mask(f64(r[b, h]), sink, 0.5) for h in range(Hkv)]
                      for b in range(B)])
    G = Hq // Hkv
    rows = list(range(T))
    for b in range(B):
        for h in range(Hkv):
            o_ref, lse_ref, _ = oracle_rows(q, k, v, masks, b, h, rows, sink, window, cap,
                                            scale_of(D), policy=O.CAP_LOWEST, r=r)
            o_g = f64(out.o[b, :, h * G:(h + 1) * G])
            lse_g = f64(out.lse[b, h * G:(h + 1) * G]).T
            assert_attention_close(o_g, lse_g, o_ref, lse_ref, dtype, f"unit {b},{h}")


@pytest.mark.parametrize("levels,cap", [(8, 6), (1024, 6), (4, 1), (64, 0), (64, 500)])
def test_retained_lifetimes_vs_oracle(layer, levels, cap):
    """lte_retained_lifetimes, exactly: for every retained count n, the ordinals
    i < n with death[i] > n are the oracle's C best of the first n retained
    tokens (and the compacted list equals the oracle's)."""
    from learnable_kv_token_b200 import lte as L
    B, T, Hq, Hkv, D, sink, window = 2, 700, 4, 2, 64, 3, 16
    g = LI.generator(500 + levels + cap)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, torch.bfloat16, g)
    r = LI.grid_scores(B, Hkv, T, levels, g)
    out = _run_prefill_scores(layer, q, k, v, r, sink, window, cap, L.LTE_CAP_LOWEST)
    idx, nret, death = out.idx.cpu().numpy(), out.nret.cpu().numpy(), out.death.cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            rr = f64(r[b, h])
            cand, n_all, _ = O.compact(O.retention_mask(rr, sink, 0.5))
            assert int(nret[b, h]) == n_all
            np.testing.assert_array_equal(idx[b, h, :n_all], cand)
            d = death[b, h, :n_all]
            assert (d > np.arange(n_all)).all() and (d <= T + 1).all()
            for n in range(n_all + 1):
                held = [i for i in range(n) if d[i] > n]
                best = set(O.top_by_score(list(cand[:n]), rr, cap))
                assert held == [i for i in range(n) if cand[i] in best], (b, h, n)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("special", ["window_covers_all", "retain_none", "retain_all", "cap_zero"])
def test_prefill_special_cases(layer, dtype, special):
    """Degenerate settings reduce to textbook attention (checked against
    torch SDPA in float64 on CPU): full causal or sink + sliding window."""
    B, T, Hq, Hkv, D = 1, 300, 8, 2, 64 if dtype == torch.float32 else 128
    sink, window = 4, 40
    g = LI.generator(7)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, dtype, g)
    mask = LI.bernoulli_mask(B, Hkv, T, 0.5, g)
    cap = 8
    if special == "window_covers_all":
        window = T
    elif special == "retain_none":
        mask = torch.zeros_like(mask)
    elif special == "retain_all":
        mask = torch.ones_like(mask)
        cap = T
    elif special == "cap_zero":
        cap = 0
    out = _run_prefill(layer, q, k, v, mask, sink, window, cap)
    # reference: SDPA with the closed-form mask
    t = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    if special in ("window_covers_all", "retain_all"):
        allowed = j <= t
    else:
        allowed = (j <= t) & ((j > t - window) | (j < sink))
    G = Hq // Hkv
    qh = q.double().permute(0, 2, 1, 3)
    kh = k.double().permute(0, 2, 1, 3).repeat_interleave(G, 1)
    vh = v.double().permute(0, 2, 1, 3).repeat_interleave(G, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(qh, kh, vh, attn_mask=allowed,
                                                           scale=scale_of(D))
    logits = (qh @ kh.transpose(-1, -2)) * scale_of(D)
    lse_ref = torch.logsumexp(logits.masked_fill(~allowed, -math.inf), -1)
    assert_attention_close(f64(out.o), f64(out.lse), ref.permute(0, 2, 1, 3).numpy(),
                           lse_ref.numpy(), dtype, special)


def test_prefill_probe_peaked_positional(layer):
    """Peaked softmax (q x16) and values that encode their position: a wrong
    or missing key shows directly in the output."""
    B, T, Hq, Hkv, D = 1, 700, 8, 2, 128
    sink, window, cap = 4, 96, 40
    g = LI.generator(21)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, torch.float32, g)
    q = (q * 16).to(torch.bfloat16)
    k = k.to(torch.bfloat16)
    pos = torch.arange(T, dtype=torch.float64)[:, None]
    omega = torch.linspace(0.001, 0.5, D, dtype=torch.float64)[None, :]
    v = torch.cos(pos * omega)[None, :, None, :].expand(B, T, Hkv, D).to(torch.bfloat16).contiguous()
    mask = LI.bernoulli_mask(B, Hkv, T, 0.2, g)
    out = _run_prefill(layer, q, k, v, mask, sink, window, cap)
    masks = fed_masks(mask, sink)
    G = Hq // Hkv
    for h in range(Hkv):
        o_ref, lse_ref, _ = oracle_rows(q, k, v, masks, 0, h, list(range(T)), sink, window, cap,
                                        scale_of(D))
        assert_attention_close(f64(out.o[0, :, h * G:(h + 1) * G]),
                               f64(out.lse[0, h * G:(h + 1) * G]).T, o_ref, lse_ref,
                               torch.bfloat16, "probe")


def test_pipeline_with_cnn_tiny_workload(L, layer):
    """The small fp32 workload end to end on the GPU (score -> compact ->
    attend), with tau placed where no oracle score is within rounding of it,
    so the GPU's mask must equal the oracle's exactly."""
    wl = LI.WORKLOADS["tiny"]
    inp = LI.lte_inputs(wl, T=wl.T)
    q, k, v = inp["q"], inp["k"], inp["v"]
    cnn = inp["cnn"]
    r_or = np.stack([O.cnn_scores(f64(k[0, :, h]), f64(v[0, :, h]), oracle_cnn(cnn, h))
                     for h in range(wl.Hkv)])
    tau, margin = clean_tau(r_or)
    # the GPU scores are within R_TOL of the oracle's (checked below), so a
    # margin above R_TOL puts every token on the same side of tau on both
    assert margin > R_TOL, margin
    p = layer.LayerParams(sink=wl.sink, window=wl.window, cap=wl.cap, tau=tau)
    qd, kd, vd = _dev(q, k, v)
    out = layer.prefill(qd, kd, vd, p, cnn=_dev(*cnn))
    torch.cuda.synchronize()
    F = 3
    r_err = np.nanmax(np.abs(f64(out.r[0, :, :wl.T - F]) - r_or[:, :wl.T - F]))
    assert r_err <= R_TOL, r_err
    for h in range(wl.Hkv):
        m_or = O.retention_mask(r_or[h], wl.sink, tau)
        np.testing.assert_array_equal(out.mask[0, h].cpu().numpy(), m_or)
        ix, n, cn = O.compact(m_or)
        assert int(out.nret[0, h]) == n
        np.testing.assert_array_equal(out.cnt[0, h].cpu().numpy(), cn)
        o_ref, lse_ref, _ = O.prefill_unit(f64(q[0, :, h:h + 1]), f64(k[0, :, h]), f64(v[0, :, h]),
                                           m_or, wl.sink, wl.window, wl.cap, wl.scale)
        assert_attention_close(f64(out.o[0, :, h:h + 1]), f64(out.lse[0, h:h + 1]).T, o_ref,
                               lse_ref, torch.float32, f"head {h}")
    assert np.isnan(f64(out.r[0, :, wl.T - F:])).all()


def test_device_error_word_clean(L, layer):
    B, T, Hq, Hkv, D = 1, 200, 4, 1, 128
    g = LI.generator(1)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, torch.bfloat16, g)
    mask = LI.bernoulli_mask(B, Hkv, T, 0.3, g)
    p = layer.LayerParams(sink=4, window=32, cap=16)
    qd, kd, vd, md = _dev(q, k, v, mask)
    out_bufs = None
    dims = p.dims(B, T, Hq, Hkv, D, torch.bfloat16)
    bufs = layer.PrefillBuffers(B, T, Hq, Hkv, D, torch.bfloat16, 4, dims, want_r=False)
    L.lte_clear_device_error(bufs.ws)
    layer.prefill(qd, kd, vd, p, mask=md, bufs=bufs)
    assert L.lte_read_device_error(bufs.ws) == (0, 0)
    del out_bufs


def test_prefill_repeatable_long_items(layer):
    """The tcgen05 prefill kernel gives bit-identical o and lse on repeated
    launches over items with many key tiles (w = 1024, 16 retained-segment
    tiles): the roles that hand work on at item boundaries (next Q rows into
    TMEM, l and the max to the epilogue) wait on one phase per item, so a
    role that runs ahead cannot pass on an older phase.  A race there shows
    as launch-to-launch differences; the first launch is also checked
    against the oracle on sampled rows."""
    B, T, Hq, Hkv, D, s, w, C = 4, 4096, 16, 4, 128, 4, 1024, 1024
    g = LI.generator(77)
    q, k, v = LI.qkv(B, T, Hq, Hkv, D, torch.bfloat16, g)
    mask = LI.bernoulli_mask(B, Hkv, T, 0.4, g)
    p = layer.LayerParams(sink=s, window=w, cap=C)
    qd, kd, vd, md = q.cuda(), k.cuda(), v.cuda(), mask.cuda()
    outs = []
    for _ in range(3):
        out = layer.prefill(qd, kd, vd, p, mask=md)
        torch.cuda.synchronize()
        outs.append((out.o.clone(), out.lse.clone()))
    for o, lse in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(lse, outs[0][1])
    masks = fed_masks(mask, s)
    rows = [0, w - 1, w, w + 5, 2 * w + 17, T // 2, T - 1]
    for b, h in [(0, 0), (3, 2)]:
        o_ref, lse_ref, _ = oracle_rows(q, k, v, masks, b, h, rows, s, w, C, scale_of(D))
        G = Hq // Hkv
        assert_attention_close(f64(outs[0][0][b, rows, h * G:(h + 1) * G]),
                               f64(outs[0][1][b, h * G:(h + 1) * G][:, rows]).T, o_ref, lse_ref,
                               torch.bfloat16, f"unit {b},{h}")
