"""The C-ABI library loads without a GPU and exports every entry point that
include/lte_api.h declares; host-side argument validation rejects bad calls
before any launch (no device needed for those paths)."""
import ctypes as C
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lte_api.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lte_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    sys.path.insert(0, ROOT)
    from learnable_kv_token_b200 import build
    path = build.build()
    return C.CDLL(path), path


def test_header_declares_expected_entry_points():
    names = _declared()
    for n in ("lte_score", "lte_evict_compact", "lte_sparse_attn_prefill", "lte_decode_step",
              "lte_cache_init_from_prefill", "lte_workspace_bytes", "lte_gla_prefill",
              "lte_gla_decode_step", "lte_read_device_error", "lte_retained_lifetimes",
              "lte_sparse_attn_backward", "lte_score_backward"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    cdll, path = lib
    for name in _declared():
        assert hasattr(cdll, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (lte_\w+)", out))
    assert set(_declared()) <= exported


def test_binding_exposes_same_names(lib):
    from learnable_kv_token_b200 import lte
    for name in _declared():
        if name == "lte_version":
            continue
        assert hasattr(lte, name), name


def test_host_validation_without_gpu(lib):
    """Invalid calls return an error status before touching the device."""
    from learnable_kv_token_b200 import lte as L
    d = L.make_dims(1, 64, 4, 4, 64, 4, 16, 8, 0.5, 0.125, L.LTE_F32)
    f = L._lib
    # null pointers -> LTE_ERR_INVALID_ARG
    assert f.lte_evict_compact(C.byref(d), None, None, 64, None, None, None, None, None, None,
                               None, None, None) == 1
    bad = L.make_dims(1, 64, 6, 4, 64, 4, 16, 8, 0.5, 0.125, L.LTE_F32)   # Hq % Hkv != 0
    assert f.lte_workspace_bytes(C.byref(bad), 0) == 0
    pol = L.make_dims(1, 64, 4, 4, 64, 4, 16, 8, 0.5, 0.125, L.LTE_F32, cap_policy=3)  # no such policy
    assert f.lte_workspace_bytes(C.byref(pol), 0) == 0
    first = L.make_dims(1, 64, 4, 4, 64, 4, 16, 8, 0.5, 0.125, L.LTE_F32, L.LTE_CAP_FIRST)
    assert f.lte_workspace_bytes(C.byref(first), 0) >= 16
    d96 = L.make_dims(1, 64, 4, 4, 96, 4, 16, 8, 0.5, 0.1, L.LTE_F32)     # D not in {64,128}
    assert f.lte_sparse_attn_prefill(C.byref(d96), None, None, None, None, None, None, None, None,
                                     None, None, None, None, None, 0, None) == 2
    # LTE_CAP_LOWEST: lifetimes need that policy and all pointers; the attention
    # needs the lifetimes
    low = L.make_dims(1, 64, 4, 4, 64, 4, 16, 8, 0.5, 0.125, L.LTE_F32, L.LTE_CAP_LOWEST)
    p16 = C.c_void_p(16)
    assert f.lte_workspace_bytes(C.byref(low), 0) >= 16
    assert f.lte_retained_lifetimes(C.byref(d), p16, p16, p16, p16, None) == 1
    assert f.lte_retained_lifetimes(C.byref(low), p16, p16, None, p16, None) == 1
    assert f.lte_sparse_attn_prefill(C.byref(low), p16, p16, p16, None, None, p16, None, p16, p16,
                                     p16, None, None, p16, 1 << 20, None) == 1
    assert f.lte_workspace_bytes(C.byref(d), 0) >= 16
    assert f.lte_workspace_bytes(C.byref(d), 1) > 16
    # score: range beyond the receptive field -> invalid
    cnn = L.lte_cnn(32, 5, 2, 3, 1, 16, 16, 16, 16)
    assert f.lte_score(C.byref(d), C.byref(cnn), C.c_void_p(16), C.c_void_p(16), None, 0, 63,
                       C.c_void_p(16), None, None) == 1
    # decode: score batch larger than the window allows -> invalid
    dd = L.make_dims(1, 64, 4, 4, 64, 4, 16, 8, 0.5, 0.125, L.LTE_BF16)
    cache = L.lte_cache(16, 16, 16, 16, 16, 16)
    assert f.lte_decode_step(C.byref(dd), C.byref(cnn), C.byref(cache), C.c_void_p(16),
                             C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), None, 11,
                             C.c_void_p(16), 1 << 20, None) == 1
    # decode under LTE_CAP_LOWEST without the retained slots' scores -> invalid
    dl = L.make_dims(1, 64, 4, 4, 64, 4, 16, 8, 0.5, 0.125, L.LTE_BF16, L.LTE_CAP_LOWEST)
    assert f.lte_decode_step(C.byref(dl), C.byref(cnn), C.byref(cache), C.c_void_p(16),
                             C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), None, 4,
                             C.c_void_p(16), 1 << 20, None) == 1
    # backward: null pointers, fp32 (unsupported), lowest-score policy without
    # lifetimes, workspace too small
    bb = L.make_dims(1, 64, 4, 4, 128, 4, 16, 8, 0.5, 0.125, L.LTE_BF16)
    p = [C.c_void_p(16)] * 16                                 # 15 tensors and the workspace
    ws_need = f.lte_workspace_bytes(C.byref(bb), L.LTE_WS_BACKWARD)
    assert ws_need >= 16 + 4 * 64 * 4
    assert f.lte_sparse_attn_backward(C.byref(bb), *([None] * 16), 0, None) == 1
    assert f.lte_sparse_attn_backward(C.byref(bb), *p, ws_need - 16, None) == 5
    bf = L.make_dims(1, 64, 4, 4, 128, 4, 16, 8, 0.5, 0.125, L.LTE_F32)
    assert f.lte_sparse_attn_backward(C.byref(bf), *p, 1 << 20, None) == 2
    bl = L.make_dims(1, 64, 4, 4, 128, 4, 16, 8, 0.5, 0.125, L.LTE_BF16, L.LTE_CAP_LOWEST)
    pl = list(p)
    pl[4] = None                                              # death
    assert f.lte_sparse_attn_backward(C.byref(bl), *pl, 1 << 20, None) == 1
    # CNN backward: null pointers, n_scored past the receptive field, short workspace
    cb = L.make_dims(2, 64, 4, 4, 64, 4, 16, 8, 0.5, 0.125, L.LTE_BF16)
    cnn5 = L.lte_cnn(32, 5, 2, 3, 1, 16, 16, 16, 16)
    need = f.lte_score_backward_workspace_bytes(C.byref(cb), C.byref(cnn5))
    assert need >= 16 + 2 * 2 * 4 * 32 * 64 * 4
    q16 = [C.c_void_p(16)] * 8                                # dr, dk, dv, dw1, db1, dw2, db2, ws
    assert f.lte_score_backward(C.byref(cb), C.byref(cnn5), p16, p16, None, 61,
                                *([None] * 8), need, None) == 1
    assert f.lte_score_backward(C.byref(cb), C.byref(cnn5), p16, p16, None, 62, *q16, need,
                                None) == 1                     # T - F = 61
    assert f.lte_score_backward(C.byref(cb), C.byref(cnn5), p16, p16, None, 61, *q16, need - 16,
                                None) == 5
    # wait probe: null or misaligned flag, limit out of range, missing workspace
    assert f.lte_wait_probe(None, 1, 1000000, C.c_void_p(16), None) == 1
    assert f.lte_wait_probe(C.c_void_p(18), 1, 1000000, C.c_void_p(16), None) == 1
    assert f.lte_wait_probe(C.c_void_p(16), 1, 10, C.c_void_p(16), None) == 1
    assert f.lte_wait_probe(C.c_void_p(16), 1, 1000000, None, None) == 5
    assert L.version().startswith("lte-b200")


def test_kernel_choice_is_reported(lib):
    """lte_sparse_attn_prefill_kernel / lte_sparse_attn_backward_kernel say
    which kernel family the call runs, so a caller can see when a shape or a
    stride leaves the tcgen05 kernels (host only, no GPU needed)."""
    from learnable_kv_token_b200 import lte as L
    mk = lambda D, dt, Hq=16, Hkv=4: L.make_dims(2, 256, Hq, Hkv, D, 4, 64, 32, 0.5, 0.1, dt)
    assert L.lte_sparse_attn_prefill_kernel(mk(128, L.LTE_BF16)) == L.LTE_KERNEL_TCGEN05
    assert L.lte_sparse_attn_prefill_kernel(mk(64, L.LTE_BF16)) == L.LTE_KERNEL_MMA_SYNC
    assert L.lte_sparse_attn_prefill_kernel(mk(128, L.LTE_F32)) == L.LTE_KERNEL_SIMT
    # q rows spaced by 1032 elements (2064 bytes, a multiple of 16) stay on tcgen05;
    # an element stride of 8 per row but 8 + 4 per head is rejected as unaligned
    ok = L.lte_strides(256 * 16 * 1032, 16 * 1032, 1032)
    assert L.lte_sparse_attn_prefill_kernel(mk(128, L.LTE_BF16), ok, None, None) == \
        L.LTE_KERNEL_TCGEN05
    with pytest.raises(L.LteError) as ei:
        L.lte_sparse_attn_prefill_kernel(mk(128, L.LTE_BF16), L.lte_strides(8, 8, 12), None, None)
    assert ei.value.status == 1
    with pytest.raises(L.LteError) as ei:                    # G = 32 is not supported in bf16
        L.lte_sparse_attn_prefill_kernel(mk(128, L.LTE_BF16, Hq=32, Hkv=1))
    assert ei.value.status == 2
    assert L.lte_sparse_attn_backward_kernel(mk(128, L.LTE_BF16)) == L.LTE_KERNEL_TCGEN05
    assert L.lte_sparse_attn_backward_kernel(mk(64, L.LTE_BF16)) == L.LTE_KERNEL_MMA_SYNC
    with pytest.raises(L.LteError) as ei:
        L.lte_sparse_attn_backward_kernel(mk(128, L.LTE_F32))
    assert ei.value.status == 2
    f = L._lib
    assert f.lte_noalloc_read_device_error(None, None, None) == 1
    assert f.lte_sparse_attn_prefill_kernel(C.byref(mk(128, L.LTE_BF16)), None, None, None,
                                            None) == 1


def test_decode_cache_snapshot_restore_on_host(lib):
    """DecodeCache.snapshot / restore copy every tensor the decode step reads or
    writes and put them back in place (same buffers, so the cache struct a
    captured graph holds stays valid).  Host tensors, no GPU needed."""
    import torch
    from learnable_kv_token_b200 import layer
    c = layer.DecodeCache(2, 3, 16, torch.float32, sink=2, window=8, cap=4, device="cpu")
    g = torch.Generator().manual_seed(3)
    for t in c._state():
        if t.dtype.is_floating_point:
            t.copy_(torch.randn(t.shape, generator=g))
        else:
            t.copy_(torch.randint(-5, 50, t.shape, generator=g, dtype=t.dtype))
    ptrs = [t.data_ptr() for t in c._state()]
    snap = c.snapshot()
    before = [t.clone() for t in c._state()]
    assert all(s.data_ptr() != p for s, p in zip(snap, ptrs))      # copies, not views
    for t in c._state():
        t.fill_(7)
    c.restore(snap)
    assert [t.data_ptr() for t in c._state()] == ptrs
    for t, b in zip(c._state(), before):
        assert torch.equal(t, b)
    # the state covers the struct the library sees: every pointer it holds is one of them
    held = {c.struct.k, c.struct.v, c.struct.pos, c.struct.win_r, c.struct.ret_total,
            c.struct.meta, c.struct.ret_r}
    assert held == set(ptrs)
