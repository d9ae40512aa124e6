"""Python binding of the LTE C ABI (include/lte_api.h).

Argument marshalling only: every function here turns torch tensors into
device pointers, calls the entry point of the same name in liblte.so, and
raises LteError on a non-zero status.  All arithmetic runs in the library's
CUDA kernels; torch only provides device memory and streams.  There is no
fallback: if liblte.so cannot be loaded, importing this module fails.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblte.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m learnable_kv_token_b200.build`")
_lib = C.CDLL(LIB_PATH)

LTE_F32, LTE_BF16 = 0, 1
LTE_CAP_RECENT, LTE_CAP_FIRST, LTE_CAP_LOWEST = 0, 1, 2
LTE_WS_PREFILL, LTE_WS_DECODE, LTE_WS_BACKWARD, LTE_WS_RELAXED = 0, 1, 2, 3
LTE_KERNEL_TCGEN05, LTE_KERNEL_MMA_SYNC, LTE_KERNEL_SIMT = 1, 2, 3
STATUS = {0: "LTE_OK", 1: "LTE_ERR_INVALID_ARG", 2: "LTE_ERR_UNSUPPORTED", 3: "LTE_ERR_CUDA",
          4: "LTE_ERR_TIMEOUT", 5: "LTE_ERR_WORKSPACE", 6: "LTE_ERR_DEVICE"}


class LteError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


class lte_dims(C.Structure):
    _fields_ = [("B", C.c_int32), ("T", C.c_int32), ("Hq", C.c_int32), ("Hkv", C.c_int32),
                ("D", C.c_int32), ("sink", C.c_int32), ("window", C.c_int32), ("cap", C.c_int32),
                ("tau", C.c_float), ("scale", C.c_float), ("dtype", C.c_int32),
                ("cap_policy", C.c_int32)]


class lte_strides(C.Structure):
    _fields_ = [("b", C.c_int64), ("t", C.c_int64), ("h", C.c_int64)]


class lte_cnn(C.Structure):
    _fields_ = [("c_hid", C.c_int32), ("k1", C.c_int32), ("past1", C.c_int32), ("k2", C.c_int32),
                ("past2", C.c_int32), ("w1", C.c_void_p), ("b1", C.c_void_p), ("w2", C.c_void_p),
                ("b2", C.c_void_p)]


class lte_cache(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("pos", C.c_void_p), ("win_r", C.c_void_p),
                ("ret_total", C.c_void_p), ("meta", C.c_void_p), ("ret_r", C.c_void_p)]


_P = C.c_void_p
_I = C.c_int32
_SIG = {
    "lte_score": [C.POINTER(lte_dims), C.POINTER(lte_cnn), _P, _P, C.POINTER(lte_strides), _I, _I,
                  _P, _P, _P],
    "lte_evict_compact": [C.POINTER(lte_dims), _P, _P, _I, _P, _P, _P, _P, _P,
                          C.POINTER(lte_strides), _P, _P, _P],
    "lte_retained_lifetimes": [C.POINTER(lte_dims), _P, _P, _P, _P, _P],
    "lte_sparse_attn_prefill": [C.POINTER(lte_dims), _P, _P, _P, C.POINTER(lte_strides),
                                C.POINTER(lte_strides), _P, _P, _P, _P, _P,
                                C.POINTER(lte_strides), _P, _P, C.c_size_t, _P],
    "lte_sparse_attn_backward": [C.POINTER(lte_dims)] + [_P] * 16 + [C.c_size_t, _P],
    "lte_sparse_attn_prefill_relaxed": [C.POINTER(lte_dims)] + [_P] * 13 + [C.c_size_t, _P],
    "lte_sparse_attn_backward_relaxed": [C.POINTER(lte_dims)] + [_P] * 18 + [C.c_size_t, _P],
    "lte_score_backward": [C.POINTER(lte_dims), C.POINTER(lte_cnn), _P, _P, C.POINTER(lte_strides),
                           _I] + [_P] * 8 + [C.c_size_t, _P],
    "lte_cache_init_from_prefill": [C.POINTER(lte_dims), C.POINTER(lte_cache), _P, _P,
                                    C.POINTER(lte_strides), _P, _P, _P, _P, _I, _I, _P],
    "lte_decode_step": [C.POINTER(lte_dims), C.POINTER(lte_cnn), C.POINTER(lte_cache), _P, _P, _P,
                        _P, _P, _I, _P, C.c_size_t, _P],
    "lte_decode_step_noalloc": [C.POINTER(lte_dims), C.POINTER(lte_cnn), C.POINTER(lte_cache), _P,
                                _P, _P, _P, _P, _I, _P],
    "lte_noalloc_read_device_error": [C.POINTER(C.c_int32), C.POINTER(C.c_int32), _P],
    "lte_sparse_attn_prefill_kernel": [C.POINTER(lte_dims), C.POINTER(lte_strides),
                                       C.POINTER(lte_strides), C.POINTER(lte_strides),
                                       C.POINTER(C.c_int32)],
    "lte_sparse_attn_backward_kernel": [C.POINTER(lte_dims), C.POINTER(C.c_int32)],
    "lte_clear_device_error": [_P, _P],
    "lte_read_device_error": [_P, C.POINTER(C.c_int32), C.POINTER(C.c_int32), _P],
    "lte_wait_probe": [_P, _I, C.c_int64, _P, _P],
    "lte_gla_prefill": [_I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P],
    "lte_gla_decode_step": [_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P],
}
for _name, _args in _SIG.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = C.c_int
_lib.lte_workspace_bytes.argtypes = [C.POINTER(lte_dims), _I]
_lib.lte_workspace_bytes.restype = C.c_size_t
_lib.lte_score_backward_workspace_bytes.argtypes = [C.POINTER(lte_dims), C.POINTER(lte_cnn)]
_lib.lte_score_backward_workspace_bytes.restype = C.c_size_t
_lib.lte_version.argtypes = []
_lib.lte_version.restype = C.c_char_p

EXPORTED = tuple(_SIG) + ("lte_workspace_bytes", "lte_score_backward_workspace_bytes", "lte_version")


def _call(name, *args):
    st = getattr(_lib, name)(*args)
    if st != 0:
        raise LteError(name, st)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _strides(t):
    """lte_strides of a [B,T,H,D] tensor (D stride must be 1)."""
    if t.stride(3) != 1:
        raise ValueError("innermost stride must be 1")
    return lte_strides(t.stride(0), t.stride(1), t.stride(2))


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return LTE_BF16
    if dt == torch.float32:
        return LTE_F32
    raise ValueError(f"unsupported dtype {dt}")


def make_dims(B, T, Hq, Hkv, D, sink, window, cap, tau, scale, dtype,
              cap_policy=LTE_CAP_RECENT) -> lte_dims:
    return lte_dims(B, T, Hq, Hkv, D, sink, window, cap, float(tau), float(scale),
                    dtype_code(dtype) if isinstance(dtype, torch.dtype) else int(dtype),
                    int(cap_policy))


def make_cnn(w1, b1, w2, b2, past1, past2) -> tuple[lte_cnn, tuple]:
    """lte_cnn over device tensors w1 [Hkv,c,2D,k1], b1 [Hkv,c], w2 [Hkv,c,k2], b2 [Hkv]
    (fp32, contiguous).  Returns the struct and the tensors it points into."""
    keep = tuple(x.contiguous().float() for x in (w1, b1, w2, b2))
    w1, b1, w2, b2 = keep
    c = lte_cnn(w1.shape[1], w1.shape[3], past1, w2.shape[2], past2, w1.data_ptr(), b1.data_ptr(),
                w2.data_ptr(), b2.data_ptr())
    return c, keep


def version() -> str:
    return _lib.lte_version().decode()


def lte_workspace_bytes(dims: lte_dims, which: int) -> int:
    return int(_lib.lte_workspace_bytes(C.byref(dims), which))


def lte_score(dims, cnn, k, v, j_begin, j_end, r, mask=None, stream=None):
    _call("lte_score", C.byref(dims), C.byref(cnn), _ptr(k), _ptr(v), C.byref(_strides(k)),
          j_begin, j_end, _ptr(r), _ptr(mask), _stream(stream))


def lte_evict_compact(dims, r, mask, n_scored, idx, nret, cnt, k=None, v=None, k_col=None,
                      v_col=None, stream=None):
    st = None if k is None else C.byref(_strides(k))
    _call("lte_evict_compact", C.byref(dims), _ptr(r), _ptr(mask), n_scored, _ptr(idx), _ptr(nret),
          _ptr(cnt), _ptr(k), _ptr(v), st, _ptr(k_col), _ptr(v_col), _stream(stream))


def lte_retained_lifetimes(dims, r, idx, nret, death, stream=None):
    _call("lte_retained_lifetimes", C.byref(dims), _ptr(r), _ptr(idx), _ptr(nret), _ptr(death),
          _stream(stream))


def lte_sparse_attn_prefill(dims, q, k, v, cnt, k_col, v_col, o, lse, workspace, stream=None,
                            death=None):
    _call("lte_sparse_attn_prefill", C.byref(dims), _ptr(q), _ptr(k), _ptr(v),
          C.byref(_strides(q)), C.byref(_strides(k)), _ptr(cnt), _ptr(death), _ptr(k_col),
          _ptr(v_col), _ptr(o), C.byref(_strides(o)), _ptr(lse), _ptr(workspace),
          workspace.numel() * workspace.element_size(), _stream(stream))


def lte_score_backward_workspace_bytes(dims, cnn) -> int:
    return int(_lib.lte_score_backward_workspace_bytes(C.byref(dims), C.byref(cnn)))


def lte_score_backward(dims, cnn, k, v, n_scored, dr, dk, dv, dw1, db1, dw2, db2, workspace,
                       stream=None):
    _call("lte_score_backward", C.byref(dims), C.byref(cnn), _ptr(k), _ptr(v), C.byref(_strides(k)),
          n_scored, _ptr(dr), _ptr(dk), _ptr(dv), _ptr(dw1), _ptr(db1), _ptr(dw2), _ptr(db2),
          _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))


def lte_sparse_attn_backward(dims, q, k, v, cnt, death, idx, nret, k_col, v_col, o, lse, do, dq,
                             dk, dv, workspace, stream=None):
    _call("lte_sparse_attn_backward", C.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(cnt),
          _ptr(death), _ptr(idx), _ptr(nret), _ptr(k_col), _ptr(v_col), _ptr(o), _ptr(lse), _ptr(do),
          _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
          workspace.numel() * workspace.element_size(), _stream(stream))


def lte_sparse_attn_prefill_relaxed(dims, q, k, v, cnt, death, idx, nret, k_col, v_col, r, o, lse,
                                    workspace, stream=None):
    _call("lte_sparse_attn_prefill_relaxed", C.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(cnt),
          _ptr(death), _ptr(idx), _ptr(nret), _ptr(k_col), _ptr(v_col), _ptr(r), _ptr(o), _ptr(lse),
          _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))


def lte_sparse_attn_backward_relaxed(dims, q, k, v, cnt, death, idx, nret, k_col, v_col, r, o, lse,
                                     do, dq, dk, dv, dr, workspace, stream=None):
    _call("lte_sparse_attn_backward_relaxed", C.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(cnt),
          _ptr(death), _ptr(idx), _ptr(nret), _ptr(k_col), _ptr(v_col), _ptr(r), _ptr(o), _ptr(lse),
          _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dr), _ptr(workspace),
          workspace.numel() * workspace.element_size(), _stream(stream))


def lte_cache_init_from_prefill(dims, cache, k, v, r, idx, cnt, T_prompt, n_scored, stream=None,
                                death=None):
    _call("lte_cache_init_from_prefill", C.byref(dims), C.byref(cache), _ptr(k), _ptr(v),
          C.byref(_strides(k)), _ptr(r), _ptr(idx), _ptr(cnt), _ptr(death), T_prompt, n_scored,
          _stream(stream))


def lte_decode_step(dims, cnn, cache, q_t, k_t, v_t, o_t, lse_t, score_batch, workspace,
                    stream=None):
    _call("lte_decode_step", C.byref(dims), C.byref(cnn), C.byref(cache), _ptr(q_t), _ptr(k_t),
          _ptr(v_t), _ptr(o_t), _ptr(lse_t), score_batch, _ptr(workspace),
          workspace.numel() * workspace.element_size(), _stream(stream))


def lte_decode_step_noalloc(dims, cnn, cache, q_t, k_t, v_t, o_t, lse_t, score_batch,
                            stream=None):
    """lte_decode_step without a workspace: the library's static device scratch
    (for callers that cannot allocate device memory; see lte_api.h)."""
    _call("lte_decode_step_noalloc", C.byref(dims), C.byref(cnn), C.byref(cache), _ptr(q_t),
          _ptr(k_t), _ptr(v_t), _ptr(o_t), _ptr(lse_t), score_batch, _stream(stream))


def lte_noalloc_read_device_error(stream=None):
    """(code, where) of the error word in lte_decode_step_noalloc's static
    scratch (the last call on the current device); synchronises the stream."""
    code, where = C.c_int32(0), C.c_int32(0)
    _call("lte_noalloc_read_device_error", C.byref(code), C.byref(where), _stream(stream))
    return code.value, where.value


def lte_sparse_attn_prefill_kernel(dims, q_strides=None, kv_strides=None, o_strides=None):
    """Kernel family (LTE_KERNEL_*) lte_sparse_attn_prefill runs for these dims
    and lte_strides (None = contiguous).  Host only."""
    kind = C.c_int32(0)
    ref = (lambda s: None if s is None else C.byref(s))
    _call("lte_sparse_attn_prefill_kernel", C.byref(dims), ref(q_strides), ref(kv_strides),
          ref(o_strides), C.byref(kind))
    return kind.value


def lte_sparse_attn_backward_kernel(dims):
    """Kernel family (LTE_KERNEL_*) lte_sparse_attn_backward runs for these dims."""
    kind = C.c_int32(0)
    _call("lte_sparse_attn_backward_kernel", C.byref(dims), C.byref(kind))
    return kind.value


def lte_clear_device_error(workspace, stream=None):
    _call("lte_clear_device_error", _ptr(workspace), _stream(stream))


def lte_read_device_error(workspace, stream=None):
    code, where = C.c_int32(0), C.c_int32(0)
    _call("lte_read_device_error", _ptr(workspace), C.byref(code), C.byref(where), _stream(stream))
    return code.value, where.value


def lte_wait_probe(flag, expect, limit_ns, workspace, stream=None):
    """Diagnostic: a bounded device wait on an mbarrier that arrives only once
    the device int32 `flag` equals `expect`; if it never does, the wait runs
    out after limit_ns and LTE_ERR_TIMEOUT lands in the workspace error word."""
    _call("lte_wait_probe", _ptr(flag), int(expect), int(limit_ns), _ptr(workspace),
          _stream(stream))


def lte_gla_prefill(q, k, v, a, o, state, stream=None):
    B, T, H, dk = q.shape
    dv = v.shape[3]
    _call("lte_gla_prefill", B, T, H, dk, dv, dtype_code(q.dtype), _ptr(q), _ptr(k), _ptr(v),
          _ptr(a), _ptr(o), _ptr(state), _stream(stream))


def lte_gla_decode_step(q_t, k_t, v_t, a_t, o_t, state, stream=None):
    B, H, dk = q_t.shape
    dv = v_t.shape[2]
    _call("lte_gla_decode_step", B, H, dk, dv, dtype_code(q_t.dtype), _ptr(q_t), _ptr(k_t),
          _ptr(v_t), _ptr(a_t), _ptr(o_t), _ptr(state), _stream(stream))
