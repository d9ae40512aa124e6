"""Thin host-side helpers over the C ABI: allocate the caller-owned buffers
(torch device memory) and chain the entry points of one LTE layer.

Nothing here computes: prefill = lte_score (when a CNN is given) ->
lte_evict_compact -> lte_sparse_attn_prefill; a decode step is one
lte_decode_step call on a DecodeCache.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import lte as L


@dataclass
class LayerParams:
    sink: int
    window: int
    cap: int
    tau: float = 0.5
    scale: float | None = None
    past1: int = 2
    past2: int = 1
    cap_policy: int = L.LTE_CAP_RECENT      # or L.LTE_CAP_FIRST

    def dims(self, B, T, Hq, Hkv, D, dtype) -> L.lte_dims:
        scale = (1.0 / D ** 0.5) if self.scale is None else self.scale
        return L.make_dims(B, T, Hq, Hkv, D, self.sink, self.window, self.cap, self.tau, scale, dtype,
                           self.cap_policy)


def cnn_future(w1, w2, past1, past2) -> int:
    return (w1.shape[3] - 1 - past1) + (w2.shape[2] - 1 - past2)


@dataclass
class PrefillOut:
    o: torch.Tensor
    lse: torch.Tensor
    r: torch.Tensor | None
    mask: torch.Tensor | None
    idx: torch.Tensor
    nret: torch.Tensor
    cnt: torch.Tensor
    k_col: torch.Tensor
    v_col: torch.Tensor
    n_scored: int
    death: torch.Tensor | None = None      # retained lifetimes (LTE_CAP_LOWEST)


class PrefillBuffers:
    """All buffers one prefill needs, allocated once (reused across calls)."""

    def __init__(self, B, T, Hq, Hkv, D, dtype, sink, dims, device="cuda", want_r=True):
        dev = torch.device(device)
        self.dims = dims
        self.o = torch.empty(B, T, Hq, D, dtype=dtype, device=dev)
        self.lse = torch.empty(B, Hq, T, dtype=torch.float32, device=dev)
        self.r = torch.full((B, Hkv, T), float("nan"), dtype=torch.float32, device=dev) if want_r else None
        self.mask = torch.zeros(B, Hkv, T, dtype=torch.uint8, device=dev) if want_r else None
        self.idx = torch.empty(B, Hkv, T, dtype=torch.int32, device=dev)
        self.nret = torch.empty(B, Hkv, dtype=torch.int32, device=dev)
        self.cnt = torch.empty(B, Hkv, T, dtype=torch.int32, device=dev)
        self.k_col = torch.empty(B, Hkv, sink + T, D, dtype=dtype, device=dev)
        self.v_col = torch.empty(B, Hkv, sink + T, D, dtype=dtype, device=dev)
        self.death = (torch.empty(B, Hkv, T, dtype=torch.int32, device=dev)
                      if dims.cap_policy == L.LTE_CAP_LOWEST else None)
        ws = L.lte_workspace_bytes(dims, L.LTE_WS_PREFILL)
        self.ws = torch.zeros((ws + 15) // 16 * 16, dtype=torch.uint8, device=dev)


def prefill(q, k, v, p: LayerParams, mask=None, cnn=None, bufs: PrefillBuffers | None = None,
            stream=None, scores=None) -> PrefillOut:
    """One LTE layer prefill.  Either a fed retention `mask` [B,Hkv,T] (uint8),
    fed `scores` [B,Hkv,T] (fp32, retained iff >= tau), or `cnn` = (w1, b1,
    w2, b2) device tensors for live scoring.  LTE_CAP_LOWEST needs scores
    (fed or live): they rank the retained tokens."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    dims = p.dims(B, T, Hq, Hkv, D, q.dtype)
    lowest = p.cap_policy == L.LTE_CAP_LOWEST
    if lowest and cnn is None and scores is None:
        raise ValueError("LTE_CAP_LOWEST ranks retained tokens by score: pass cnn or scores")
    if bufs is None:
        bufs = PrefillBuffers(B, T, Hq, Hkv, D, q.dtype, p.sink, dims, q.device, want_r=cnn is not None)
    r = scores
    if cnn is not None:
        w1, b1, w2, b2 = cnn
        c, _keep = L.make_cnn(w1, b1, w2, b2, p.past1, p.past2)
        n_scored = max(0, T - cnn_future(w1, w2, p.past1, p.past2))
        L.lte_score(dims, c, k, v, 0, n_scored, bufs.r, bufs.mask, stream)
        L.lte_evict_compact(dims, None, bufs.mask, n_scored, bufs.idx, bufs.nret, bufs.cnt, k, v,
                            bufs.k_col, bufs.v_col, stream)
        r = bufs.r
    elif scores is not None:
        n_scored = T
        L.lte_evict_compact(dims, scores, None, T, bufs.idx, bufs.nret, bufs.cnt, k, v, bufs.k_col,
                            bufs.v_col, stream)
    else:
        n_scored = T
        L.lte_evict_compact(dims, None, mask, T, bufs.idx, bufs.nret, bufs.cnt, k, v, bufs.k_col,
                            bufs.v_col, stream)
    if lowest:
        L.lte_retained_lifetimes(dims, r, bufs.idx, bufs.nret, bufs.death, stream)
    L.lte_sparse_attn_prefill(dims, q, k, v, bufs.cnt, bufs.k_col, bufs.v_col, bufs.o, bufs.lse,
                              bufs.ws, stream, death=bufs.death if lowest else None)
    return PrefillOut(bufs.o, bufs.lse, r, bufs.mask if cnn is not None else mask, bufs.idx,
                      bufs.nret, bufs.cnt, bufs.k_col, bufs.v_col, n_scored,
                      bufs.death if lowest else None)


def prefill_relaxed(q, k, v, out: PrefillOut, r, p: LayerParams, stream=None):
    """Training-time forward with relaxed retention over the attended sets of
    `out` (from prefill on the same q, k, v): every retained-segment key j
    enters the softmax with weight r[j] (r [B,Hkv,T] fp32, the scores behind
    the retention mask).  Returns (o, lse, workspace); pass the workspace on
    to backward_relaxed."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    dims = p.dims(B, T, Hq, Hkv, D, q.dtype)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device=q.device)
    ws_bytes = L.lte_workspace_bytes(dims, L.LTE_WS_RELAXED)
    ws = torch.zeros((ws_bytes + 15) // 16 * 16, dtype=torch.uint8, device=q.device)
    L.lte_sparse_attn_prefill_relaxed(dims, q, k, v, out.cnt, out.death, out.idx, out.nret,
                                      out.k_col, out.v_col, r, o, lse, ws, stream)
    return o, lse, ws


def backward_relaxed(q, k, v, out: PrefillOut, r, o, lse, do, p: LayerParams, ws=None,
                     stream=None, check_errors=False):
    """Gradients of the relaxed-retention forward (o, lse from
    prefill_relaxed): dq [B,T,Hq,D], dk, dv [B,T,Hkv,D] and dr [B,Hkv,T]
    (fp32), dr being the dL/dr that lte_score_backward takes."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    dims = p.dims(B, T, Hq, Hkv, D, q.dtype)
    dev = q.device
    dq = torch.empty(B, T, Hq, D, dtype=torch.float32, device=dev)
    dk = torch.empty(B, T, Hkv, D, dtype=torch.float32, device=dev)
    dv = torch.empty(B, T, Hkv, D, dtype=torch.float32, device=dev)
    dr = torch.empty(B, Hkv, T, dtype=torch.float32, device=dev)
    if ws is None:
        ws_bytes = L.lte_workspace_bytes(dims, L.LTE_WS_RELAXED)
        ws = torch.zeros((ws_bytes + 15) // 16 * 16, dtype=torch.uint8, device=dev)
    L.lte_sparse_attn_backward_relaxed(dims, q, k, v, out.cnt, out.death, out.idx, out.nret,
                                       out.k_col, out.v_col, r, o, lse, do, dq, dk, dv, dr, ws,
                                       stream)
    if check_errors:
        code, where = L.lte_read_device_error(ws, stream)
        if code != 0:
            raise L.LteError(f"lte_sparse_attn_backward_relaxed (device check {where})", code)
    return dq, dk, dv, dr


def backward(q, k, v, out: PrefillOut, do, p: LayerParams, stream=None, check_errors=False):
    """Gradients (fp32) of the prefill attention for the attended sets that
    `out` (from prefill on the same q, k, v) used, given dO = do.
    Returns dq [B,T,Hq,D], dk, dv [B,T,Hkv,D].  check_errors: synchronise and
    raise if a device-side check or wait failed."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    dims = p.dims(B, T, Hq, Hkv, D, q.dtype)
    dev = q.device
    dq = torch.empty(B, T, Hq, D, dtype=torch.float32, device=dev)
    dk = torch.empty(B, T, Hkv, D, dtype=torch.float32, device=dev)
    dv = torch.empty(B, T, Hkv, D, dtype=torch.float32, device=dev)
    ws_bytes = L.lte_workspace_bytes(dims, L.LTE_WS_BACKWARD)
    ws = torch.zeros((ws_bytes + 15) // 16 * 16, dtype=torch.uint8, device=dev)
    L.lte_sparse_attn_backward(dims, q, k, v, out.cnt, out.death, out.idx, out.nret, out.k_col,
                               out.v_col, out.o, out.lse, do, dq, dk, dv, ws, stream)
    if check_errors:
        code, where = L.lte_read_device_error(ws, stream)
        if code != 0:
            raise L.LteError(f"lte_sparse_attn_backward (device check {where})", code)
    return dq, dk, dv


class DecodeCache:
    """Caller-owned decode cache (window ring + sink slots + retained ring)."""

    def __init__(self, B, Hkv, D, dtype, sink, window, cap, device="cuda"):
        dev = torch.device(device)
        Ls = window + sink + cap
        self.k = torch.zeros(B, Hkv, Ls, D, dtype=dtype, device=dev)
        self.v = torch.zeros(B, Hkv, Ls, D, dtype=dtype, device=dev)
        self.pos = torch.full((B, Hkv, Ls), -1, dtype=torch.int32, device=dev)
        self.win_r = torch.full((B, Hkv, window), float("nan"), dtype=torch.float32, device=dev)
        self.ret_total = torch.zeros(B, Hkv, dtype=torch.int32, device=dev)
        self.meta = torch.zeros(4, dtype=torch.int32, device=dev)
        # scores of the retained slots' tokens (read under LTE_CAP_LOWEST only)
        self.ret_r = torch.full((B, Hkv, max(cap, 1)), float("nan"), dtype=torch.float32, device=dev)
        self.sink, self.window, self.cap = sink, window, cap
        self.struct = L.lte_cache(self.k.data_ptr(), self.v.data_ptr(), self.pos.data_ptr(),
                                  self.win_r.data_ptr(), self.ret_total.data_ptr(),
                                  self.meta.data_ptr(), self.ret_r.data_ptr())

    def init_from_prefill(self, dims, k, v, out: PrefillOut, T_prompt, stream=None):
        L.lte_cache_init_from_prefill(dims, self.struct, k, v, out.r, out.idx, out.cnt, T_prompt,
                                      out.n_scored, stream, death=out.death)

    def _state(self):
        return (self.k, self.v, self.pos, self.win_r, self.ret_total, self.meta, self.ret_r)

    def snapshot(self):
        """Device copies of every tensor the decode step reads or writes (the
        step index and its ticket live in `meta`), for `restore`."""
        return tuple(t.clone() for t in self._state())

    def restore(self, snap):
        """Put the cache back to a `snapshot` in place, on the current stream
        (same buffers, so a CUDA graph captured over this cache stays valid).
        No decode step of this cache may be in flight."""
        for t, s in zip(self._state(), snap):
            t.copy_(s)

    def retained_positions(self):
        """Sorted retained positions per unit (host copy, for checks)."""
        w, s = self.window, self.sink
        pos = self.pos[:, :, w + s:].cpu()
        return [[sorted(int(x) for x in pos[b, h] if x >= 0) for h in range(pos.shape[1])]
                for b in range(pos.shape[0])]


class Decoder:
    """Runs lte_decode_step with fixed output buffers (graph-capturable)."""

    def __init__(self, dims, cnn, past1, past2, cache: DecodeCache, score_batch, device="cuda"):
        self.dims = dims
        w1, b1, w2, b2 = cnn
        self.cnn, self._keep = L.make_cnn(w1, b1, w2, b2, past1, past2)
        self.cache = cache
        self.score_batch = score_batch
        B, Hq, D = dims.B, dims.Hq, dims.D
        dt = torch.bfloat16 if dims.dtype == L.LTE_BF16 else torch.float32
        self.o = torch.empty(B, Hq, D, dtype=dt, device=device)
        self.lse = torch.empty(B, Hq, dtype=torch.float32, device=device)
        ws = L.lte_workspace_bytes(dims, L.LTE_WS_DECODE)
        self.ws = torch.zeros((ws + 15) // 16 * 16, dtype=torch.uint8, device=device)

    def step(self, q_t, k_t, v_t, stream=None):
        L.lte_decode_step(self.dims, self.cnn, self.cache.struct, q_t, k_t, v_t, self.o, self.lse,
                          self.score_batch, self.ws, stream)
        return self.o, self.lse

    def device_error(self, stream=None):
        """(code, where) of this decoder's workspace error word (synchronises)."""
        return L.lte_read_device_error(self.ws, stream)


class HostPrefill:
    """Prefill of a batch that lives in pinned host memory, streamed through
    the device in sub-batches of `chunk` sequences.

    Two device slots alternate.  Sub-batch c is copied in on one stream, computed
    (lte_evict_compact with a fed mask, then lte_sparse_attn_prefill) on a
    second and copied out on a third, so the input copy of c + 1 and the output
    copy of c - 1 overlap the compute of c, and the two copy directions overlap
    each other.  The copies are the only work outside the library's kernels."""

    def __init__(self, B, T, Hq, Hkv, D, dtype, p: LayerParams, chunk, device="cuda"):
        if B % chunk:
            raise ValueError("the batch must be a multiple of the sub-batch")
        if p.cap_policy == L.LTE_CAP_LOWEST:
            raise ValueError("a fed mask carries no scores to rank retained tokens by")
        dev = torch.device(device)
        self.B, self.T, self.chunk, self.p = B, T, chunk, p
        self.dims = p.dims(chunk, T, Hq, Hkv, D, dtype)
        self.slots = []
        for _ in range(2):
            self.slots.append(dict(
                q=torch.empty(chunk, T, Hq, D, dtype=dtype, device=dev),
                k=torch.empty(chunk, T, Hkv, D, dtype=dtype, device=dev),
                v=torch.empty(chunk, T, Hkv, D, dtype=dtype, device=dev),
                mask=torch.empty(chunk, Hkv, T, dtype=torch.uint8, device=dev),
                bufs=PrefillBuffers(chunk, T, Hq, Hkv, D, dtype, p.sink, self.dims, dev, want_r=False)))
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream(dev) for _ in range(3))
        ev = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
        self.in_done, self.comp_done, self.out_done = ev(), ev(), ev()

    def run(self, hq, hk, hv, hmask, ho, stream=None):
        """hq, hk, hv [B,T,H,D], hmask [B,Hkv,T] uint8 and ho [B,T,Hq,D]: pinned host
        tensors.  Work is ordered after `stream` (default: the current stream),
        which in turn waits for the last output copy."""
        stream = torch.cuda.current_stream() if stream is None else stream
        start = torch.cuda.Event()
        start.record(stream)
        for st in (self.s_in, self.s_comp, self.s_out):
            st.wait_event(start)
        n = self.B // self.chunk
        for c in range(n):
            s, sl = c % 2, self.slots[c % 2]
            b0, b1 = c * self.chunk, (c + 1) * self.chunk
            if c >= 2:
                self.s_in.wait_event(self.comp_done[s])       # the slot's inputs have been read
            with torch.cuda.stream(self.s_in):
                sl["q"].copy_(hq[b0:b1], non_blocking=True)
                sl["k"].copy_(hk[b0:b1], non_blocking=True)
                sl["v"].copy_(hv[b0:b1], non_blocking=True)
                sl["mask"].copy_(hmask[b0:b1], non_blocking=True)
            self.in_done[s].record(self.s_in)
            self.s_comp.wait_event(self.in_done[s])
            if c >= 2:
                self.s_comp.wait_event(self.out_done[s])      # the slot's o has been copied out
            bufs = sl["bufs"]
            L.lte_evict_compact(self.dims, None, sl["mask"], self.T, bufs.idx, bufs.nret, bufs.cnt,
                                sl["k"], sl["v"], bufs.k_col, bufs.v_col, self.s_comp)
            L.lte_sparse_attn_prefill(self.dims, sl["q"], sl["k"], sl["v"], bufs.cnt, bufs.k_col,
                                      bufs.v_col, bufs.o, bufs.lse, bufs.ws, self.s_comp)
            self.comp_done[s].record(self.s_comp)
            self.s_out.wait_event(self.comp_done[s])
            with torch.cuda.stream(self.s_out):
                ho[b0:b1].copy_(bufs.o, non_blocking=True)
            self.out_done[s].record(self.s_out)
        stream.wait_stream(self.s_out)
        stream.wait_stream(self.s_comp)
        stream.wait_stream(self.s_in)

    def device_errors(self):
        return [L.lte_read_device_error(sl["bufs"].ws) for sl in self.slots]
