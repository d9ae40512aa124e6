"""Shared helpers of the GPU parity tests (no method arithmetic here: the
expected values come from oracle/, the inputs from lte_inputs)."""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import lte_oracle as O

# Tolerances: bf16 inputs with fp32 accumulation / fp32 inputs (max-abs on o),
# plus two gates that a wrong key set cannot pass: lse max-abs (one missing
# key moves lse by ~1/|S_t|) and max-abs error relative to max |o|.
TOL = {
    torch.float32: dict(o=1e-4, rel=1e-5, lse=1e-5),
    torch.bfloat16: dict(o=2e-2, rel=1e-2, lse=1e-4),
}
R_TOL = 1e-6          # retention scores, fp32 vs float64
MASK_BAND = 1e-5      # masks are compared only where |r - tau| exceeds this


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float64 values rounded to bf16 (round to nearest even) and widened back:
    the storage format of a bf16 output."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


def oracle_cnn(cnn, h: int, past1=2, past2=1) -> O.CNN:
    w1, b1, w2, b2 = (f64(x) for x in cnn)
    return O.CNN(w1[h], b1[h], w2[h], float(b2[h]), past1, past2)


def clean_tau(r: np.ndarray, lo_q=0.3, hi_q=0.7) -> tuple[float, float]:
    """A threshold in the widest gap between the oracle's scores (between
    the given quantiles) and its distance to the nearest score.  Used by
    end-to-end tests so that no score sits within rounding of tau."""
    x = np.sort(r[np.isfinite(r)].ravel())
    a, b = int(lo_q * len(x)), int(hi_q * len(x))
    seg = x[a:b + 1]
    gaps = np.diff(seg)
    i = int(np.argmax(gaps))
    return float((seg[i] + seg[i + 1]) / 2), float(gaps[i] / 2)


def assert_attention_close(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what=""):
    tol = TOL[dtype]
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    err = np.abs(o_gpu - o_ref)
    max_err = float(np.nanmax(err))
    scale = float(np.nanmax(np.abs(o_ref)))
    assert max_err <= tol["o"], f"{what}: o max-abs {max_err:.3g} > {tol['o']}"
    assert max_err <= tol["rel"] * scale + 1e-30 or max_err <= 1e-7, \
        f"{what}: o max-abs/max|o| {max_err / scale:.3g} > {tol['rel']}"
    if lse_gpu is not None:
        lerr = float(np.nanmax(np.abs(np.asarray(lse_gpu, np.float64) - lse_ref)))
        assert lerr <= tol["lse"], f"{what}: lse max-abs {lerr:.3g} > {tol['lse']}"
    return max_err


def fed_masks(mask: torch.Tensor, sink: int) -> np.ndarray:
    m = mask.cpu().numpy().astype(np.uint8).copy()
    m[..., :sink] = 0
    return m


def oracle_rows(q, k, v, masks, b, h, rows, sink, window, cap, scale, policy=O.CAP_RECENT,
                r=None):
    """Oracle o [len(rows), G, D], lse [len(rows), G] for one unit (r [B,Hkv,T]:
    the scores, for policy "lowest")."""
    Hq, Hkv = q.shape[2], k.shape[2]
    G = Hq // Hkv
    qn = f64(q[b, :, h * G:(h + 1) * G])
    kn, vn = f64(k[b, :, h]), f64(v[b, :, h])
    o, lse, cnt = O.prefill_unit(qn, kn, vn, masks[b, h], sink, window, cap, scale, rows=rows,
                                 policy=policy, r=None if r is None else f64(r[b, h]))
    return o[rows], lse[rows], cnt[rows]


def scale_of(D):
    return 1.0 / math.sqrt(D)


# Gradients of the attention (bf16 products, fp32 accumulation): every element
# of a row (one position of dk / dv, one (position, head) of dq) within
# GRAD_ROW of that row's largest reference entry, plus GRAD_ABS.  P and dS are
# rounded to bf16 (2^-9 relative) before the products that use them, so a
# gradient sum carries about 2^-8 relative error per term, well inside 2e-2;
# a missing or doubled contribution to one row (a slot attended from many
# rows) moves that row by far more.
GRAD_ROW = 2e-2
GRAD_ABS = 1e-6


def assert_grad_close(g, ref, what="", extra=None):
    """Element-wise gate of a gradient tensor [..., D] against the oracle's:
    |g - ref| <= GRAD_ROW * max_row |ref| + GRAD_ABS (+ extra, an allowance
    per element derived from the arithmetic, see dq_delta_allowance) at every
    element.  Returns the largest error relative to its row's scale."""
    g, ref = np.asarray(g, np.float64), np.asarray(ref, np.float64)
    row = np.abs(ref).max(axis=-1, keepdims=True)
    err = np.abs(g - ref)
    bound = GRAD_ROW * row + GRAD_ABS
    if extra is not None:
        bound = bound + np.asarray(extra, np.float64)
    bound = np.broadcast_to(bound, err.shape)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(int(np.argmax(err - bound)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} element(s) outside the row bound; worst at "
                             f"{i}: |err| {err[i]:.3g} > {bound[i]:.3g} (row max {row[i[:-1] + (0,)]:.3g}; row {i[:-1]})")
    return float((err / np.maximum(row, 1e-30)).max())


# The backward takes D_t = <dO_t, o_t> from the forward's stored output o.
# That o differs from the exact one by at most 2^-8 |o| per element (P and
# the output rounded to bf16), so D_t is off by up to 2^-8 sum_d |dO_td o_td|,
# which moves dq_t by scale * dD_t * (P K)_t (dS = P (dP - D_t)).  On rows
# with many keys this is far below the row gate; on rows with two or three
# keys, where dq is a near-cancelling sum, it is not.
def dq_delta_allowance(do, o, pk, scale):
    """Per-element allowance for dq [..., D]: do, o the incoming gradient and
    the oracle's output, pk the oracle's attention-weighted keys sum_j P_j k_j
    (all [..., D])."""
    do, o, pk = (np.asarray(x, np.float64) for x in (do, o, pk))
    dD = 2.0 ** -8 * np.abs(do * o).sum(axis=-1, keepdims=True)
    return scale * dD * np.abs(pk)
