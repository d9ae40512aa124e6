"""Plain CPU oracle for contextualized Learnable Token Eviction (LTE).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The GPU library never
calls it and shares no code with it.

Everything is computed in float64 with numpy, one (batch element, KV head) unit
at a time, in the order the method is described.  Inputs given in bf16 or fp32
are widened exactly to float64 by the caller (``np.asarray(x, np.float64)``).

Sources (web pages; cited by title and figure/section):

* [LTE] "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse
  Attention and Contextualized Learnable Token Eviction" (He & Garner, 2025),
  TL;DR, Abstract, and the captions of Figure 2 (eviction scheme: CNN
  retention score r_{j,h}, attention sink s, sliding window w, decision taken
  when a KV pair leaves the window, A-plus-column pattern) and Figure 3
  (inference cache: circular SWA segment plus a capped out-of-window segment
  holding sink and retained KVs; scoring batched and deferred).
* [SWA-LA] "Sparse Linear Attention: Viewing SWA from the Perspective of
  Linear Attention", section "Viewing SWA from the linear-state perspective"
  (the window as a FIFO of slots, one slot overwritten per token).

Readings taken where the pages are silent (each is restated where used):

* window (t-w, t] holds w keys including the current token;
* the cap C counts retained tokens only (sinks are extra); when more than C
  tokens qualify, the C most recent are kept (FIFO ring) -- policy "recent".
  The pages leave the capped segment's policy open; policy "first" keeps the
  first C retained tokens instead (later ones are dropped once the segment is
  full); policy "lowest" drops, when a retained token arrives at a full
  segment, the one with the lowest retention score among the C held and the
  newcomer (equal scores: the older token goes);
* retain iff r >= tau; the first s tokens are sinks and are never "retained";
* CNN: conv1d over the channel concatenation [k; v] (k first), PyTorch
  cross-correlation convention, per-layer zero padding outside [0, n), a
  token is scorable only once its whole receptive field exists;
* softmax scale is a parameter (1/sqrt(D) by default); KV head of query head
  q is q // (Hq / Hkv);
* backward: the pages say the model is trained end to end but give no
  gradient for the keep/evict decision, so the attention backward holds the
  attended sets fixed, and the CNN backward takes dL/dr as an input.

Parity pins: every function here is checked in ``tests/test_oracle_*.py``
against something other than itself (library routines on special cases,
closed forms, brute-force enumeration, an independent simulation).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def sigmoid(x):
    """Logistic function 1 / (1 + exp(-x)) in float64."""
    x = _f64(x)
    return 1.0 / (1.0 + np.exp(-x))


def silu(x):
    """SiLU(x) = x * sigmoid(x) in float64."""
    x = _f64(x)
    return x * sigmoid(x)


# ---------------------------------------------------------------------------
# (1) retention scores: the per-KV-head CNN  [LTE, TL;DR; Abstract; Fig. 2]
# ---------------------------------------------------------------------------

@dataclass
class CNN:
    """Weights of one two-layer scoring CNN stack for ONE KV head.

    w1 [C1, 2D, K1], b1 [C1], w2 [C1, K2], b2 scalar.  Layer l reads
    ``past_l`` tokens before and ``K_l - 1 - past_l`` after the output token.
    """
    w1: np.ndarray
    b1: np.ndarray
    w2: np.ndarray
    b2: float
    past1: int
    past2: int

    @property
    def future(self) -> int:
        """F: how many tokens after j the score r_j depends on."""
        return (self.w1.shape[2] - 1 - self.past1) + (self.w2.shape[1] - 1 - self.past2)

    @property
    def past(self) -> int:
        """P: how many tokens before j the score r_j depends on."""
        return self.past1 + self.past2


def _shifted(x: np.ndarray, shift: int) -> np.ndarray:
    """y[:, j] = x[:, j + shift] where 0 <= j + shift < n, else 0 (zero padding)."""
    n = x.shape[1]
    y = np.zeros_like(x)
    lo, hi = max(0, -shift), min(n, n - shift)
    if hi > lo:
        y[:, lo:hi] = x[:, lo + shift:hi + shift]
    return y


def cnn_scores(k, v, cnn: CNN, n_avail: int | None = None) -> np.ndarray:
    """Retention scores r_j of one (batch element, KV head) unit.

    [LTE, Fig. 2]: a CNN stack reads short-range past and future context of
    each KV pair and outputs a per-token, per-head retention score; the score
    can be computed once the CNN receptive field is available.

    Layer 1: u[c, j] = SiLU(b1[c] + sum_ch sum_kk w1[c, ch, kk] * x[ch, j+kk-past1])
    Layer 2: r[j]    = sigmoid(b2 + sum_c sum_kk w2[c, kk] * u[c, j+kk-past2])
    with x = [k; v] (channels 0..D-1 from k, D..2D-1 from v), and each layer's
    input taken as 0 outside [0, n_avail).

    k, v: [n, D] (any float dtype).  Returns r [n] float64; tokens whose
    receptive field reaches past n_avail - 1 are not yet scorable and get NaN.
    """
    k = _f64(k)
    v = _f64(v)
    n = k.shape[0] if n_avail is None else int(n_avail)
    x = np.concatenate([k[:n], v[:n]], axis=1).T            # [2D, n]
    c1, two_d, k1 = cnn.w1.shape
    assert two_d == x.shape[0]
    u = np.zeros((c1, n))
    for kk in range(k1):
        u += _f64(cnn.w1[:, :, kk]) @ _shifted(x, kk - cnn.past1)
    u = silu(u + _f64(cnn.b1)[:, None])
    z = np.full(n, float(cnn.b2))
    for kk in range(cnn.w2.shape[1]):
        z += _f64(cnn.w2[:, kk]) @ _shifted(u, kk - cnn.past2)
    r = sigmoid(z)
    last = n - 1 - cnn.future                                 # last scorable token
    r[max(0, last + 1):] = np.nan
    return r


def cnn_backward(k, v, cnn: CNN, dr, n_scored: int):
    """Gradients of L = sum_{j < n_scored} dr[j] r[j] through the scoring CNN
    of one (batch element, KV head) unit, r as in ``cnn_scores`` with
    n_avail = n (the whole sequence).  [LTE, Abstract: trained end to end;
    the pages fix no dL/dr, so dr is an input.]

    Chain rule through the two layers, written out:
      dz2[j] = dr[j] r[j] (1 - r[j])                     (j < n_scored, else 0)
      du[c, i]  = sum_kk w2[c, kk] dz2[i - kk + past2]   (u read at j + kk - past2)
      dz1[c, i] = du[c, i] SiLU'(z1[c, i]),  SiLU'(z) = s(z) (1 + z (1 - s(z)))
      dx[ch, m] = sum_{c, kk} w1[c, ch, kk] dz1[c, m - kk + past1]
      dw1[c, ch, kk] = sum_i dz1[c, i] x[ch, i + kk - past1],  db1 = sum_i dz1
      dw2[c, kk] = sum_j dz2[j] u[c, j + kk - past2],       db2 = sum_j dz2
    with every shifted read 0 outside [0, n), as in the forward.
    Returns dk, dv [n, D], dw1 [C1, 2D, K1], db1 [C1], dw2 [C1, K2], db2."""
    k, v = _f64(k), _f64(v)
    n, D = k.shape
    x = np.concatenate([k, v], axis=1).T                      # [2D, n]
    w1, w2 = _f64(cnn.w1), _f64(cnn.w2)
    c1, _, k1 = w1.shape
    k2 = w2.shape[1]
    z1 = np.zeros((c1, n))
    for kk in range(k1):
        z1 += w1[:, :, kk] @ _shifted(x, kk - cnn.past1)
    z1 += _f64(cnn.b1)[:, None]
    u = silu(z1)
    z2 = np.full(n, float(cnn.b2))
    for kk in range(k2):
        z2 += w2[:, kk] @ _shifted(u, kk - cnn.past2)
    r = sigmoid(z2)
    g = np.zeros(n)
    g[:n_scored] = _f64(dr)[:n_scored]
    dz2 = g * r * (1.0 - r)
    du = np.zeros((c1, n))
    dw2 = np.zeros((c1, k2))
    for kk in range(k2):
        us = _shifted(u, kk - cnn.past2)                      # us[:, j] = u[:, j + kk - past2]
        dw2[:, kk] = us @ dz2
        du += w2[:, kk][:, None] * _shifted(dz2[None, :], -(kk - cnn.past2))
    sg = sigmoid(z1)
    dz1 = du * sg * (1.0 + z1 * (1.0 - sg))
    dx = np.zeros_like(x)
    dw1 = np.zeros_like(w1)
    for kk in range(k1):
        xs = _shifted(x, kk - cnn.past1)
        dw1[:, :, kk] = dz1 @ xs.T
        dx += w1[:, :, kk].T @ _shifted(dz1, -(kk - cnn.past1))
    return (dx[:D].T.copy(), dx[D:].T.copy(), dw1, dz1.sum(axis=1), dw2, float(dz2.sum()))


# ---------------------------------------------------------------------------
# (2) eviction decision and compaction  [LTE, Fig. 2 and Fig. 3]
# ---------------------------------------------------------------------------

def retention_mask(r, sink: int, tau: float) -> np.ndarray:
    """m_j = (j >= s) and (r_j >= tau); unscored tokens (NaN) get 0.

    [LTE, Fig. 2]: r_{j,h} decides whether the KV pair is evicted when it
    moves out of the window; sinks are kept regardless, so they are never
    counted as retained.
    """
    r = _f64(r)
    m = np.zeros(r.shape[0], dtype=np.uint8)
    for j in range(r.shape[0]):
        if j >= sink and not math.isnan(r[j]) and r[j] >= tau:
            m[j] = 1
    return m


def fed_mask(mask, sink: int) -> np.ndarray:
    """A retention mask given directly (attention isolated from scoring), with
    the sink positions forced to 0 because sinks are never 'retained'."""
    m = np.asarray(mask, dtype=np.uint8).copy()
    m[:sink] = 0
    return m


def compact(m) -> tuple[np.ndarray, int, np.ndarray]:
    """Ascending list of retained positions, its length, and inclusive
    prefix counts cnt[j] = #{i <= j : m_i = 1}.  Plain definition."""
    m = np.asarray(m, dtype=np.int64)
    idx = [j for j in range(m.shape[0]) if m[j]]
    cnt = np.zeros(m.shape[0], dtype=np.int64)
    running = 0
    for j in range(m.shape[0]):
        running += int(m[j])
        cnt[j] = running
    return np.array(idx, dtype=np.int64), len(idx), cnt


# ---------------------------------------------------------------------------
# (3) attended set and attention  [LTE, Fig. 2 right: A-plus-column pattern]
# ---------------------------------------------------------------------------

CAP_RECENT, CAP_FIRST, CAP_LOWEST = "recent", "first", "lowest"   # capped-segment policies


def top_by_score(candidates, r, cap: int) -> list[int]:
    """The `cap` candidates j with the largest (r_j, j), i.e. the highest
    retention scores, the later token first among equal scores.

    This is what policy "lowest" holds after the candidates have arrived one by
    one (in position order) at a segment of capacity C that, when full, drops
    the lowest-scoring of its C tokens and the newcomer: a token is dropped
    exactly when C others that beat it have arrived, so the survivors are the
    C best of all arrivals.  ``test_oracle_sets`` checks this against the
    arrival-by-arrival simulation."""
    ranked = sorted(candidates, key=lambda j: (float(r[j]), j), reverse=True)
    return ranked[:cap]


def retained_set(t: int, m, sink: int, window: int, cap: int,
                 policy: str = CAP_RECENT, r=None) -> list[int]:
    """Ret_t: the retained tokens query t attends to, drawn from the tokens j
    in [s, t-w] with m_j = 1 (kept when they left the window):
    policy "recent": the `cap` largest such j (the C most recent);
    policy "first":  the `cap` smallest such j (the segment fills, then later
    retained tokens are dropped);
    policy "lowest": the `cap` such j with the highest scores r_j (the
    lowest-scoring token is dropped when the segment overflows; `r` required).
    Every member lies outside the window and the sink."""
    candidates = [j for j in range(sink, t - window + 1) if m[j]]
    if cap <= 0:
        return []
    if policy == CAP_RECENT:
        return candidates[-cap:]
    if policy == CAP_FIRST:
        return candidates[:cap]
    return sorted(top_by_score(candidates, r, cap))


def attended_set(t: int, m, sink: int, window: int, cap: int,
                 policy: str = CAP_RECENT, r=None) -> list[int]:
    """Key positions query t attends to, for one KV head:
    S_t = ([0, s) n [0, t])  u  (t-w, t]  u  Ret_t  (Ret_t: ``retained_set``).
    """
    keys = set(range(0, min(sink, t + 1)))
    keys |= set(range(max(0, t - window + 1), t + 1))
    keys |= set(retained_set(t, m, sink, window, cap, policy, r))
    return sorted(keys)


def attend(q_rows, K, V, scale: float):
    """Softmax attention of the rows of q over keys K / values V (float64).

    q_rows [G, D], K [n, D], V [n, Dv] -> (o [G, Dv], lse [G]) where
    lse = log sum_j exp(scale * q . k_j).  Max-subtracted for range safety.
    """
    q_rows, K, V = _f64(q_rows), _f64(K), _f64(V)
    logits = scale * (q_rows @ K.T)                           # [G, n]
    mx = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - mx)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ V) / l
    lse = (mx + np.log(l))[:, 0]
    return o, lse


def prefill_unit(q, k, v, m, sink: int, window: int, cap: int, scale: float,
                 rows=None, policy: str = CAP_RECENT, r=None):
    """Prefill of one (batch element, KV head) unit.

    q [T, G, D] (the G query heads that share this KV head), k, v [T, D],
    m [T] retention mask, r [T] retention scores (policy "lowest" only).
    Returns o [T, G, D], lse [T, G] and the attended count per row (rows not
    in `rows` are left as NaN / -1).
    """
    T, G, D = q.shape
    o = np.full((T, G, v.shape[1]), np.nan)
    lse = np.full((T, G), np.nan)
    count = np.full(T, -1, dtype=np.int64)
    k = _f64(k)
    v = _f64(v)
    for t in (range(T) if rows is None else rows):
        S = attended_set(t, m, sink, window, cap, policy, r)
        o[t], lse[t] = attend(q[t], k[S], v[S], scale)
        count[t] = len(S)
    return o, lse, count


def prefill(q, k, v, masks, sink: int, window: int, cap: int, scale: float | None = None,
            policy: str = CAP_RECENT, r=None):
    """Prefill over a batch: q [B,T,Hq,D], k, v [B,T,Hkv,D], masks [B,Hkv,T]
    (and scores r [B,Hkv,T] under policy "lowest").

    GQA: query head qh uses KV head qh // (Hq // Hkv).  Returns o [B,T,Hq,D],
    lse [B,Hq,T], count [B,Hkv,T].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = np.zeros((B, T, Hq, v.shape[3]))
    lse = np.zeros((B, Hq, T))
    count = np.zeros((B, Hkv, T), dtype=np.int64)
    for b in range(B):
        for h in range(Hkv):
            ou, lu, cu = prefill_unit(q[b, :, h * G:(h + 1) * G], k[b, :, h], v[b, :, h],
                                      masks[b, h], sink, window, cap, scale, policy=policy,
                                      r=None if r is None else r[b, h])
            o[b, :, h * G:(h + 1) * G] = ou
            lse[b, h * G:(h + 1) * G] = lu.T
            count[b, h] = cu
    return o, lse, count


# ---------------------------------------------------------------------------
# (3b) backward of the prefill attention for fixed attended sets
#      [LTE, Abstract: the model is trained end to end; the pages give no rule
#      for differentiating the eviction decisions, so the sets S_t are held
#      fixed and only the softmax attention over them is differentiated]
# ---------------------------------------------------------------------------

def prefill_backward_unit(q, k, v, m, sink: int, window: int, cap: int, scale: float, do,
                          policy: str = CAP_RECENT, r=None, o_out=None):
    """Gradients of L = sum_t <do_t, o_t> for one (batch element, KV head)
    unit, o_t the prefill output over the fixed attended set S_t.

    q, do [T, G, D]; k, v [T, D].  Row by row, with P the softmax weights of
    row t over S_t and o_t = P V_S:
      dP = do_t V_S^T,  D_t = <do_t, o_t> per head,  dS = P * (dP - D_t),
      dq_t = scale dS K_S,  dk_S += scale dS^T q_t,  dv_S += P^T do_t.
    A position attended both from the window and, later, from the retained
    segment receives both contributions in the same dk / dv row.
    o_out [T, G, D] (optional): the forward output as stored (e.g. rounded to
    bf16), used for D_t in place of the exact o -- the usual contract of an
    attention backward that is handed the forward's output; None = exact.
    Returns dq [T, G, D], dk [T, D], dv [T, D] (float64)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    T, G, D = q.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for t in range(T):
        S = attended_set(t, m, sink, window, cap, policy, r)
        Ks, Vs = k[S], v[S]
        logits = scale * (q[t] @ Ks.T)                        # [G, n]
        P = np.exp(logits - logits.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        o = P @ Vs if o_out is None else _f64(o_out[t])
        dP = do[t] @ Vs.T
        Dt = (do[t] * o).sum(axis=1, keepdims=True)
        dS = P * (dP - Dt)
        dq[t] = scale * (dS @ Ks)
        dk[S] += scale * (dS.T @ q[t])
        dv[S] += P.T @ do[t]
    return dq, dk, dv


def prefill_backward(q, k, v, masks, sink: int, window: int, cap: int, do,
                     scale: float | None = None, policy: str = CAP_RECENT, r=None, o_out=None):
    """prefill_backward_unit over a batch: q, do [B,T,Hq,D], k, v [B,T,Hkv,D],
    masks (and r) [B,Hkv,T], o_out [B,T,Hq,D] (optional, the stored forward
    output for D_t).  GQA as in ``prefill``: dk, dv of KV head h sum the
    contributions of its G query heads.  Returns dq, dk, dv (float64)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(Hkv):
            gq, gk, gv = prefill_backward_unit(
                q[b, :, h * G:(h + 1) * G], k[b, :, h], v[b, :, h], masks[b, h], sink, window,
                cap, scale, do[b, :, h * G:(h + 1) * G], policy, None if r is None else r[b, h],
                None if o_out is None else o_out[b, :, h * G:(h + 1) * G])
            dq[b, :, h * G:(h + 1) * G] = gq
            dk[b, :, h] = gk
            dv[b, :, h] = gv
    return dq, dk, dv


# ---------------------------------------------------------------------------
# (3c) relaxed retention for training  [LTE, Abstract: the CNN and the model
#      are trained end to end; Fig. 2 caption: r_{j,h} decides whether a KV
#      pair is kept.  The pages give no rule for how the loss reaches r, so this
#      reading is taken: the attended sets stay the hard ones (r >= tau, the
#      cap policy), and every retained-segment key j of row t (j in Ret_t)
#      enters the softmax with weight r_j, i.e. its logit gains log r_j.
#      Window and sink keys are unweighted.  r then receives
#        dL/dr_j = sum over rows t with j in Ret_t, heads g, of dS_{t,g,j} / r_j,
#      dS the gradient at the logits.  With r = 1 everything reduces to the
#      hard attention above.]
# ---------------------------------------------------------------------------

def _relaxed_row(t, q_t, k, v, m, sink, window, cap, scale, r, policy, r_rank):
    """Logits and the pieces of row t under relaxed retention: keys S (list),
    the bias vector (log r_j on Ret_t, else 0), logits [G, |S|]."""
    S = attended_set(t, m, sink, window, cap, policy, r_rank)
    ret = set(retained_set(t, m, sink, window, cap, policy, r_rank))
    bias = np.array([math.log(r[j]) if j in ret else 0.0 for j in S])
    logits = scale * (q_t @ k[S].T) + bias[None, :]
    return S, ret, logits


def prefill_relaxed_unit(q, k, v, m, sink: int, window: int, cap: int, scale: float, r,
                         rows=None, policy: str = CAP_RECENT):
    """Relaxed-retention prefill of one (batch element, KV head) unit: as
    ``prefill_unit``, with the logit of every key j in Ret_t raised by
    log r_j (r [T] > 0 on retained tokens: the retention scores; they also
    rank the tokens under policy "lowest").  Returns o [T, G, D], lse [T, G]."""
    q, k, v, r = _f64(q), _f64(k), _f64(v), _f64(r)
    T, G, D = q.shape
    o = np.full((T, G, v.shape[1]), np.nan)
    lse = np.full((T, G), np.nan)
    for t in (range(T) if rows is None else rows):
        S, _, logits = _relaxed_row(t, q[t], k, v, m, sink, window, cap, scale, r, policy, r)
        mx = logits.max(axis=1, keepdims=True)
        p = np.exp(logits - mx)
        l = p.sum(axis=1, keepdims=True)
        o[t] = (p @ v[S]) / l
        lse[t] = (mx + np.log(l))[:, 0]
    return o, lse


def prefill_relaxed_backward_unit(q, k, v, m, sink: int, window: int, cap: int, scale: float,
                                  do, r, policy: str = CAP_RECENT, o_out=None):
    """Gradients of L = sum_t <do_t, o_t> under relaxed retention, for one unit.

    Row by row, with P the softmax weights over S_t (logits with the log r
    bias) and o_t = P V_S:  dP = do_t V_S^T,  D_t = <do_t, o_t>,
    dS = P * (dP - D_t),  dq_t = scale dS K_S,  dk_S += scale dS^T q_t,
    dv_S += P^T do_t,  and for j in Ret_t:  dr_j += sum_g dS[g, j] / r_j.
    o_out: as in ``prefill_backward_unit`` (the stored output for D_t).
    Returns dq [T, G, D], dk [T, D], dv [T, D], dr [T] (float64)."""
    q, k, v, do, r = _f64(q), _f64(k), _f64(v), _f64(do), _f64(r)
    T, G, D = q.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dr = np.zeros(T)
    for t in range(T):
        S, ret, logits = _relaxed_row(t, q[t], k, v, m, sink, window, cap, scale, r, policy, r)
        P = np.exp(logits - logits.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        Vs, Ks = v[S], k[S]
        o = P @ Vs if o_out is None else _f64(o_out[t])
        dP = do[t] @ Vs.T
        Dt = (do[t] * o).sum(axis=1, keepdims=True)
        dS = P * (dP - Dt)
        dq[t] = scale * (dS @ Ks)
        dk[S] += scale * (dS.T @ q[t])
        dv[S] += P.T @ do[t]
        for c, j in enumerate(S):
            if j in ret:
                dr[j] += dS[:, c].sum() / r[j]
    return dq, dk, dv, dr


# ---------------------------------------------------------------------------
# (4) decode: the inference cache simulated slot by slot  [LTE, Fig. 3]
#     window as a FIFO of w slots  [SWA-LA, "Viewing SWA from the
#     linear-state perspective": one slot overwritten per token]
# ---------------------------------------------------------------------------

@dataclass
class DecodeCache:
    """Inference cache of one (batch element, KV head) unit, held literally.

    * window ring: w slots, token j lives in slot j mod w while in (t-w, t];
    * sink slots: s slots, token j < s moves to slot j when it leaves the window;
    * retained ring: C slots.  Policy "recent": the i-th retained token
      (0-based) goes to slot i mod C, overwriting the oldest one (the cap
      keeps the C most recent).  Policy "first": the i-th retained token goes
      to slot i while i < C and is dropped afterwards (ret_total then counts
      the stored tokens).  Policy "lowest": the i-th retained token goes to
      slot i while i < C; afterwards it replaces the held token with the
      lowest (score, position) unless its own score is lower (ret_total counts
      the stored tokens; ret_r holds their scores);
    * r of window tokens, filled by deferred batched scoring.
    """
    D: int
    sink: int
    window: int
    cap: int
    tau: float
    cnn: CNN | None
    score_batch: int
    win_k: np.ndarray = field(init=False)
    win_v: np.ndarray = field(init=False)
    win_pos: np.ndarray = field(init=False)
    win_r: np.ndarray = field(init=False)
    sink_k: np.ndarray = field(init=False)
    sink_v: np.ndarray = field(init=False)
    sink_pos: np.ndarray = field(init=False)
    ret_k: np.ndarray = field(init=False)
    ret_v: np.ndarray = field(init=False)
    ret_pos: np.ndarray = field(init=False)
    ret_r: np.ndarray = field(init=False)     # score of each retained slot's token
    ret_total: int = 0
    t: int = 0              # tokens received so far
    n_scored: int = 0       # tokens [0, n_scored) have a score
    fed: np.ndarray | None = None   # optional fed mask instead of the CNN
    policy: str = CAP_RECENT

    def __post_init__(self):
        w, s, C, D = self.window, self.sink, self.cap, self.D
        self.win_k = np.zeros((w, D)); self.win_v = np.zeros((w, D))
        self.win_pos = np.full(w, -1, dtype=np.int64); self.win_r = np.full(w, np.nan)
        self.sink_k = np.zeros((s, D)); self.sink_v = np.zeros((s, D))
        self.sink_pos = np.full(s, -1, dtype=np.int64)
        self.ret_k = np.zeros((C, D)); self.ret_v = np.zeros((C, D))
        self.ret_pos = np.full(C, -1, dtype=np.int64)
        self.ret_r = np.full(C, np.nan)

    # -- deferred scoring ---------------------------------------------------
    def _score_from_window(self, j: int) -> float:
        """r_j computed from the window ring alone; asserts that the whole
        receptive field [j-P, j+F] (clipped at 0) is inside the window."""
        if self.fed is not None:
            return 1.0 if self.fed[j] else 0.0
        P, F = self.cnn.past, self.cnn.future
        lo = max(0, j - P)            # positions before 0 do not exist (padding)
        n = j + F + 1 - lo
        ks = np.zeros((n, self.D)); vs = np.zeros((n, self.D))
        for i in range(lo, j + F + 1):
            slot = i % self.window
            assert self.win_pos[slot] == i, "receptive field left the window before scoring"
            ks[i - lo] = self.win_k[slot]
            vs[i - lo] = self.win_v[slot]
        r = cnn_scores(ks, vs, self.cnn)
        return float(r[j - lo])

    def _maybe_score(self):
        """Score the oldest `score_batch` scorable tokens once that many are
        scorable (a token j is scorable when j + F < t)."""
        F = 0 if self.cnn is None else self.cnn.future
        last_scorable = self.t - 1 - F
        while last_scorable - self.n_scored + 1 >= self.score_batch:
            for j in range(self.n_scored, self.n_scored + self.score_batch):
                self.win_r[j % self.window] = self._score_from_window(j)
            self.n_scored += self.score_batch

    # -- one token arrives ----------------------------------------------------
    def append(self, k_t, v_t):
        """Token t = self.t arrives: token t-w leaves the window first."""
        t, w = self.t, self.window
        leaving = t - w
        if leaving >= 0:
            slot = leaving % w
            assert self.win_pos[slot] == leaving
            if leaving < self.sink:
                self.sink_k[leaving] = self.win_k[slot]
                self.sink_v[leaving] = self.win_v[slot]
                self.sink_pos[leaving] = leaving
            else:
                assert leaving < self.n_scored, "token left the window unscored"
                r = self.win_r[slot]
                keep = r >= self.tau and self.cap > 0
                rs = self.ret_total % self.cap if self.cap > 0 else 0
                full = self.ret_total >= self.cap
                if keep and self.policy == CAP_FIRST and full:
                    keep = False                     # the segment is full: dropped
                if keep and self.policy == CAP_LOWEST and full:
                    # drop the lowest (score, position) of the held tokens and the
                    # newcomer; the newcomer is the latest, so it stays iff its
                    # score is not below the lowest held score
                    rs = min(range(self.cap), key=lambda i: (self.ret_r[i], self.ret_pos[i]))
                    keep = r >= self.ret_r[rs]
                if keep:
                    self.ret_k[rs] = self.win_k[slot]
                    self.ret_v[rs] = self.win_v[slot]
                    self.ret_pos[rs] = leaving
                    self.ret_r[rs] = r
                    if not (self.policy == CAP_LOWEST and full):
                        self.ret_total += 1
        slot = t % w
        self.win_k[slot] = _f64(k_t); self.win_v[slot] = _f64(v_t)
        self.win_pos[slot] = t; self.win_r[slot] = np.nan
        self.t = t + 1
        self._maybe_score()

    def retained_positions(self) -> list[int]:
        return sorted(int(p) for p in self.ret_pos if p >= 0)

    def keys(self):
        """All valid (position, k, v) of the cache, position-sorted."""
        items = []
        for i in range(self.window):
            if self.win_pos[i] >= 0:
                items.append((int(self.win_pos[i]), self.win_k[i], self.win_v[i]))
        for i in range(self.sink):
            if self.sink_pos[i] >= 0:
                items.append((int(self.sink_pos[i]), self.sink_k[i], self.sink_v[i]))
        for i in range(self.cap):
            if self.ret_pos[i] >= 0:
                items.append((int(self.ret_pos[i]), self.ret_k[i], self.ret_v[i]))
        items.sort(key=lambda it: it[0])
        return items

    def attend(self, q_rows, scale: float):
        """Attention of the newest token's G query rows over the cache."""
        items = self.keys()
        K = np.stack([it[1] for it in items])
        V = np.stack([it[2] for it in items])
        o, lse = attend(q_rows, K, V, scale)
        return o, lse, [it[0] for it in items]


def decode_unit(q, k, v, T0: int, sink: int, window: int, cap: int, tau: float,
                cnn: CNN | None, score_batch: int, scale: float, fed=None,
                policy: str = CAP_RECENT):
    """Feed tokens 0..T-1 of one unit through the cache; for every token
    t >= T0 return its attention output, lse and attended positions.

    q [T, G, D], k, v [T, D].  The prompt (t < T0) goes through the same
    cache updates as decoding (no attention output is kept for it).
    """
    cache = DecodeCache(D=k.shape[1], sink=sink, window=window, cap=cap, tau=tau,
                        cnn=cnn, score_batch=score_batch, policy=policy)
    cache.fed = None if fed is None else np.asarray(fed)
    outs, lses, sets, rets = [], [], [], []
    for t in range(k.shape[0]):
        cache.append(k[t], v[t])
        if t >= T0:
            o, lse, pos = cache.attend(q[t], scale)
            outs.append(o); lses.append(lse); sets.append(pos)
            rets.append(cache.retained_positions())
    return np.array(outs), np.array(lses), sets, rets, cache


def cache_after_prompt(k, v, m, T0: int, sink: int, window: int, cap: int,
                       policy: str = CAP_RECENT, r=None):
    """The cache contents after a prompt of T0 tokens, read off the prefill
    mask: window = positions (T0-1-w, T0-1], sinks = j < s with j <= T0-1-w,
    retained = the C most recent j in [s, T0-1-w] with m_j = 1, with the
    i-th retained token (0-based over all retained) in ring slot i mod C
    (policy "first": the C earliest such j, the i-th in slot i, and ret_total
    counts the stored ones; policy "lowest": the C such j with the highest
    scores, in position order in slots 0, 1, ..., ret_total = their number).

    Returns dict of position arrays (-1 = empty) and ret_total.
    """
    last_out = T0 - 1 - window
    win_pos = np.full(window, -1, dtype=np.int64)
    for j in range(max(0, T0 - window), T0):
        win_pos[j % window] = j
    sink_pos = np.full(sink, -1, dtype=np.int64)
    for j in range(min(sink, last_out + 1)):
        sink_pos[j] = j
    ret = [j for j in range(sink, last_out + 1) if m[j]]
    if policy == CAP_FIRST:
        ret = ret[:cap]
    elif policy == CAP_LOWEST:
        ret = sorted(top_by_score(ret, r, cap))
    ret_pos = np.full(cap, -1, dtype=np.int64)
    for i, j in enumerate(ret):
        if cap > 0:
            ret_pos[i % cap] = j
    return {"win_pos": win_pos, "sink_pos": sink_pos, "ret_pos": ret_pos,
            "ret_total": len(ret)}
