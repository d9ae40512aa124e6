/*
 * lte_api.h -- C ABI of the B200 (sm_100a) library for contextualized
 * Learnable Token Eviction (LTE), the sparse-attention token mixer of the
 * laLTE linear/sparse hybrid.
 *
 * Source of the method: "Alleviating Forgetfulness of Linear Attention by
 * Hybrid Sparse Attention and Contextualized Learnable Token Eviction"
 * (He & Garner, 2025): TL;DR and Abstract (a lightweight CNN over past and
 * future neighbouring KVs predicts per-head retention; combined with an
 * attention sink and sliding-window attention; constant time and space per
 * step), Figure 2 caption (retention score r_{j,h} decides eviction when a
 * KV pair leaves the window; the score can be computed once the CNN's
 * receptive field is inside the window; per-head "A-plus-column" pattern),
 * Figure 3 caption (inference cache = circular window segment + capped
 * out-of-window segment holding sink and retained KVs; scoring batched and
 * deferred).  The companion linear layer follows "Sparse Linear Attention:
 * Viewing SWA from the Perspective of Linear Attention", section
 * "Background: Linear attention" (state update equation).
 *
 * Conventions for every call
 *  - All tensor arguments are DEVICE pointers owned by the caller; the
 *    library allocates no memory (scratch comes in `workspace`, sized by
 *    lte_workspace_bytes) and synchronises nothing except
 *    lte_read_device_error.  Every call enqueues its kernels on `stream`
 *    (a cudaStream_t passed as void*; NULL = legacy default stream) and
 *    returns immediately.
 *  - Layouts are row-major.  Activations are [B, T, H, D] with the D
 *    dimension contiguous; `lte_strides` gives the other three element
 *    strides (NULL = contiguous).  Pointers must be 16-byte aligned and
 *    strides multiples of 16 bytes.
 *  - Notation: B batch, T tokens, Hq query heads, Hkv KV heads, G = Hq/Hkv,
 *    D head dim, s sink, w window, C cap, tau threshold.  Query head q uses
 *    KV head q / G.
 *  - Errors: arguments are validated on the host before any launch; an
 *    invalid call returns a non-zero lte_status and launches nothing.  A
 *    failed launch returns LTE_ERR_CUDA.  Conditions only the device can see
 *    (a bounded wait that ran out, an index out of range) are recorded in
 *    the first 16 bytes of the workspace and read by lte_read_device_error.
 *    Nothing aborts the process.
 */
#ifndef LTE_API_H
#define LTE_API_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LTE_OK = 0,
  LTE_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or parameter */
  LTE_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. D not in {64,128}) */
  LTE_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed */
  LTE_ERR_TIMEOUT = 4,       /* a device-side bounded wait ran out */
  LTE_ERR_WORKSPACE = 5,     /* workspace missing or smaller than required */
  LTE_ERR_DEVICE = 6         /* a device-side check failed (see error word) */
} lte_status;

typedef enum { LTE_F32 = 0, LTE_BF16 = 1 } lte_dtype;

/* Which retained tokens the capped out-of-window segment keeps once more
 * than C qualify.  [LTE paper, Fig. 3 caption: the segment has capped
 * capacity; the pages leave the policy open.]
 *   LTE_CAP_RECENT: the C most recent (a ring; the oldest is overwritten);
 *   LTE_CAP_FIRST:  the first C (later retained tokens are dropped once the
 *                   segment is full);
 *   LTE_CAP_LOWEST: when a retained token arrives at a full segment, the
 *                   token with the lowest (score r, position) among the C
 *                   held and the newcomer is dropped -- equal scores drop the
 *                   older token.  The segment then holds the C retained
 *                   tokens with the highest (r, position) so far.  Needs the
 *                   scores: prefill takes lifetimes from
 *                   lte_retained_lifetimes, the decode cache its ret_r. */
typedef enum { LTE_CAP_RECENT = 0, LTE_CAP_FIRST = 1, LTE_CAP_LOWEST = 2 } lte_cap_policy;

/* Shapes and method parameters of one LTE layer.
 * sink = s >= 0, window = w >= 1, cap = C >= 0 (retained tokens only; sinks
 * are extra), tau = retention threshold (retain iff r >= tau), scale =
 * softmax scale (1/sqrt(D) in the usual setting), dtype of q/k/v/o/caches,
 * cap_policy = lte_cap_policy (0, the C most recent, when zero-initialised). */
typedef struct {
  int32_t B, T, Hq, Hkv, D;
  int32_t sink, window, cap;
  float tau, scale;
  int32_t dtype;
  int32_t cap_policy;
} lte_dims;

/* Element strides of a [B, T, H, D] tensor (D stride is 1). */
typedef struct { int64_t b, t, h; } lte_strides;

/* Weights of the per-KV-head scoring CNN (device pointers, fp32):
 *   w1 [Hkv, c_hid, 2D, k1], b1 [Hkv, c_hid], w2 [Hkv, c_hid, k2], b2 [Hkv].
 * Layer l reads past_l tokens before and (k_l - 1 - past_l) after the output
 * token (PyTorch conv1d cross-correlation, zero padding outside the
 * sequence); input channels are [k; v] (k first).  r_j depends on tokens
 * [j - P, j + F] with P = past1 + past2, F = (k1-1-past1) + (k2-1-past2).
 * Supported: c_hid <= 64, k1 <= 9, k2 <= 9. */
typedef struct {
  int32_t c_hid, k1, past1, k2, past2;
  const float *w1, *b1, *w2, *b2;
} lte_cnn;

/* ---------------------------------------------------------------------------
 * lte_score -- retention scores r_{j,h} of tokens j in [j_begin, j_end).
 * [LTE paper, Fig. 2 caption: CNN stack over short-range past and future
 * context; TL;DR: per-head retention scores.]
 *   layer 1: u[c,j] = SiLU(b1[c] + sum_{ch<2D, kk<k1} w1[c,ch,kk] x[ch, j+kk-past1])
 *   layer 2: r[j]   = sigmoid(b2 + sum_{c, kk<k2} w2[c,kk] u[c, j+kk-past2])
 * k, v: [B,T,Hkv,D] (dtype), kv_strides may be NULL.  Requires
 * 0 <= j_begin <= j_end <= T - F (the receptive field must be complete).
 * r: fp32 [B, Hkv, T]; mask (nullable): uint8 [B, Hkv, T], written as
 * (j >= sink) && (r >= tau).  Only positions [j_begin, j_end) are written.
 * Arithmetic: fp32 accumulation in a fixed per-output order (results do not
 * depend on j_begin/j_end or on the launch).
 * ------------------------------------------------------------------------- */
lte_status lte_score(const lte_dims* d, const lte_cnn* cnn,
                     const void* k, const void* v, const lte_strides* kv_strides,
                     int32_t j_begin, int32_t j_end,
                     float* r, uint8_t* mask, void* stream);

/* ---------------------------------------------------------------------------
 * lte_score_backward -- gradients through the scoring CNN, given dL/dr.
 * [LTE paper, Abstract: trained end to end; Fig. 2 caption: the CNN.  The
 * pages give no rule for dL/dr (the eviction decision is discrete), so it is
 * an input.]  With r computed as in lte_score over the whole sequence (each
 * layer's input 0 outside [0, T)) and L = sum_{j < n_scored} dr[j] r[j]:
 *   dk, dv (fp32 [B,T,Hkv,D], contiguous): dL/dk, dL/dv ADDED to their
 *          contents (so the attention backward's gradients can be summed in);
 *   dw1 [Hkv,c_hid,2D,k1], db1 [Hkv,c_hid], dw2 [Hkv,c_hid,k2], db2 [Hkv]
 *          (fp32): dL/dweights summed over the batch, OVERWRITTEN.
 * k, v as in lte_score (kv_strides may be NULL); dr: fp32 [B,Hkv,T], entries
 * j >= n_scored ignored; 0 <= n_scored <= T - F.  Arithmetic: fp32 throughout,
 * except that for bf16 inputs with head dim 128 and c_hid 32 the three
 * contractions (the layer-1 recompute, dx and dw1) run on tcgen05 tensor
 * cores with fp32 operands split into bf16 hi + lo pairs (relative error
 * about 2^-16) and fp32 accumulation; elsewhere fp32 CUDA-core kernels.  The
 * weight gradients add fp32 partial sums with atomics (last bits may vary).
 * Workspace: lte_score_backward_workspace_bytes(d, cnn) bytes (error word,
 * 2 x B x Hkv x c_hid x T floats, and on the tensor-core path the hidden
 * gradient again as two bf16 planes).
 * ------------------------------------------------------------------------- */
size_t lte_score_backward_workspace_bytes(const lte_dims* d, const lte_cnn* cnn);
lte_status lte_score_backward(const lte_dims* d, const lte_cnn* cnn, const void* k, const void* v,
                              const lte_strides* kv_strides, int32_t n_scored, const float* dr,
                              float* dk, float* dv, float* dw1, float* db1, float* dw2, float* db2,
                              void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * lte_evict_compact -- eviction decision and compaction of retained tokens.
 * [LTE paper, Fig. 2 caption: a KV pair is kept or evicted when it moves out
 * of the window; Fig. 3 caption: capped out-of-window segment with sink and
 * retained KVs.]
 * m_j = (j >= sink) && (j < n_scored) && (mask ? mask[j] != 0 : r[j] >= tau);
 * exactly one of r / mask is non-NULL ([B,Hkv,T]).
 * Outputs (per (b, KV head) unit):
 *   idx  int32 [B,Hkv,T]: ascending positions j with m_j = 1 (first nret valid),
 *   nret int32 [B,Hkv]:   number of such positions,
 *   cnt  int32 [B,Hkv,T]: inclusive prefix count cnt[j] = #{i <= j : m_i}.
 * Column segment (k_col, v_col both NULL or both set): [B, Hkv, sink + T, D]
 * contiguous, slot i < sink holds the sink row k[i] (zeros for i >= T),
 * slot sink + i holds k[idx[i]] for i < nret, and the next 64 slots (those
 * within the segment) are zeros, so that every 64-row tile the attention
 * kernels read holds finite values; likewise for v.  Later slots are left
 * unwritten.
 * ------------------------------------------------------------------------- */
lte_status lte_evict_compact(const lte_dims* d, const float* r, const uint8_t* mask,
                             int32_t n_scored, int32_t* idx, int32_t* nret, int32_t* cnt,
                             const void* k, const void* v, const lte_strides* kv_strides,
                             void* k_col, void* v_col, void* stream);

/* ---------------------------------------------------------------------------
 * lte_retained_lifetimes -- for LTE_CAP_LOWEST, the retained counts during
 * which each retained token is held.  [LTE paper, Fig. 3 caption: capped
 * out-of-window segment; the drop-the-lowest-score reading of the cap.]
 * Token i of the compacted list (0-based, position idx[i], score
 * r[idx[i]]) is beaten by token i' != i when r[idx[i']] > r[idx[i]], or the
 * scores are equal and i' > i.  Then, per (b, KV head) unit:
 *   death[i] = the smallest n > i such that at least C of the tokens
 *              0 .. n-1 beat token i, or T + 1 if there is none;
 * the segment holds token i exactly while the retained count n satisfies
 * i < n < death[i].  r: fp32 [B,Hkv,T] (the scores behind the mask);
 * idx, nret from lte_evict_compact; death: int32 [B,Hkv,T], entries
 * i >= nret left unwritten.  Requires d->cap_policy == LTE_CAP_LOWEST.
 * Work: O(nret^2) comparisons per unit, none when nret <= C.
 * ------------------------------------------------------------------------- */
lte_status lte_retained_lifetimes(const lte_dims* d, const float* r, const int32_t* idx,
                                  const int32_t* nret, int32_t* death, void* stream);

/* ---------------------------------------------------------------------------
 * lte_sparse_attn_prefill -- causal softmax attention of every query over its
 * per-KV-head attended set.  [LTE paper, Fig. 2 caption (right): per-head
 * A-plus-column sparsity pattern: sink and window form the "A", retained
 * tokens the "columns".]
 * For row t, KV head h, n_t = (t >= w) ? cnt[t - w] : 0:
 *   S_t = { j < s : j <= t - w }  u  (t - w, t]  u  { idx[i] : i in R_t }, where
 *   R_t = [max(0, n_t - C), n_t)               under LTE_CAP_RECENT,
 *         [0, min(n_t, C))                     under LTE_CAP_FIRST,
 *         { i < n_t : death[i] > n_t }         under LTE_CAP_LOWEST;
 *   o[t,q] = sum_{j in S_t} softmax_j(scale * q_t . k_j) v_j,
 *   lse[q,t] = log sum_{j in S_t} exp(scale * q_t . k_j)   (natural log).
 * q, o: [B,T,Hq,D]; k, v: [B,T,Hkv,D]; cnt from lte_evict_compact; k_col,
 * v_col: the column segment written by lte_evict_compact (required); death:
 * from lte_retained_lifetimes, required under LTE_CAP_LOWEST, else ignored.
 * Under LTE_CAP_LOWEST every row scans retained slots [0, n_t), so its cost
 * grows with n_t rather than with C once the cap binds.
 * lse (nullable): fp32 [B,Hq,T].  bf16 inputs: fp32 accumulation, P rounded
 * to bf16 for the PV product, o rounded to bf16 (round-to-nearest-even).
 * Workspace: lte_workspace_bytes(d, LTE_WS_PREFILL) bytes (16-byte aligned,
 * caller-owned; it holds the device error word).
 * ------------------------------------------------------------------------- */
lte_status lte_sparse_attn_prefill(const lte_dims* d, const void* q, const void* k,
                                   const void* v, const lte_strides* q_strides,
                                   const lte_strides* kv_strides, const int32_t* cnt,
                                   const int32_t* death, const void* k_col, const void* v_col,
                                   void* o, const lte_strides* o_strides, float* lse,
                                   void* workspace, size_t ws_bytes, void* stream);

/* Which kernel family a call runs.  Every family is GPU code and gives the
 * same results within the stated tolerances; they differ in speed. */
typedef enum {
  LTE_KERNEL_TCGEN05 = 1,   /* 5th-generation tensor cores (tcgen05, TMEM, TMA) */
  LTE_KERNEL_MMA_SYNC = 2,  /* warp-level mma.sync tensor-core kernels (slower) */
  LTE_KERNEL_SIMT = 3       /* fp32 CUDA-core kernels (fp32 inputs) */
} lte_kernel_kind;

/* lte_sparse_attn_prefill_kernel -- the kernel family lte_sparse_attn_prefill
 * would run for these dims and strides (same meaning as in that call; NULL =
 * contiguous), written to *kind.  The tcgen05 kernel serves bf16 with head
 * dim 128, G in {1,2,4,8,16} and byte strides that are multiples of 16; other
 * bf16 shapes run the mma.sync kernel, fp32 runs the SIMT kernel.  Host only:
 * launches nothing.  Errors: LTE_ERR_INVALID_ARG / LTE_ERR_UNSUPPORTED as the
 * call itself would return for these dims and strides. */
lte_status lte_sparse_attn_prefill_kernel(const lte_dims* d, const lte_strides* q_strides,
                                          const lte_strides* kv_strides,
                                          const lte_strides* o_strides, int32_t* kind);

/* ---------------------------------------------------------------------------
 * lte_sparse_attn_backward -- gradients of the prefill sparse attention with
 * the attended sets held fixed.  [LTE paper, Abstract: the hybrids are
 * trained end to end; the pages give no gradient for the eviction decisions,
 * so S_t (as in lte_sparse_attn_prefill) is fixed and only the softmax
 * attention over it is differentiated.]  With P the softmax weights of row t
 * (recomputed from lse), o the forward output and dO its incoming gradient:
 *   D_t = <dO_t, o_t>,  dS = P * (dO V^T - D_t),
 *   dq = scale dS K,  dk = scale dS^T Q,  dv = P^T dO,
 * summed, for dk and dv, over the G query heads of a KV head and over every
 * way a position is attended (window band, sink slot, retained slot).
 * q, o, dO: [B,T,Hq,D] bf16 contiguous; k, v: [B,T,Hkv,D] bf16 contiguous;
 * cnt, idx, nret, k_col, v_col: from lte_evict_compact (the column segment
 * is required); death: from lte_retained_lifetimes, required under
 * LTE_CAP_LOWEST, else ignored; o and lse (natural log, [B,Hq,T]): from
 * lte_sparse_attn_prefill on the same inputs.
 * Outputs (overwritten): dq fp32 [B,T,Hq,D], dk, dv fp32 [B,T,Hkv,D].
 * Arithmetic: fp32 accumulation; P and dS rounded to bf16 for the products;
 * dk and dv of retained and sink positions add fp32 partial sums with
 * atomics, so their last bits may vary between runs.
 * bf16 only, G = Hq/Hkv dividing 64 (else LTE_ERR_UNSUPPORTED).
 * Workspace: lte_workspace_bytes(d, LTE_WS_BACKWARD) (error word + D_t).
 * ------------------------------------------------------------------------- */
lte_status lte_sparse_attn_backward(const lte_dims* d, const void* q, const void* k, const void* v,
                                    const int32_t* cnt, const int32_t* death, const int32_t* idx,
                                    const int32_t* nret, const void* k_col, const void* v_col,
                                    const void* o, const float* lse, const void* dO, float* dq,
                                    float* dk, float* dv, void* workspace, size_t ws_bytes,
                                    void* stream);

/* ---------------------------------------------------------------------------
 * Relaxed retention for training.  [LTE paper, Abstract: the model, CNN
 * included, is trained end to end; Fig. 2 caption: the score r_{j,h} decides
 * whether a KV pair is kept.  The pages give no rule for how the loss reaches
 * r; the reading taken here:]  the attended sets stay the hard ones (as in
 * lte_sparse_attn_prefill: r >= tau, the cap policy), and every key j that
 * row t attends through the retained segment (j in R_t's positions) enters
 * the softmax with weight r_j -- its logit gains log r_j.  Sink and window
 * keys are unweighted.  With r = 1 the calls equal the hard ones.
 *
 * lte_sparse_attn_prefill_relaxed -- o and lse as lte_sparse_attn_prefill
 * with those weights:
 *   o[t,q] = sum_{j in S_t} w_j exp(scale q_t.k_j) v_j / sum_{j in S_t} w_j exp(scale q_t.k_j),
 *   lse[q,t] = log sum_{j in S_t} w_j exp(scale q_t.k_j),  w_j = r_j on retained
 *   keys, 1 otherwise.
 * lte_sparse_attn_backward_relaxed -- dq, dk, dv as lte_sparse_attn_backward
 * for that forward, and
 *   dr[j] = sum over rows t (and their G query heads) attending j through
 *           the retained segment of dS_{t,j} / r_j   (dS: dL/dlogit),
 *   dr: fp32 [B,Hkv,T], OVERWRITTEN (0 where no row attends j that way) --
 *   the dL/dr that lte_score_backward takes.
 * Arguments as in lte_sparse_attn_prefill / lte_sparse_attn_backward with
 * contiguous [B,T,H,D] layouts, plus r: fp32 [B,Hkv,T] > 0 on retained tokens
 * (clamped below at 1e-30; the scores behind the mask, e.g. from lte_score)
 * and idx, nret from lte_evict_compact.  Supported: bf16, head dim 128,
 * G in {1,2,4,8,16} (tcgen05 kernels), else LTE_ERR_UNSUPPORTED.
 * Workspace: lte_workspace_bytes(d, LTE_WS_RELAXED) (error word, per-slot log
 * weights, D_t); the calls share nothing through it.  dk, dv of retained and
 * sink positions and dr add fp32 partial sums with atomics.
 * ------------------------------------------------------------------------- */
lte_status lte_sparse_attn_prefill_relaxed(const lte_dims* d, const void* q, const void* k,
                                           const void* v, const int32_t* cnt, const int32_t* death,
                                           const int32_t* idx, const int32_t* nret,
                                           const void* k_col, const void* v_col, const float* r,
                                           void* o, float* lse, void* workspace, size_t ws_bytes,
                                           void* stream);
lte_status lte_sparse_attn_backward_relaxed(const lte_dims* d, const void* q, const void* k,
                                            const void* v, const int32_t* cnt,
                                            const int32_t* death, const int32_t* idx,
                                            const int32_t* nret, const void* k_col,
                                            const void* v_col, const float* r, const void* o,
                                            const float* lse, const void* dO, float* dq,
                                            float* dk, float* dv, float* dr, void* workspace,
                                            size_t ws_bytes, void* stream);

/* lte_sparse_attn_backward_kernel -- the kernel family lte_sparse_attn_backward
 * would run for these dims (*kind): LTE_KERNEL_TCGEN05 for head dim 128,
 * LTE_KERNEL_MMA_SYNC for head dim 64.  Host only.  Errors as the call's. */
lte_status lte_sparse_attn_backward_kernel(const lte_dims* d, int32_t* kind);

/* ---------------------------------------------------------------------------
 * Decode cache.  [LTE paper, Fig. 3 caption: circular window segment plus an
 * out-of-window segment of capped capacity for sink and retained KVs;
 * "Sparse Linear Attention ...", section "Viewing SWA from the linear-state
 * perspective": the window as a FIFO of slots.]
 * All buffers are caller-owned device memory; L = window + sink + cap slots.
 *   k, v     [B, Hkv, L, D] (dtype): slots [0,w) window ring (token j in slot
 *            j mod w), [w, w+s) sinks (token j < s in slot w+j once it left
 *            the window), [w+s, w+s+C) retained ring (the i-th retained token
 *            of the unit, 0-based, in slot w+s+(i mod C); under
 *            LTE_CAP_FIRST and LTE_CAP_LOWEST slots fill in order and never
 *            wrap, and under LTE_CAP_LOWEST a newcomer takes the slot of the
 *            token it displaces);
 *   pos      int32 [B, Hkv, L]: token position held by each slot, -1 = empty;
 *   win_r    fp32  [B, Hkv, w]: score of the token in each window slot;
 *   ret_total int32 [B, Hkv]: tokens retained so far (the ring's write count;
 *            the number held, at most C, under LTE_CAP_FIRST / LOWEST);
 *   meta     int32 [4]: {t = tokens held so far, n_scored = tokens [0,n_scored)
 *            have a score, internal, internal};
 *   ret_r    fp32  [B, Hkv, C]: score of the token in each retained slot
 *            (required under LTE_CAP_LOWEST, else may be NULL). */
typedef struct {
  void *k, *v;
  int32_t* pos;
  float* win_r;
  int32_t* ret_total;
  int32_t* meta;
  float* ret_r;
} lte_cache;

/* lte_cache_init_from_prefill -- fill an empty cache with the state after a
 * prompt of T_prompt tokens (T_prompt <= d->T):
 * window = tokens (T_prompt-1-w, T_prompt-1], sinks that left the window,
 * with n = cnt[T_prompt-1-w] (0 if negative) the retained tokens are
 *   LTE_CAP_RECENT: idx[max(0,n-C) .. n), the i-th in ring slot i mod C,
 *                   ret_total = n;
 *   LTE_CAP_FIRST:  idx[0 .. min(n,C)), in slots 0, 1, ..., ret_total = min(n,C);
 *   LTE_CAP_LOWEST: idx[i] for i < n with death[i] > n, in that order in
 *                   slots 0, 1, ..., with ret_r = their scores and
 *                   ret_total = their number;
 * win_r = r of window tokens below n_scored (NaN otherwise),
 * meta = {T_prompt, n_scored, 0, 0}.
 * k, v [B,T,Hkv,D]; r [B,Hkv,T] from lte_score; idx, cnt from
 * lte_evict_compact run with the same n_scored; death (LTE_CAP_LOWEST only,
 * else ignored) from lte_retained_lifetimes. */
lte_status lte_cache_init_from_prefill(const lte_dims* d, const lte_cache* cache,
                                       const void* k, const void* v,
                                       const lte_strides* kv_strides, const float* r,
                                       const int32_t* idx, const int32_t* cnt,
                                       const int32_t* death,
                                       int32_t T_prompt, int32_t n_scored, void* stream);

/* lte_decode_step -- one generated token for every sequence in the batch.
 * Reads t = meta[0] on the device (no host synchronisation), then:
 *  (1) token t-w leaves the window: a sink (t-w < s) moves to its sink slot;
 *      otherwise it enters the retained segment iff win_r >= tau and C > 0,
 *      else it is dropped.  When the segment is full, LTE_CAP_RECENT
 *      overwrites the oldest, LTE_CAP_FIRST drops the newcomer, and
 *      LTE_CAP_LOWEST replaces the held token with the lowest (ret_r, pos)
 *      if win_r is not below that score (else drops the newcomer);
 *  (2) the new token is written to window slot t mod w;
 *  (3) deferred batched scoring: once score_batch tokens are scorable
 *      (j + F <= t), the oldest score_batch unscored tokens are scored from
 *      the window segment (same arithmetic as lte_score);
 *  (4) attention of q_t over every valid slot (split over the keys, merged
 *      with log-sum-exp), o_t and lse_t written;  meta[0] = t + 1.
 * q_t, o_t: [B, Hq, D]; k_t, v_t: [B, Hkv, D]; lse_t (nullable) fp32 [B, Hq].
 * Requires 1 <= score_batch <= w - P - F (every token is scored before it
 * leaves the window).  Workspace: lte_workspace_bytes(d, LTE_WS_DECODE).
 * The same kernels run every step, so a step can be captured in a CUDA graph
 * and replayed. */
lte_status lte_decode_step(const lte_dims* d, const lte_cnn* cnn, const lte_cache* cache,
                           const void* q_t, const void* k_t, const void* v_t,
                           void* o_t, float* lse_t, int32_t score_batch,
                           void* workspace, size_t ws_bytes, void* stream);

/* lte_decode_step_noalloc -- lte_decode_step for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is a library
 * convenience.  Some callers are not allowed to call cudaMalloc: a host
 * runtime that has reserved the whole device for its own memory pool and
 * hands a plugin only its input and output buffers, or a latency-critical
 * loop where the device-wide synchronisation a cudaMalloc can imply is not
 * acceptable.  This entry point takes the same arguments minus the workspace
 * and keeps its scratch (error word, split partials, completion counters)
 * in one file-scope device array of LTE_NOALLOC_SCRATCH_BYTES bytes, which
 * every GPU that loads the library holds until the process exits.  It calls
 * no cudaMalloc, cudaFree or other allocating routine.
 *  - Limit: returns LTE_ERR_WORKSPACE, launching nothing, when
 *    lte_workspace_bytes(d, LTE_WS_DECODE) > LTE_NOALLOC_SCRATCH_BYTES
 *    (the decode workload -- B*Hkv = 128 units, 1028 cache slots, G = 4,
 *    D = 128 -- needs about 0.3 MB).
 *  - Set-up: the first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Sharing: all calls on a device share the one array and it keeps the
 *    last call's contents; every call zeroes the error word and the counters
 *    it relies on.  Calls that overlap on the GPU (e.g. on two streams at
 *    once) race on the array: serialise them.
 *  - Device errors: the error word lives in the array too; every call
 *    clears it first, and lte_noalloc_read_device_error reads it.  Check it
 *    after a call (before the next one clears it) as you would check a
 *    workspace with lte_read_device_error.
 *  - The cached address belongs to the device's primary context.  After
 *    cudaDeviceReset (or anything else that destroys that context) the entry
 *    point must not be called again in this process.
 *  - Results are the same as lte_decode_step's (same kernels). */
#define LTE_NOALLOC_SCRATCH_BYTES (4u << 20)
lte_status lte_decode_step_noalloc(const lte_dims* d, const lte_cnn* cnn, const lte_cache* cache,
                                   const void* q_t, const void* k_t, const void* v_t,
                                   void* o_t, float* lse_t, int32_t score_batch, void* stream);

/* lte_noalloc_read_device_error -- the device error word of the last
 * lte_decode_step_noalloc call on the current device: synchronises `stream`,
 * then *code = 0 or LTE_ERR_TIMEOUT / LTE_ERR_DEVICE and *where = the id of
 * the wait or check that failed (where may be NULL).  Allocates nothing.
 * Errors: LTE_ERR_INVALID_ARG (code NULL), LTE_ERR_CUDA. */
lte_status lte_noalloc_read_device_error(int32_t* code, int32_t* where, void* stream);

enum { LTE_WS_PREFILL = 0, LTE_WS_DECODE = 1, LTE_WS_BACKWARD = 2, LTE_WS_RELAXED = 3 };

/* Bytes of workspace a call needs (>= 16: the first 16 bytes hold the device
 * error word).  Returns 0 for invalid dims. */
size_t lte_workspace_bytes(const lte_dims* d, int32_t which);

/* Zero the error word of a workspace (enqueued on stream). */
lte_status lte_clear_device_error(void* workspace, void* stream);

/* Synchronise `stream`, then copy the workspace's error word to the host:
 * *code = 0 if no device-side check failed, else LTE_ERR_TIMEOUT or
 * LTE_ERR_DEVICE; *where = the id of the wait or check that failed. */
lte_status lte_read_device_error(const void* workspace, int32_t* code, int32_t* where,
                                 void* stream);

/* lte_wait_probe -- diagnostic: shows on the live device that a bounded wait
 * ends in an error status instead of a hang.  The pages have no counterpart;
 * it exercises the failure path of the library's device waits (the bounded
 * mbarrier wait of the fused decode step).  One small kernel: a thread
 * arrives on an mbarrier once the device word *flag equals `expect`, another
 * waits for that barrier for at most limit_ns.  If the flag never holds
 * `expect`, the wait runs out after ~limit_ns, LTE_ERR_TIMEOUT is recorded in
 * the workspace's error word (read it with lte_read_device_error) and the
 * kernel returns; otherwise the error word is left as it was.
 * flag: device int32, 4-byte aligned, read only.  limit_ns in [1e3, 1e10].
 * workspace: any workspace of >= 16 bytes (only its error word is used).
 * Errors: LTE_ERR_INVALID_ARG (flag, limit), LTE_ERR_WORKSPACE, LTE_ERR_CUDA. */
lte_status lte_wait_probe(const int32_t* flag, int32_t expect, int64_t limit_ns, void* workspace,
                          void* stream);

/* ---------------------------------------------------------------------------
 * Gated linear attention, the hybrid's companion layer.  ["Sparse Linear
 * Attention: Viewing SWA from the Perspective of Linear Attention", section
 * "Background: Linear attention": the state is decayed, the value-key outer
 * product is written, the query reads; the decay here is diag(a_t).]
 *   S_t = S_{t-1} diag(a_t) + v_t k_t^T,  o_t = S_t q_t.
 * q, k: [B,T,H,dk]; v, o: [B,T,H,dv] (dtype); a: fp32 [B,T,H,dk] in [0,1];
 * state: fp32 [B,H,dv,dk], read as S_0 and overwritten with S_T.
 * Supported: dk = dv = 128; prefill bf16 with T % 64 == 0 (chunk-wise, 64
 * tokens per chunk, bf16 operands with fp32 accumulation and an fp32 state);
 * decode bf16 or fp32 (one step, fp32 arithmetic).  Other shapes return
 * LTE_ERR_UNSUPPORTED.  Any gate in [0, 1] is accepted.  The chunk form
 * multiplies q and k by products of up to 32 gates (or their reciprocals);
 * a chunk in which some channel's product of 32 gates falls below 2^-100 runs
 * the recurrence token by token instead (fp32 state, same result within the
 * stated tolerance, slower for that chunk).
 * ------------------------------------------------------------------------- */
lte_status lte_gla_prefill(int32_t B, int32_t T, int32_t H, int32_t dk, int32_t dv,
                           int32_t dtype, const void* q, const void* k, const void* v,
                           const float* a, void* o, float* state, void* stream);

lte_status lte_gla_decode_step(int32_t B, int32_t H, int32_t dk, int32_t dv, int32_t dtype,
                               const void* q_t, const void* k_t, const void* v_t,
                               const float* a_t, void* o_t, float* state, void* stream);

/* Library version string (static storage). */
const char* lte_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LTE_API_H */
