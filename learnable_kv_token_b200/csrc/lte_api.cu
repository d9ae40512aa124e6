// C-ABI entry points: host-side validation, then kernel dispatch.
// Every call validates before it launches anything and never synchronises
// (except lte_read_device_error); see lte_api.h for the contract.
#include <cmath>
#include <cstring>

#include "lte_api.h"
#include "lte_common.cuh"
#include "lte_internal.h"

using lte::Strides4;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int elt_size(int dtype) { return dtype == LTE_BF16 ? 2 : 4; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

lte_status check_dims(const lte_dims* d) {
  if (d == nullptr) return LTE_ERR_INVALID_ARG;
  if (d->B < 1 || d->T < 1 || d->Hq < 1 || d->Hkv < 1 || d->D < 1) return LTE_ERR_INVALID_ARG;
  if (d->Hq % d->Hkv != 0) return LTE_ERR_INVALID_ARG;
  if (d->sink < 0 || d->window < 1 || d->cap < 0) return LTE_ERR_INVALID_ARG;
  if (d->dtype != LTE_F32 && d->dtype != LTE_BF16) return LTE_ERR_INVALID_ARG;
  if (d->cap_policy != LTE_CAP_RECENT && d->cap_policy != LTE_CAP_FIRST &&
      d->cap_policy != LTE_CAP_LOWEST)
    return LTE_ERR_INVALID_ARG;
  if (!(d->scale > 0.f) || !std::isfinite(d->scale)) return LTE_ERR_INVALID_ARG;
  if (std::isnan(d->tau)) return LTE_ERR_INVALID_ARG;
  if (d->D != 64 && d->D != 128) return LTE_ERR_UNSUPPORTED;
  // int32 indexing of per-unit rows and of the column segment
  if ((long long)d->T + d->sink >= (1ll << 30)) return LTE_ERR_UNSUPPORTED;
  return LTE_OK;
}

// strides: NULL -> contiguous [B,T,H,D]; otherwise 16-byte multiples
lte_status get_strides(const lte_dims* d, const lte_strides* s, int H, Strides4* out) {
  if (s == nullptr) {
    out->h = d->D;
    out->t = (long long)H * d->D;
    out->b = (long long)d->T * H * d->D;
    return LTE_OK;
  }
  const int per16 = 16 / elt_size(d->dtype);
  if (s->b % per16 || s->t % per16 || s->h % per16) return LTE_ERR_INVALID_ARG;
  if (s->b < 0 || s->t < 0 || s->h < 0) return LTE_ERR_INVALID_ARG;
  out->b = s->b;
  out->t = s->t;
  out->h = s->h;
  return LTE_OK;
}

lte_status check_cnn(const lte_cnn* c) {
  if (c == nullptr || c->w1 == nullptr || c->b1 == nullptr || c->w2 == nullptr ||
      c->b2 == nullptr)
    return LTE_ERR_INVALID_ARG;
  if (c->k1 < 1 || c->k2 < 1 || c->past1 < 0 || c->past2 < 0 || c->past1 > c->k1 - 1 ||
      c->past2 > c->k2 - 1 || c->c_hid < 1)
    return LTE_ERR_INVALID_ARG;
  if (!lte::score_supported(c)) return LTE_ERR_UNSUPPORTED;
  return LTE_OK;
}

inline int cnn_future(const lte_cnn* c) {
  return (c->k1 - 1 - c->past1) + (c->k2 - 1 - c->past2);
}
inline int cnn_past(const lte_cnn* c) { return c->past1 + c->past2; }

inline lte_status from_cuda(cudaError_t e) { return e == cudaSuccess ? LTE_OK : LTE_ERR_CUDA; }

constexpr size_t kErrBytes = 256;   // error word + padding (keeps scratch 256-aligned)

}  // namespace

extern "C" {

const char* lte_version(void) { return "lte-b200 0.1 (sm_100a)"; }

lte_status lte_score(const lte_dims* d, const lte_cnn* cnn, const void* k, const void* v,
                     const lte_strides* kv_strides, int32_t j_begin, int32_t j_end, float* r,
                     uint8_t* mask, void* stream) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if ((st = check_cnn(cnn)) != LTE_OK) return st;
  if (k == nullptr || v == nullptr || r == nullptr) return LTE_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v)) return LTE_ERR_INVALID_ARG;
  if (j_begin < 0 || j_end < j_begin || j_end > d->T - cnn_future(cnn)) return LTE_ERR_INVALID_ARG;
  Strides4 s;
  if ((st = get_strides(d, kv_strides, d->Hkv, &s)) != LTE_OK) return st;
  if (j_end == j_begin) return LTE_OK;
  return from_cuda(lte::score_linear(d, cnn, k, v, s, j_begin, j_end, r, mask, as_stream(stream)));
}

lte_status lte_evict_compact(const lte_dims* d, const float* r, const uint8_t* mask,
                             int32_t n_scored, int32_t* idx, int32_t* nret, int32_t* cnt,
                             const void* k, const void* v, const lte_strides* kv_strides,
                             void* k_col, void* v_col, void* stream) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if ((r == nullptr) == (mask == nullptr)) return LTE_ERR_INVALID_ARG;
  if (idx == nullptr || nret == nullptr || cnt == nullptr) return LTE_ERR_INVALID_ARG;
  if (n_scored < 0 || n_scored > d->T) return LTE_ERR_INVALID_ARG;
  if ((k_col == nullptr) != (v_col == nullptr)) return LTE_ERR_INVALID_ARG;
  Strides4 s{};
  if (k_col != nullptr) {
    if (k == nullptr || v == nullptr || !aligned16(k) || !aligned16(v) || !aligned16(k_col) ||
        !aligned16(v_col))
      return LTE_ERR_INVALID_ARG;
    if ((st = get_strides(d, kv_strides, d->Hkv, &s)) != LTE_OK) return st;
  }
  return from_cuda(lte::evict_compact(d, r, mask, n_scored, idx, nret, cnt, k, v, s, k_col,
                                      v_col, as_stream(stream)));
}

lte_status lte_retained_lifetimes(const lte_dims* d, const float* r, const int32_t* idx,
                                  const int32_t* nret, int32_t* death, void* stream) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if (d->cap_policy != LTE_CAP_LOWEST) return LTE_ERR_INVALID_ARG;
  if (!r || !idx || !nret || !death) return LTE_ERR_INVALID_ARG;
  return from_cuda(lte::retained_lifetimes(d, r, idx, nret, death, as_stream(stream)));
}

// relaxed-retention workspace: error word, the slot offsets, then (backward) D_t
inline size_t relaxed_bias_bytes(const lte_dims* d) {
  return (lte::slot_bias_floats(d) * sizeof(float) + 255) & ~(size_t)255;
}

size_t lte_workspace_bytes(const lte_dims* d, int32_t which) {
  if (check_dims(d) != LTE_OK) return 0;
  if (which == LTE_WS_PREFILL) return kErrBytes + lte::attn_prefill_scratch_bytes(d);
  if (which == LTE_WS_DECODE) return kErrBytes + lte::decode_scratch_bytes(d);
  if (which == LTE_WS_BACKWARD) return kErrBytes + lte::attn_backward_scratch_bytes(d);
  if (which == LTE_WS_RELAXED)
    return kErrBytes + relaxed_bias_bytes(d) + lte::attn_backward_scratch_bytes(d);
  return 0;
}

size_t lte_score_backward_workspace_bytes(const lte_dims* d, const lte_cnn* cnn) {
  if (check_dims(d) != LTE_OK || check_cnn(cnn) != LTE_OK) return 0;
  return kErrBytes + lte::score_backward_scratch_bytes(d, cnn);
}

lte_status lte_score_backward(const lte_dims* d, const lte_cnn* cnn, const void* k, const void* v,
                              const lte_strides* kv_strides, int32_t n_scored, const float* dr,
                              float* dk, float* dv, float* dw1, float* db1, float* dw2, float* db2,
                              void* workspace, size_t ws_bytes, void* stream) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if ((st = check_cnn(cnn)) != LTE_OK) return st;
  if (!k || !v || !dr || !dk || !dv || !dw1 || !db1 || !dw2 || !db2) return LTE_ERR_INVALID_ARG;
  if (n_scored < 0 || n_scored > d->T - cnn_future(cnn)) return LTE_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned16(workspace)) return LTE_ERR_WORKSPACE;
  if (ws_bytes < lte_score_backward_workspace_bytes(d, cnn)) return LTE_ERR_WORKSPACE;
  Strides4 s;
  if ((st = get_strides(d, kv_strides, d->Hkv, &s)) != LTE_OK) return st;
  return from_cuda(lte::score_backward(d, cnn, k, v, s, n_scored, dr, dk, dv, dw1, db1, dw2, db2,
                                       static_cast<char*>(workspace) + kErrBytes,
                                       reinterpret_cast<lte::DevError*>(workspace),
                                       as_stream(stream)));
}

lte_status lte_sparse_attn_backward(const lte_dims* d, const void* q, const void* k, const void* v,
                                    const int32_t* cnt, const int32_t* death, const int32_t* idx,
                                    const int32_t* nret, const void* k_col, const void* v_col,
                                    const void* o, const float* lse, const void* dO, float* dq,
                                    float* dk, float* dv, void* workspace, size_t ws_bytes,
                                    void* stream) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if (!q || !k || !v || !cnt || !idx || !nret || !k_col || !v_col || !o || !lse || !dO || !dq ||
      !dk || !dv)
    return LTE_ERR_INVALID_ARG;
  if (d->cap_policy == LTE_CAP_LOWEST && death == nullptr) return LTE_ERR_INVALID_ARG;
  const void* vec[] = {q, k, v, k_col, v_col, o, dO, dq, dk, dv};
  for (const void* p : vec)
    if (!aligned16(p)) return LTE_ERR_INVALID_ARG;
  if (d->dtype != LTE_BF16) return LTE_ERR_UNSUPPORTED;
  const int G = d->Hq / d->Hkv;
  if (64 % G != 0 || G > 16) return LTE_ERR_UNSUPPORTED;
  if (workspace == nullptr || !aligned16(workspace)) return LTE_ERR_WORKSPACE;
  if (ws_bytes < lte_workspace_bytes(d, LTE_WS_BACKWARD)) return LTE_ERR_WORKSPACE;
  lte::BackwardArgs a{};
  a.d = d;
  a.q = q; a.k = k; a.v = v; a.o = o; a.dO = dO;
  a.cnt = cnt; a.death = d->cap_policy == LTE_CAP_LOWEST ? death : nullptr; a.idx = idx;
  a.nret = nret; a.k_col = k_col; a.v_col = v_col; a.lse = lse;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.err = reinterpret_cast<lte::DevError*>(workspace);
  a.scratch = static_cast<char*>(workspace) + kErrBytes;
  return from_cuda(lte::attn_backward(a, as_stream(stream)));
}

lte_status lte_sparse_attn_prefill(const lte_dims* d, const void* q, const void* k,
                                   const void* v, const lte_strides* q_strides,
                                   const lte_strides* kv_strides, const int32_t* cnt,
                                   const int32_t* death, const void* k_col, const void* v_col,
                                   void* o, const lte_strides* o_strides, float* lse,
                                   void* workspace, size_t ws_bytes, void* stream) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if (!q || !k || !v || !cnt || !k_col || !v_col || !o) return LTE_ERR_INVALID_ARG;
  if (d->cap_policy == LTE_CAP_LOWEST && death == nullptr) return LTE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(k_col) || !aligned16(v_col) ||
      !aligned16(o))
    return LTE_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned16(workspace)) return LTE_ERR_WORKSPACE;
  if (ws_bytes < lte_workspace_bytes(d, LTE_WS_PREFILL)) return LTE_ERR_WORKSPACE;
  const int G = d->Hq / d->Hkv;
  if (d->dtype == LTE_BF16 && (64 % G != 0 || G > 16)) return LTE_ERR_UNSUPPORTED;
  lte::PrefillArgs a{};
  a.d = d;
  a.q = q; a.k = k; a.v = v;
  if ((st = get_strides(d, q_strides, d->Hq, &a.qs)) != LTE_OK) return st;
  if ((st = get_strides(d, kv_strides, d->Hkv, &a.kvs)) != LTE_OK) return st;
  if ((st = get_strides(d, o_strides, d->Hq, &a.os)) != LTE_OK) return st;
  a.cnt = cnt; a.k_col = k_col; a.v_col = v_col; a.o = o; a.lse = lse;
  a.death = d->cap_policy == LTE_CAP_LOWEST ? death : nullptr;
  a.err = reinterpret_cast<lte::DevError*>(workspace);
  a.scratch = static_cast<char*>(workspace) + kErrBytes;
  a.scratch_bytes = ws_bytes - kErrBytes;
  // bf16, head dim 128, 16-byte strides: tcgen05/TMEM/TMA kernel; other bf16
  // shapes: warp-MMA kernel; fp32: SIMT kernel.  All three are GPU kernels;
  // there is no host path.
  cudaError_t e;
  if (lte::attn_prefill_tc_supported(d) && lte::attn_prefill_tc_layout_ok(a))
    e = lte::attn_prefill_tc(a, as_stream(stream));
  else if (d->dtype == LTE_BF16) e = lte::attn_prefill_mma(a, as_stream(stream));
  else e = lte::attn_prefill_simt(a, as_stream(stream));
  return from_cuda(e);
}

// Shared checks of the relaxed-retention calls (contiguous bf16, head dim 128,
// the tcgen05 kernels' group sizes).
static lte_status check_relaxed(const lte_dims* d, const int32_t* death, const void* workspace,
                                size_t ws_bytes) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if (d->cap_policy == LTE_CAP_LOWEST && death == nullptr) return LTE_ERR_INVALID_ARG;
  if (d->dtype != LTE_BF16 || !lte::attn_prefill_tc_supported(d) ||
      !lte::attn_backward_dq_tc_supported(d))
    return LTE_ERR_UNSUPPORTED;
  if (workspace == nullptr || !aligned16(workspace)) return LTE_ERR_WORKSPACE;
  if (ws_bytes < lte_workspace_bytes(d, LTE_WS_RELAXED)) return LTE_ERR_WORKSPACE;
  return LTE_OK;
}

lte_status lte_sparse_attn_prefill_relaxed(const lte_dims* d, const void* q, const void* k,
                                           const void* v, const int32_t* cnt, const int32_t* death,
                                           const int32_t* idx, const int32_t* nret,
                                           const void* k_col, const void* v_col, const float* r,
                                           void* o, float* lse, void* workspace, size_t ws_bytes,
                                           void* stream) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if (!q || !k || !v || !cnt || !idx || !nret || !k_col || !v_col || !r || !o)
    return LTE_ERR_INVALID_ARG;
  const void* vec[] = {q, k, v, k_col, v_col, o};
  for (const void* p : vec)
    if (!aligned16(p)) return LTE_ERR_INVALID_ARG;
  if ((st = check_relaxed(d, death, workspace, ws_bytes)) != LTE_OK) return st;
  float* bias = reinterpret_cast<float*>(static_cast<char*>(workspace) + kErrBytes);
  cudaError_t e = lte::slot_bias(d, r, idx, nret, bias, as_stream(stream));
  if (e != cudaSuccess) return LTE_ERR_CUDA;
  lte::PrefillArgs a{};
  a.d = d;
  a.q = q; a.k = k; a.v = v;
  get_strides(d, nullptr, d->Hq, &a.qs);
  get_strides(d, nullptr, d->Hkv, &a.kvs);
  get_strides(d, nullptr, d->Hq, &a.os);
  a.cnt = cnt; a.k_col = k_col; a.v_col = v_col; a.o = o; a.lse = lse;
  a.death = d->cap_policy == LTE_CAP_LOWEST ? death : nullptr;
  a.err = reinterpret_cast<lte::DevError*>(workspace);
  a.scratch = nullptr;
  a.scratch_bytes = 0;
  a.bias = bias;
  return from_cuda(lte::attn_prefill_tc(a, as_stream(stream)));
}

lte_status lte_sparse_attn_backward_relaxed(const lte_dims* d, const void* q, const void* k,
                                            const void* v, const int32_t* cnt,
                                            const int32_t* death, const int32_t* idx,
                                            const int32_t* nret, const void* k_col,
                                            const void* v_col, const float* r, const void* o,
                                            const float* lse, const void* dO, float* dq,
                                            float* dk, float* dv, float* dr, void* workspace,
                                            size_t ws_bytes, void* stream) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if (!q || !k || !v || !cnt || !idx || !nret || !k_col || !v_col || !r || !o || !lse || !dO ||
      !dq || !dk || !dv || !dr)
    return LTE_ERR_INVALID_ARG;
  const void* vec[] = {q, k, v, k_col, v_col, o, dO, dq, dk, dv};
  for (const void* p : vec)
    if (!aligned16(p)) return LTE_ERR_INVALID_ARG;
  if ((st = check_relaxed(d, death, workspace, ws_bytes)) != LTE_OK) return st;
  char* ws = static_cast<char*>(workspace);
  float* bias = reinterpret_cast<float*>(ws + kErrBytes);
  cudaError_t e = lte::slot_bias(d, r, idx, nret, bias, as_stream(stream));
  if (e != cudaSuccess) return LTE_ERR_CUDA;
  lte::BackwardArgs a{};
  a.d = d;
  a.q = q; a.k = k; a.v = v; a.o = o; a.dO = dO;
  a.cnt = cnt; a.death = d->cap_policy == LTE_CAP_LOWEST ? death : nullptr; a.idx = idx;
  a.nret = nret; a.k_col = k_col; a.v_col = v_col; a.lse = lse;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.err = reinterpret_cast<lte::DevError*>(workspace);
  a.scratch = ws + kErrBytes + relaxed_bias_bytes(d);
  a.bias = bias;
  a.dr = dr;
  return from_cuda(lte::attn_backward(a, as_stream(stream)));
}

lte_status lte_sparse_attn_prefill_kernel(const lte_dims* d, const lte_strides* q_strides,
                                          const lte_strides* kv_strides,
                                          const lte_strides* o_strides, int32_t* kind) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if (kind == nullptr) return LTE_ERR_INVALID_ARG;
  const int G = d->Hq / d->Hkv;
  if (d->dtype == LTE_BF16 && (64 % G != 0 || G > 16)) return LTE_ERR_UNSUPPORTED;
  lte::PrefillArgs a{};
  a.d = d;
  if ((st = get_strides(d, q_strides, d->Hq, &a.qs)) != LTE_OK) return st;
  if ((st = get_strides(d, kv_strides, d->Hkv, &a.kvs)) != LTE_OK) return st;
  if ((st = get_strides(d, o_strides, d->Hq, &a.os)) != LTE_OK) return st;
  if (lte::attn_prefill_tc_supported(d) && lte::attn_prefill_tc_layout_ok(a))
    *kind = LTE_KERNEL_TCGEN05;
  else
    *kind = d->dtype == LTE_BF16 ? LTE_KERNEL_MMA_SYNC : LTE_KERNEL_SIMT;
  return LTE_OK;
}

lte_status lte_sparse_attn_backward_kernel(const lte_dims* d, int32_t* kind) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if (kind == nullptr) return LTE_ERR_INVALID_ARG;
  if (d->dtype != LTE_BF16) return LTE_ERR_UNSUPPORTED;
  const int G = d->Hq / d->Hkv;
  if (64 % G != 0 || G > 16) return LTE_ERR_UNSUPPORTED;
  *kind = lte::attn_backward_dq_tc_supported(d) ? LTE_KERNEL_TCGEN05 : LTE_KERNEL_MMA_SYNC;
  return LTE_OK;
}

lte_status lte_cache_init_from_prefill(const lte_dims* d, const lte_cache* cache, const void* k,
                                       const void* v, const lte_strides* kv_strides,
                                       const float* r, const int32_t* idx, const int32_t* cnt,
                                       const int32_t* death, int32_t T_prompt, int32_t n_scored,
                                       void* stream) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if (cache == nullptr || !cache->k || !cache->v || !cache->pos || !cache->win_r ||
      !cache->ret_total || !cache->meta)
    return LTE_ERR_INVALID_ARG;
  if (!aligned16(cache->k) || !aligned16(cache->v)) return LTE_ERR_INVALID_ARG;
  if (T_prompt < 0 || T_prompt > d->T) return LTE_ERR_INVALID_ARG;
  if (n_scored < 0 || n_scored > T_prompt) return LTE_ERR_INVALID_ARG;
  if (T_prompt > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return LTE_ERR_INVALID_ARG;
  if (T_prompt > d->window && (!idx || !cnt)) return LTE_ERR_INVALID_ARG;
  if (n_scored > 0 && r == nullptr) return LTE_ERR_INVALID_ARG;
  const bool lowest = d->cap_policy == LTE_CAP_LOWEST;
  if (lowest && (cache->ret_r == nullptr || (T_prompt > d->window && (!death || !r))))
    return LTE_ERR_INVALID_ARG;
  Strides4 s;
  if ((st = get_strides(d, kv_strides, d->Hkv, &s)) != LTE_OK) return st;
  return from_cuda(lte::cache_init(d, cache, k, v, s, r, idx, cnt, lowest ? death : nullptr,
                                   T_prompt, n_scored, as_stream(stream)));
}

lte_status lte_decode_step(const lte_dims* d, const lte_cnn* cnn, const lte_cache* cache,
                           const void* q_t, const void* k_t, const void* v_t, void* o_t,
                           float* lse_t, int32_t score_batch, void* workspace, size_t ws_bytes,
                           void* stream) {
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if ((st = check_cnn(cnn)) != LTE_OK) return st;
  if (d->dtype != LTE_BF16) return LTE_ERR_UNSUPPORTED;
  if (cache == nullptr || !cache->k || !cache->v || !cache->pos || !cache->win_r ||
      !cache->ret_total || !cache->meta)
    return LTE_ERR_INVALID_ARG;
  if (d->cap_policy == LTE_CAP_LOWEST && cache->ret_r == nullptr) return LTE_ERR_INVALID_ARG;
  if (!q_t || !k_t || !v_t || !o_t) return LTE_ERR_INVALID_ARG;
  if (!aligned16(q_t) || !aligned16(k_t) || !aligned16(v_t) || !aligned16(o_t) ||
      !aligned16(cache->k) || !aligned16(cache->v))
    return LTE_ERR_INVALID_ARG;
  if (score_batch < 1 || score_batch > d->window - cnn_past(cnn) - cnn_future(cnn))
    return LTE_ERR_INVALID_ARG;
  const int G = d->Hq / d->Hkv;
  if (G > 16 || !lte::decode_supported(d)) return LTE_ERR_UNSUPPORTED;
  if (workspace == nullptr || !aligned16(workspace)) return LTE_ERR_WORKSPACE;
  if (ws_bytes < lte_workspace_bytes(d, LTE_WS_DECODE)) return LTE_ERR_WORKSPACE;
  return from_cuda(lte::decode_step(d, cnn, cache, q_t, k_t, v_t, o_t, lse_t, score_batch,
                                    reinterpret_cast<lte::DevError*>(workspace),
                                    static_cast<char*>(workspace) + kErrBytes,
                                    as_stream(stream)));
}

lte_status lte_decode_step_noalloc(const lte_dims* d, const lte_cnn* cnn, const lte_cache* cache,
                                   const void* q_t, const void* k_t, const void* v_t, void* o_t,
                                   float* lse_t, int32_t score_batch, void* stream) {
  // Same validation as lte_decode_step, then the static scratch in place of a workspace.
  lte_status st = check_dims(d);
  if (st != LTE_OK) return st;
  if ((st = check_cnn(cnn)) != LTE_OK) return st;
  if (d->dtype != LTE_BF16) return LTE_ERR_UNSUPPORTED;
  if (cache == nullptr || !cache->k || !cache->v || !cache->pos || !cache->win_r ||
      !cache->ret_total || !cache->meta)
    return LTE_ERR_INVALID_ARG;
  if (d->cap_policy == LTE_CAP_LOWEST && cache->ret_r == nullptr) return LTE_ERR_INVALID_ARG;
  if (!q_t || !k_t || !v_t || !o_t) return LTE_ERR_INVALID_ARG;
  if (!aligned16(q_t) || !aligned16(k_t) || !aligned16(v_t) || !aligned16(o_t) ||
      !aligned16(cache->k) || !aligned16(cache->v))
    return LTE_ERR_INVALID_ARG;
  if (score_batch < 1 || score_batch > d->window - cnn_past(cnn) - cnn_future(cnn))
    return LTE_ERR_INVALID_ARG;
  if (d->Hq / d->Hkv > 16 || !lte::decode_supported(d)) return LTE_ERR_UNSUPPORTED;
  if (lte_workspace_bytes(d, LTE_WS_DECODE) > (size_t)LTE_NOALLOC_SCRATCH_BYTES)
    return LTE_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (lte::noalloc_scratch(&scratch) != cudaSuccess) return LTE_ERR_CUDA;
  // the error word must start at zero for this call (counters are zeroed by the step itself)
  if (cudaMemsetAsync(scratch, 0, sizeof(lte::DevError), as_stream(stream)) != cudaSuccess)
    return LTE_ERR_CUDA;
  return from_cuda(lte::decode_step(d, cnn, cache, q_t, k_t, v_t, o_t, lse_t, score_batch,
                                    reinterpret_cast<lte::DevError*>(scratch),
                                    static_cast<char*>(scratch) + kErrBytes, as_stream(stream)));
}

lte_status lte_noalloc_read_device_error(int32_t* code, int32_t* where, void* stream) {
  if (code == nullptr) return LTE_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if (lte::noalloc_scratch(&scratch) != cudaSuccess) return LTE_ERR_CUDA;
  return lte_read_device_error(scratch, code, where, stream);
}

lte_status lte_clear_device_error(void* workspace, void* stream) {
  if (workspace == nullptr) return LTE_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(workspace, 0, sizeof(lte::DevError), as_stream(stream)));
}

lte_status lte_read_device_error(const void* workspace, int32_t* code, int32_t* where,
                                 void* stream) {
  if (workspace == nullptr || code == nullptr) return LTE_ERR_INVALID_ARG;
  lte::DevError e{};
  cudaError_t ce = cudaMemcpyAsync(&e, workspace, sizeof(e), cudaMemcpyDeviceToHost,
                                   as_stream(stream));
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(as_stream(stream));
  if (ce != cudaSuccess) return LTE_ERR_CUDA;
  *code = e.code;
  if (where) *where = e.where;
  return LTE_OK;
}

lte_status lte_wait_probe(const int32_t* flag, int32_t expect, int64_t limit_ns, void* workspace,
                          void* stream) {
  if (flag == nullptr || reinterpret_cast<uintptr_t>(flag) % 4 != 0) return LTE_ERR_INVALID_ARG;
  if (limit_ns < 1000 || limit_ns > 10000000000ll) return LTE_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned16(workspace)) return LTE_ERR_WORKSPACE;
  return from_cuda(lte::wait_probe(flag, expect, (unsigned long long)limit_ns,
                                   reinterpret_cast<lte::DevError*>(workspace), as_stream(stream)));
}

lte_status lte_gla_prefill(int32_t B, int32_t T, int32_t H, int32_t dk, int32_t dv,
                           int32_t dtype, const void* q, const void* k, const void* v,
                           const float* a, void* o, float* state, void* stream) {
  if (B < 1 || T < 1 || H < 1 || dk < 1 || dv < 1) return LTE_ERR_INVALID_ARG;
  if (dtype != LTE_F32 && dtype != LTE_BF16) return LTE_ERR_INVALID_ARG;
  if (!q || !k || !v || !a || !o || !state) return LTE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(a) || !aligned16(o) ||
      !aligned16(state))
    return LTE_ERR_INVALID_ARG;
  if (dk != 128 || dv != 128 || dtype != LTE_BF16 || T % 64 != 0) return LTE_ERR_UNSUPPORTED;
  return from_cuda(lte::gla_prefill(B, T, H, dk, dv, dtype, q, k, v, a, o, state,
                                    as_stream(stream)));
}

lte_status lte_gla_decode_step(int32_t B, int32_t H, int32_t dk, int32_t dv, int32_t dtype,
                               const void* q_t, const void* k_t, const void* v_t,
                               const float* a_t, void* o_t, float* state, void* stream) {
  if (B < 1 || H < 1 || dk < 1 || dv < 1) return LTE_ERR_INVALID_ARG;
  if (dtype != LTE_F32 && dtype != LTE_BF16) return LTE_ERR_INVALID_ARG;
  if (!q_t || !k_t || !v_t || !a_t || !o_t || !state) return LTE_ERR_INVALID_ARG;
  if (!aligned16(q_t) || !aligned16(k_t) || !aligned16(v_t) || !aligned16(a_t) ||
      !aligned16(o_t) || !aligned16(state))
    return LTE_ERR_INVALID_ARG;
  if (dk != 128 || dv != 128) return LTE_ERR_UNSUPPORTED;
  return from_cuda(lte::gla_decode(B, H, dk, dv, dtype, q_t, k_t, v_t, a_t, o_t, state,
                                   as_stream(stream)));
}

}  // extern "C"
