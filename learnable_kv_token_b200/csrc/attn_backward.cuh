// Shared by the backward kernels of the prefill sparse attention: the
// arguments of one call and the retained range a query row sees.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "lte_common.cuh"

namespace lte {
namespace bwd {

struct Args {
  int T, Hq, Hkv, G, TOK, sink, window, cap, cap_policy;
  float scale, scale_log2;
  const __nv_bfloat16 *q, *k, *v, *o, *dO, *k_col, *v_col;
  const int32_t *cnt, *death, *idx, *nret;
  const float* lse;       // natural log, [B, Hq, T]
  float* delta;           // [B, Hq, T]
  float *dq, *dk, *dv;    // fp32, [B,T,Hq,D] and [B,T,Hkv,D]
  // relaxed retention (NULL otherwise): logit offset per column-segment slot
  // ([B*Hkv][sink + T] + 64 padding, log r_j / scale on retained slots, 0 on
  // sinks) and dL/dr ([B,Hkv,T], accumulated with atomics onto zeros)
  const float* bias;
  float* dr;
  // the tcgen05 column pass's work list: item count (int) at offset 0, items
  // (16 bytes each) from offset 256
  void* col_work;
};

// retained count a row sees and the start of its retained range
__device__ __forceinline__ void row_range(const Args& a, long long crow, int t, int& lo, int& hi) {
  hi = 0;
  if (t < a.T && t >= a.window) hi = held_retained(__ldg(a.cnt + crow + t - a.window), a.cap, a.cap_policy);
  lo = (a.cap_policy == LTE_CAP_RECENT && hi - a.cap > 0) ? hi - a.cap : 0;
}

// Tokens [lo_t, hi_t] of the query rows that attend to some key of a tile
// (lo_t > hi_t: none).  Window part (column = false): key positions
// [k0, k0 + nk), attended by rows t in [j, j + w).  Column part (column =
// true): slots [k0, k0 + nk) of the column segment; a sink slot j is attended
// by rows t >= j + w, a retained slot i by the rows whose retained count n_t
// (nondecreasing in t) holds it: n_t > i, and n_t < i + C (most recent C),
// i < C (first C) or n_t < death[i] (lowest score) -- found by binary search.
__device__ __forceinline__ void attending_tokens(const Args& a, long long crow, bool column, int k0,
                                                 int nk, int& lo_t, int& hi_t) {
  if (!column) {
    lo_t = k0;
    hi_t = min(a.T - 1, k0 + nk - 1 + a.window - 1);
    return;
  }
  lo_t = a.T;
  hi_t = -1;
  const int s_end = min(min(a.sink, k0 + nk), a.T);
  if (k0 < s_end) {
    lo_t = k0 + a.window;
    hi_t = a.T - 1;
  }
  const int i0 = max(k0, a.sink) - a.sink, i1 = k0 + nk - a.sink;
  if (i1 > i0 && a.cap > 0 && (a.cap_policy != LTE_CAP_FIRST || i0 < a.cap)) {
    int l = a.window, r = a.T;                       // first row with cnt[t - w] > i0
    while (l < r) {
      const int m = (l + r) >> 1;
      if (__ldg(a.cnt + crow + m - a.window) > i0) r = m; else l = m + 1;
    }
    if (l < a.T) {
      long long bound;                               // rows need cnt[t - w] < bound
      if (a.cap_policy == LTE_CAP_RECENT) bound = (long long)i1 + a.cap;
      else if (a.cap_policy == LTE_CAP_FIRST) bound = 1ll << 40;
      else {
        int md = 0;
        for (int i = i0; i < i1; ++i) md = max(md, __ldg(a.death + crow + i));
        bound = md;
      }
      int l2 = l, r2 = a.T;                          // first row with cnt >= bound
      while (l2 < r2) {
        const int m = (l2 + r2) >> 1;
        if ((long long)__ldg(a.cnt + crow + m - a.window) >= bound) r2 = m; else l2 = m + 1;
      }
      if (l2 > l) {
        lo_t = min(lo_t, l);
        hi_t = max(hi_t, l2 - 1);
      }
    }
  }
}

}  // namespace bwd
}  // namespace lte
