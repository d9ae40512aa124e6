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
};

// retained count a row sees and the start of its retained range
__device__ __forceinline__ void row_range(const Args& a, long long crow, int t, int& lo, int& hi) {
  hi = 0;
  if (t < a.T && t >= a.window) hi = held_retained(__ldg(a.cnt + crow + t - a.window), a.cap, a.cap_policy);
  lo = (a.cap_policy == LTE_CAP_RECENT && hi - a.cap > 0) ? hi - a.cap : 0;
}

}  // namespace bwd
}  // namespace lte
