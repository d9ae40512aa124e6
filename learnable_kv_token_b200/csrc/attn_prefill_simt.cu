// Prefill sparse attention, fp32 SIMT path (fp32 inputs).
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction", Fig. 2 caption (right): each
// query attends, per KV head, to the attention sink, the sliding window and
// the LTE-retained tokens (the "A-plus-column" pattern).  For row t:
//   S_t = { j < s : j <= t-w } u (t-w, t] u { idx[i] : max(0, n_t-C) <= i < n_t },
//   n_t = cnt[t-w] (0 for t < w); under the first-C cap the range is
//   [0, min(n_t, C)), under the drop-the-lowest-score cap { i < n_t :
//   death[i] > n_t } (death from lte_retained_lifetimes).
//
// One CTA handles 32 rows of one query head.  Keys stream in chunks of 32
// from three ranges (sink slots and retained slots of the column segment,
// and the window band of the key tensor); a per-(row, key) predicate keeps
// exactly S_t; online softmax in fp32 with expf.
#include <math.h>

#include "lte_common.cuh"
#include "lte_internal.h"

namespace lte {

constexpr int kSimtRows = 32;
constexpr int kSimtKeys = 32;
constexpr int kSimtThreads = 128;
constexpr int kSimtMaxD = 128;

__global__ void __launch_bounds__(kSimtThreads)
attn_prefill_simt_kernel(int T, int Hq, int Hkv, int D, int sink, int window, int cap,
                         int cap_policy, float scale, const float* __restrict__ q, const float* __restrict__ k,
                         const float* __restrict__ v, Strides4 qs, Strides4 kvs,
                         const int32_t* __restrict__ cnt, const int32_t* __restrict__ death,
                         const float* __restrict__ k_col,
                         const float* __restrict__ v_col, float* __restrict__ o, Strides4 os,
                         float* __restrict__ lse) {
  extern __shared__ float sm[];
  const int ld = D + 1;                                   // odd row pitch: no bank conflicts
  float* q_s = sm;                                        // [32][D+1]
  float* k_s = q_s + kSimtRows * ld;                      // [32][D+1]
  float* v_s = k_s + kSimtKeys * ld;                      // [32][D+1]
  float* p_s = v_s + kSimtKeys * ld;                      // [32][33]

  const int t0 = blockIdx.x * kSimtRows, qh = blockIdx.y, b = blockIdx.z;
  const int G = Hq / Hkv, h = qh / G, u = b * Hkv + h;
  const int tid = threadIdx.x, row = tid >> 2, quarter = tid & 3;
  const int t = t0 + row;
  const int t_last = min(t0 + kSimtRows - 1, T - 1);
  const long long crow = (long long)u * T;

  for (int i = tid; i < kSimtRows * D; i += kSimtThreads) {
    const int rr = i / D, dd = i % D, tt = t0 + rr;
    q_s[rr * ld + dd] = tt < T ? q[(long long)b * qs.b + (long long)tt * qs.t + (long long)qh * qs.h + dd]
                         : 0.f;
  }
  // per-row retained range [lo_t, hi_t) of the compacted list
  const bool lowest = death != nullptr;      // held set filtered by lifetime, scanned from 0
  int hi_t = 0, lo_t = 0;
  if (t < T && t >= window) {
    hi_t = held_retained(cnt[crow + t - window], cap, cap_policy);
    lo_t = hi_t - cap > 0 && !lowest ? hi_t - cap : 0;
  }
  // tile-wide ranges
  const int n_first = (t0 >= window) ? held_retained(cnt[crow + t0 - window], cap, cap_policy) : 0;
  const int n_last = (t_last >= window) ? held_retained(cnt[crow + t_last - window], cap, cap_policy) : 0;
  const int lo_min = n_first - cap > 0 && !lowest ? n_first - cap : 0;
  int nsink = t_last - window + 1;
  nsink = nsink < 0 ? 0 : (nsink > sink ? sink : nsink);
  nsink = nsink > T ? T : nsink;
  const int w_lo = t0 - window + 1 > 0 ? t0 - window + 1 : 0;
  // ranges: 0 = sink slots [0,nsink), 1 = retained slots [sink+lo_min, sink+n_last),
  //         2 = window band [w_lo, t_last]
  int r_start[3] = {0, sink + lo_min, w_lo};
  int r_count[3] = {nsink, n_last - lo_min > 0 ? n_last - lo_min : 0, t_last - w_lo + 1};

  const int dq = D / 4;
  float acc[kSimtMaxD / 4];
  for (int i = 0; i < kSimtMaxD / 4; ++i) acc[i] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

  for (int rg = 0; rg < 3; ++rg) {
    for (int off = 0; off < r_count[rg]; off += kSimtKeys) {
      const int nk = min(kSimtKeys, r_count[rg] - off);
      __syncthreads();
      for (int i = tid; i < kSimtKeys * D; i += kSimtThreads) {
        const int kk = i / D, dd = i % D;
        float kv0 = 0.f, vv0 = 0.f;
        if (kk < nk) {
          const int key = r_start[rg] + off + kk;
          if (rg == 2) {
            const long long a = (long long)b * kvs.b + (long long)key * kvs.t + (long long)h * kvs.h + dd;
            kv0 = k[a]; vv0 = v[a];
          } else {
            const long long a = ((long long)u * (sink + T) + key) * D + dd;
            kv0 = k_col[a]; vv0 = v_col[a];
          }
        }
        k_s[kk * ld + dd] = kv0;
        v_s[kk * ld + dd] = vv0;
      }
      __syncthreads();
      // scores for this row, keys quarter*8 .. +8
      float sc[8];
      float cmax = -INFINITY;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int kk = quarter * 8 + e;
        const int key = r_start[rg] + off + kk;
        bool ok = (kk < nk) && (t < T);
        if (ok) {
          if (rg == 2) ok = key <= t && key > t - window;
          else if (key < sink) ok = key <= t - window;
          else ok = (key - sink) >= lo_t && (key - sink) < hi_t &&
                    (!lowest || death[crow + key - sink] > hi_t);
        }
        float s = -INFINITY;
        if (ok) {
          float dot = 0.f;
          for (int dd = 0; dd < D; ++dd) dot = fmaf(q_s[row * ld + dd], k_s[kk * ld + dd], dot);
          s = dot * scale;
        }
        sc[e] = s;
        cmax = fmaxf(cmax, s);
      }
      cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));
      cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 2));
      const float m_new = fmaxf(m_run, cmax);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float corr = (m_run == -INFINITY) ? 0.f : expf(m_run - m_use);
      float psum = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float pe = (sc[e] == -INFINITY) ? 0.f : expf(sc[e] - m_use);
        p_s[row * (kSimtKeys + 1) + quarter * 8 + e] = pe;
        psum += pe;
      }
      psum += __shfl_xor_sync(0xffffffffu, psum, 1);
      psum += __shfl_xor_sync(0xffffffffu, psum, 2);
      l_run = l_run * corr + psum;
      m_run = m_new;
      __syncwarp();
      for (int i = 0; i < dq; ++i) {
        const int dd = quarter * dq + i;
        float a = acc[i] * corr;
        for (int kk = 0; kk < nk; ++kk) a = fmaf(p_s[row * (kSimtKeys + 1) + kk], v_s[kk * ld + dd], a);
        acc[i] = a;
      }
    }
  }
  if (t < T) {
    const float inv = 1.f / l_run;
    for (int i = 0; i < dq; ++i) {
      const int dd = quarter * dq + i;
      o[(long long)b * os.b + (long long)t * os.t + (long long)qh * os.h + dd] = acc[i] * inv;
    }
    if (lse != nullptr && quarter == 0) lse[((long long)b * Hq + qh) * T + t] = m_run + logf(l_run);
  }
}

cudaError_t attn_prefill_simt(const PrefillArgs& a, cudaStream_t stream) {
  const lte_dims* d = a.d;
  dim3 grid((d->T + kSimtRows - 1) / kSimtRows, d->Hq, d->B);
  const size_t smem = sizeof(float) * ((size_t)3 * 32 * (d->D + 1) + 32 * 33);
  cudaError_t e = cudaFuncSetAttribute(attn_prefill_simt_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attn_prefill_simt_kernel<<<grid, kSimtThreads, smem, stream>>>(
      d->T, d->Hq, d->Hkv, d->D, d->sink, d->window, d->cap, d->cap_policy, d->scale, (const float*)a.q,
      (const float*)a.k, (const float*)a.v, a.qs, a.kvs, a.cnt, a.death, (const float*)a.k_col,
      (const float*)a.v_col, (float*)a.o, a.os, a.lse);
  return cudaGetLastError();
}

}  // namespace lte
