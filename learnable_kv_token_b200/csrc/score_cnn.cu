// Retention-score CNN of LTE, fp32 SIMT.
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction", Fig. 2 caption: a CNN stack
// reads each KV pair's short-range past and future context and outputs a
// per-token, per-head retention score r_{j,h}; TL;DR: a lightweight CNN
// predicts per-head retention scores.
//
//   u[c,p] = SiLU(b1[c] + sum_{ch<2D} sum_{kk<k1} w1[c,ch,kk] * x[ch, p+kk-past1])
//   r[j]   = sigmoid(b2 + sum_{c} sum_{kk<k2} w2[c,kk] * u[c, j+kk-past2])
// with x = [k; v] and both layers' inputs zero outside the existing tokens.
//
// One CTA scores NT consecutive tokens of one (batch, KV head) unit.  The
// [k; v] rows of the tile plus its halo are staged once in shared memory as
// fp32; w1 is streamed through shared memory in chunks of 16 input channels.
// Every layer-1 output accumulates over (channel, tap) in ascending order and
// every score over (hidden channel, tap) in ascending order, so a token's
// score is bit-identical whichever tile, launch or addressing mode computes
// it.  The same kernel template serves lte_score (tokens addressed in a
// [B,T,H,D] tensor) and the decode step's deferred scoring (tokens addressed
// in the circular window segment of the cache).
#include <algorithm>

#include "lte_common.cuh"
#include "lte_internal.h"

namespace lte {

constexpr int kScoreNT = 64;       // output tokens per CTA
constexpr int kScoreThreads = 256;
constexpr int kScoreCH = 16;       // input channels per w1 chunk
constexpr int kScoreMaxC = 64;     // hidden channels supported
constexpr int kScoreMaxK = 9;      // taps per layer supported

template <typename T>
struct LinearKV {
  const T* k;
  const T* v;
  Strides4 s;
  __device__ __forceinline__ const T* krow(int b, int h, int j) const {
    return k + (long long)b * s.b + (long long)j * s.t + (long long)h * s.h;
  }
  __device__ __forceinline__ const T* vrow(int b, int h, int j) const {
    return v + (long long)b * s.b + (long long)j * s.t + (long long)h * s.h;
  }
};

template <typename T>
struct RingKV {
  const T* k;
  const T* v;
  int Hkv, L, w, D;
  __device__ __forceinline__ const T* krow(int b, int h, int j) const {
    return k + ((long long)(b * Hkv + h) * L + (j % w)) * D;
  }
  __device__ __forceinline__ const T* vrow(int b, int h, int j) const {
    return v + ((long long)(b * Hkv + h) * L + (j % w)) * D;
  }
};

struct ScoreParams {
  int Hkv, D, T;                      // T: length of the r/mask rows (linear mode)
  int c_hid, k1, past1, k2, past2;
  const float *w1, *b1, *w2, *b2;
  int sink;
  float tau;
  // linear mode: score [j_begin, j_end), tokens [0, T_avail) exist
  int j_begin, j_end, T_avail;
  float* r;
  uint8_t* mask;
  // ring mode (meta != nullptr): tokens [0, meta[0]] exist; when
  // score_batch tokens are scorable, score [meta[1], meta[1]+score_batch)
  // into win_r[unit, j mod window]; meta[2] receives the new n_scored.
  int32_t* meta;
  int score_batch, future, window;
  float* win_r;
};

template <typename T>
__device__ __forceinline__ void load8(const T* src, float* dst);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* src, float* dst) {
  uint4 raw = *reinterpret_cast<const uint4*>(src);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    dst[2 * i] = f.x;
    dst[2 * i + 1] = f.y;
  }
}

template <>
__device__ __forceinline__ void load8<float>(const float* src, float* dst) {
  float4 a = *reinterpret_cast<const float4*>(src);
  float4 b = *reinterpret_cast<const float4*>(src + 4);
  dst[0] = a.x; dst[1] = a.y; dst[2] = a.z; dst[3] = a.w;
  dst[4] = b.x; dst[5] = b.y; dst[6] = b.z; dst[7] = b.w;
}

template <typename T, typename KV>
__global__ void __launch_bounds__(kScoreThreads)
score_cnn_kernel(ScoreParams p, KV kv) {
  extern __shared__ float smem[];
  const int b = blockIdx.z, h = blockIdx.y, tid = threadIdx.x;
  const int twoD = 2 * p.D;

  int j_begin = p.j_begin, j_end = p.j_end, T_avail = p.T_avail;
  if (p.meta != nullptr) {
    const int t = p.meta[0];              // newest token, already in the window
    const int n_scored = p.meta[1];
    const bool due = (t - p.future) - n_scored + 1 >= p.score_batch;
    if (blockIdx.x == 0 && h == 0 && b == 0 && tid == 0)
      p.meta[2] = due ? n_scored + p.score_batch : n_scored;
    if (!due) return;
    j_begin = n_scored;
    j_end = n_scored + p.score_batch;
    T_avail = t + 1;
  }
  const int jb = j_begin + blockIdx.x * kScoreNT;      // first output token of the tile
  if (jb >= j_end) return;

  const int NU = kScoreNT + p.k2 - 1;                  // layer-1 positions needed
  const int NX = NU + p.k1 - 1;                        // input positions needed
  const int x0 = jb - p.past2 - p.past1;               // global position of xs row 0
  const int u0 = jb - p.past2;                         // global position of us column 0
  const int wstride = kScoreCH * p.k1 + 1;             // odd: conflict-free per-c rows

  float* xs = smem;                                    // [NX][2D]
  float* ws = xs + NX * twoD;                          // [c_hid][wstride]
  float* us = ws + p.c_hid * wstride;                  // [c_hid][NU]

  // ---- stage [k; v] rows of the tile and halo (zero outside [0, T_avail))
  const int vec_per_row = twoD / 8;
  for (int i = tid; i < NX * vec_per_row; i += kScoreThreads) {
    const int row = i / vec_per_row, c8 = (i % vec_per_row) * 8;
    const int xg = x0 + row;
    float vals[8];
    if (xg >= 0 && xg < T_avail) {
      const T* src = (c8 < p.D) ? kv.krow(b, h, xg) + c8 : kv.vrow(b, h, xg) + (c8 - p.D);
      load8<T>(src, vals);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) vals[e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) xs[row * twoD + c8 + e] = vals[e];
  }

  // ---- layer 1: thread owns hidden channels lane + 32*cc, positions grp + 8*i
  const int lane = tid & 31, grp = tid >> 5;
  constexpr int kMaxCC = kScoreMaxC / 32;
  constexpr int kMaxPI = (kScoreNT + kScoreMaxK - 1 + 7) / 8;
  float acc[kMaxCC][kMaxPI];
#pragma unroll
  for (int cc = 0; cc < kMaxCC; ++cc)
#pragma unroll
    for (int i = 0; i < kMaxPI; ++i) acc[cc][i] = 0.f;

  const float* w1h = p.w1 + (long long)h * p.c_hid * twoD * p.k1;
  for (int ch0 = 0; ch0 < twoD; ch0 += kScoreCH) {
    __syncthreads();
    for (int i = tid; i < p.c_hid * kScoreCH * p.k1; i += kScoreThreads) {
      const int c = i / (kScoreCH * p.k1), rem = i % (kScoreCH * p.k1);
      ws[c * wstride + rem] = w1h[((long long)c * twoD + ch0) * p.k1 + rem];
    }
    __syncthreads();
    for (int chl = 0; chl < kScoreCH; ++chl) {
      for (int kk = 0; kk < p.k1; ++kk) {
        float wv[kMaxCC];
#pragma unroll
        for (int cc = 0; cc < kMaxCC; ++cc) {
          const int c = lane + 32 * cc;
          wv[cc] = (c < p.c_hid) ? ws[c * wstride + chl * p.k1 + kk] : 0.f;
        }
#pragma unroll
        for (int i = 0; i < kMaxPI; ++i) {
          const int pos = grp + 8 * i;
          if (pos < NU) {
            const float xv = xs[(pos + kk) * twoD + ch0 + chl];
#pragma unroll
            for (int cc = 0; cc < kMaxCC; ++cc) acc[cc][i] = fmaf(wv[cc], xv, acc[cc][i]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int cc = 0; cc < kMaxCC; ++cc) {
    const int c = lane + 32 * cc;
    if (c >= p.c_hid) continue;
    const float bias = p.b1[h * p.c_hid + c];
#pragma unroll
    for (int i = 0; i < kMaxPI; ++i) {
      const int pos = grp + 8 * i;
      if (pos < NU) {
        const int ug = u0 + pos;
        us[c * NU + pos] = (ug >= 0 && ug < T_avail) ? siluf_(acc[cc][i] + bias) : 0.f;
      }
    }
  }
  __syncthreads();

  // ---- layer 2 + sigmoid + threshold
  if (tid < kScoreNT) {
    const int j = jb + tid;
    if (j < j_end) {
      float z = p.b2[h];
      const float* w2h = p.w2 + (long long)h * p.c_hid * p.k2;
      for (int c = 0; c < p.c_hid; ++c)
        for (int kk = 0; kk < p.k2; ++kk) z = fmaf(w2h[c * p.k2 + kk], us[c * NU + tid + kk], z);
      const float r = sigmoidf_(z);
      if (p.meta != nullptr) {
        p.win_r[(long long)(b * p.Hkv + h) * p.window + (j % p.window)] = r;
      } else {
        const long long o = (long long)(b * p.Hkv + h) * p.T + j;
        p.r[o] = r;
        if (p.mask) p.mask[o] = (j >= p.sink && r >= p.tau) ? 1 : 0;
      }
    }
  }
}

static size_t score_smem_bytes(int D, int c_hid, int k1, int k2) {
  const int NU = kScoreNT + k2 - 1, NX = NU + k1 - 1;
  return sizeof(float) * ((size_t)NX * 2 * D + (size_t)c_hid * (kScoreCH * k1 + 1) +
                          (size_t)c_hid * NU);
}

template <typename T, typename KV>
static cudaError_t launch(const ScoreParams& p, const KV& kv, int B, int tiles,
                          cudaStream_t stream) {
  const size_t smem = score_smem_bytes(p.D, p.c_hid, p.k1, p.k2);
  cudaError_t e = cudaFuncSetAttribute(score_cnn_kernel<T, KV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(tiles, p.Hkv, B);
  score_cnn_kernel<T, KV><<<grid, kScoreThreads, smem, stream>>>(p, kv);
  return cudaGetLastError();
}

static ScoreParams base_params(const lte_dims* d, const lte_cnn* cnn) {
  ScoreParams p{};
  p.Hkv = d->Hkv; p.D = d->D; p.T = d->T;
  p.c_hid = cnn->c_hid; p.k1 = cnn->k1; p.past1 = cnn->past1; p.k2 = cnn->k2; p.past2 = cnn->past2;
  p.w1 = cnn->w1; p.b1 = cnn->b1; p.w2 = cnn->w2; p.b2 = cnn->b2;
  p.sink = d->sink; p.tau = d->tau;
  p.future = (cnn->k1 - 1 - cnn->past1) + (cnn->k2 - 1 - cnn->past2);
  return p;
}

cudaError_t score_linear(const lte_dims* d, const lte_cnn* cnn, const void* k, const void* v,
                         Strides4 s, int j_begin, int j_end, float* r, uint8_t* mask,
                         cudaStream_t stream) {
  ScoreParams p = base_params(d, cnn);
  p.j_begin = j_begin; p.j_end = j_end; p.T_avail = d->T; p.r = r; p.mask = mask;
  const int tiles = (j_end - j_begin + kScoreNT - 1) / kScoreNT;
  if (tiles == 0) return cudaSuccess;
  if (d->dtype == LTE_BF16)
    return launch<__nv_bfloat16>(p, LinearKV<__nv_bfloat16>{(const __nv_bfloat16*)k,
                                                             (const __nv_bfloat16*)v, s},
                                 d->B, tiles, stream);
  return launch<float>(p, LinearKV<float>{(const float*)k, (const float*)v, s}, d->B, tiles,
                       stream);
}

cudaError_t score_ring(const lte_dims* d, const lte_cnn* cnn, const lte_cache* c,
                       int score_batch, cudaStream_t stream) {
  ScoreParams p = base_params(d, cnn);
  p.meta = c->meta; p.score_batch = score_batch; p.window = d->window; p.win_r = c->win_r;
  const int L = d->window + d->sink + d->cap;
  const int tiles = (score_batch + kScoreNT - 1) / kScoreNT;
  if (d->dtype == LTE_BF16)
    return launch<__nv_bfloat16>(
        p, RingKV<__nv_bfloat16>{(const __nv_bfloat16*)c->k, (const __nv_bfloat16*)c->v, d->Hkv,
                                 L, d->window, d->D},
        d->B, tiles, stream);
  return launch<float>(p, RingKV<float>{(const float*)c->k, (const float*)c->v, d->Hkv, L,
                                        d->window, d->D},
                       d->B, tiles, stream);
}

bool score_supported(const lte_cnn* cnn) {
  return cnn->c_hid >= 1 && cnn->c_hid <= kScoreMaxC && cnn->k1 >= 1 && cnn->k1 <= kScoreMaxK &&
         cnn->k2 >= 1 && cnn->k2 <= kScoreMaxK;
}

}  // namespace lte
