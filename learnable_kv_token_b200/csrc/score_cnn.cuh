// Retention-score CNN tile (device code shared by lte_score and the decode step).
#pragma once

#include "lte_common.cuh"

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
  // linear mode: score [j_begin, j_end), tokens [0, T_avail) exist, r/mask rows of length T
  int j_begin, j_end, T_avail;
  float* r;
  uint8_t* mask;
  // ring mode (win_r != nullptr): scores go to win_r[unit, j mod window]
  int window;
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


// ScoreParams with the CNN and method fields of a call filled in (score_cnn.cu)
ScoreParams score_params(const lte_dims* d, const lte_cnn* cnn);

__host__ __device__ inline int score_smem_floats(int D, int c_hid, int k1, int k2) {
  const int NU = kScoreNT + k2 - 1, NX = NU + k1 - 1;
  return NX * 2 * D + c_hid * (kScoreCH * k1 + 1) + c_hid * NU;
}

// Scores of tokens [jb, min(jb + kScoreNT, j_end)) of unit (b, h); tokens
// [0, T_avail) exist.  Called by every thread of a kScoreThreads-thread CTA
// (it synchronises the CTA); `smem` holds score_smem_floats() floats.
// Each output accumulates in a fixed order, so the result for a token does
// not depend on the tile it falls in or on the addressing mode.
template <typename T, typename KV>
__device__ __forceinline__ void score_tile(const ScoreParams& p, const KV& kv, int b, int h, int jb,
                                           int j_end, int T_avail, float* smem) {
  const int tid = threadIdx.x;
  const int twoD = 2 * p.D;
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
      if (p.win_r != nullptr) {
        p.win_r[(long long)(b * p.Hkv + h) * p.window + (j % p.window)] = r;
      } else {
        const long long o = (long long)(b * p.Hkv + h) * p.T + j;
        p.r[o] = r;
        if (p.mask) p.mask[o] = (j >= p.sink && r >= p.tau) ? 1 : 0;
      }
    }
  }
  __syncthreads();   // shared memory is reused by the next tile
}

}  // namespace lte
