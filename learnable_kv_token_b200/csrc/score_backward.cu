// Backward through the per-KV-head scoring CNN, given dL/dr.
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction": TL;DR, Abstract and Fig. 2
// caption (the CNN stack over past and future keys and values that gives
// r_{j,h}; the model is trained end to end).  The pages fix no gradient for
// the eviction decision, so dL/dr is an input; from it, by the chain rule
// through the two layers (each layer's input 0 outside [0, T)):
//   dz2[j] = dr[j] r[j] (1 - r[j])                       (j < n_scored, else 0)
//   du[c, i]  = sum_kk w2[c, kk] dz2[i - kk + past2]
//   dz1[c, i] = du[c, i] SiLU'(z1[c, i])
//   dx[ch, m] = sum_{c, kk} w1[c, ch, kk] dz1[c, m - kk + past1]      (x = [k; v])
//   dw1[c, ch, kk] = sum_{b, i} dz1[c, i] x[ch, i + kk - past1],  db1 = sum dz1
//   dw2[c, kk] = sum_{b, j} dz2[j] u[c, j + kk - past2],          db2 = sum dz2
// Kernels, fp32 SIMT, one 64-position tile of one (batch, KV head) unit per
// CTA unless stated:
//   cnnb_z1_kernel   z1 = b1 + W1 * x (the forward's first layer, kept);
//   cnnb_dz_kernel   u, z2, r, dz2 over the tile and its halo, then du and
//                    dz1 for the tile; dw2 and db2 partial sums (atomics);
//   cnnb_dx_kernel   dx of the tile, added to dk, dv;
//   cnnb_dw1_kernel  dw1, db1 per KV head over 2048-position chunks of one
//                    sequence (32 hidden channels x 32 input channels x k1
//                    taps per CTA), added with atomics.
#include <math.h>

#include "lte_common.cuh"
#include "lte_internal.h"

namespace lte {
namespace cnnb {

constexpr int kTile = 64;           // positions per CTA
constexpr int kThreads = 256;
constexpr int kChanChunk = 32;      // input channels per pass
constexpr int kMaxK = 9;            // taps (lte_cnn: k1, k2 <= 9)
constexpr int kMaxHid = 64;         // hidden channels (lte_cnn: c_hid <= 64)
constexpr int kDwChunk = 2048;      // positions per CTA of the dw1 reduction
constexpr int kDwSub = 256;         // positions of a dw1 CTA staged at once

struct Args {
  int B, T, Hkv, D, c_hid, k1, past1, k2, past2, n_scored, elt;
  Strides4 s;
  const char *k, *v;
  const float *w1, *b1, *w2, *b2, *dr;
  float *dk, *dv, *dw1, *db1, *dw2, *db2;
  float *z1, *dz1;                  // scratch [B*Hkv][c_hid][T]
  __nv_bfloat16* dzp;               // dz1 as bf16 hi, lo planes [2][B*Hkv][T][32] for the
                                    // tensor-core dw1 pass, else NULL (then dw1 pass adds db1)
};

// x[ch][i] of unit (b, h): k channels first, then v; 0 outside [0, T)
__device__ __forceinline__ float load_x(const Args& a, int b, int h, int ch, int i) {
  if (i < 0 || i >= a.T) return 0.f;
  const bool is_v = ch >= a.D;
  const char* base = is_v ? a.v : a.k;
  const long long off =
      (long long)b * a.s.b + (long long)i * a.s.t + (long long)h * a.s.h + (is_v ? ch - a.D : ch);
  if (a.elt == 2) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[off]);
  return reinterpret_cast<const float*>(base)[off];
}

__device__ __forceinline__ float sigm(float z) { return 1.f / (1.f + expf(-z)); }

// ---------------------------------------------------------------- z1
__global__ void __launch_bounds__(kThreads) cnnb_z1_kernel(const Args a) {
  __shared__ float xs[kChanChunk][kTile + kMaxK];
  extern __shared__ float ws[];                  // [c_hid][32][k1] weights of a channel chunk
  const int u = blockIdx.y, b = u / a.Hkv, h = u % a.Hkv, tid = threadIdx.x;
  const int p0 = blockIdx.x * kTile;
  const int C = a.c_hid, K1 = a.k1, width = kTile + K1 - 1;
  // thread: hidden channels c = tid / 8 (+ 32), positions (tid % 8) * 8 .. + 8
  float acc[2][8];
#pragma unroll
  for (int q = 0; q < 2; ++q)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[q][e] = 0.f;
  const int c0 = tid >> 3, i0 = (tid & 7) * 8;
  for (int ch0 = 0; ch0 < 2 * a.D; ch0 += kChanChunk) {
    __syncthreads();
    for (int t = tid; t < kChanChunk * width; t += kThreads) {
      const int ch = t / width, i = t % width;
      xs[ch][i] = load_x(a, b, h, ch0 + ch, p0 + i - a.past1);
    }
    for (int t = tid; t < C * kChanChunk * K1; t += kThreads) {
      const int c = t / (kChanChunk * K1), r = t % (kChanChunk * K1);
      ws[t] = a.w1[(((long long)h * C + c) * 2 * a.D + ch0 + r / K1) * K1 + r % K1];
    }
    __syncthreads();
    for (int ch = 0; ch < kChanChunk; ++ch) {
      // the 8 + k1 - 1 inputs this thread's 8 positions read, once per channel
      float xr[8 + kMaxK - 1];
#pragma unroll
      for (int t = 0; t < 8 + kMaxK - 1; ++t) xr[t] = t < 8 + K1 - 1 ? xs[ch][i0 + t] : 0.f;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int c = c0 + q * 32;
        if (c >= C) continue;
#pragma unroll
        for (int kk = 0; kk < kMaxK; ++kk) {
          if (kk >= K1) break;
          const float w = ws[(c * kChanChunk + ch) * K1 + kk];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[q][e] = fmaf(w, xr[e + kk], acc[q][e]);
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int c = c0 + q * 32;
    if (c >= C) continue;
    float* z = a.z1 + ((long long)u * C + c) * a.T;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (p0 + i0 + e < a.T) z[p0 + i0 + e] = acc[q][e] + a.b1[h * C + c];
  }
}

// ---------------------------------------------------------------- dz2, du, dz1
__global__ void __launch_bounds__(kThreads) cnnb_dz_kernel(const Args a) {
  constexpr int kW = kTile + 2 * (kMaxK - 1);
  __shared__ float us[kMaxHid][kW];              // u over [p0 - (k2-1), p0 + 64 + k2 - 1)
  __shared__ float dz2s[kTile + kMaxK];          // dz2 over [p0 - (k2-1-past2), p0 + 64 + past2)
  __shared__ float w2s[kMaxHid * kMaxK];
  __shared__ float db1s[kMaxHid];
  __shared__ float dzt[kTile][33];               // dz1 of the tile, [position][c] (32 channels)
  const int u = blockIdx.y, h = u % a.Hkv, tid = threadIdx.x;
  if (tid < kMaxHid) db1s[tid] = 0.f;
  const int p0 = blockIdx.x * kTile;
  const int C = a.c_hid, K2 = a.k2, P2 = a.past2, F2 = K2 - 1 - P2;
  const int ulo = p0 - (K2 - 1), uw = kTile + 2 * (K2 - 1);
  const int jlo = p0 - F2, jw = kTile + K2 - 1;
  for (int t = tid; t < C * K2; t += kThreads) w2s[t] = a.w2[(long long)h * C * K2 + t];
  for (int t = tid; t < C * uw; t += kThreads) {
    const int c = t / uw, i = ulo + t % uw;
    float x = 0.f;
    if (i >= 0 && i < a.T) {
      const float z = a.z1[((long long)u * C + c) * a.T + i];
      x = z * sigm(z);
    }
    us[c][t % uw] = x;
  }
  __syncthreads();
  // z2, r and dz2 at positions jlo .. jlo + jw - 1
  for (int t = tid; t < jw; t += kThreads) {
    const int j = jlo + t;
    float g = 0.f;
    if (j >= 0 && j < a.n_scored) {
      float z = a.b2[h];
      for (int c = 0; c < C; ++c)
        for (int kk = 0; kk < K2; ++kk) z = fmaf(w2s[c * K2 + kk], us[c][j + kk - P2 - ulo], z);
      const float r = sigm(z);
      g = a.dr[(long long)u * a.T + j] * r * (1.f - r);
    }
    dz2s[t] = g;
  }
  __syncthreads();
  // du, dz1 of the tile; dw2 / db2 partial sums over the tile's own j
  for (int t = tid; t < C * kTile; t += kThreads) {   // whole warps (C * kTile % 256 == 0)
    const int c = t / kTile, i = p0 + t % kTile;
    float dz = 0.f;                                    // 0 past the sequence
    if (i < a.T) {
      float du = 0.f;
      for (int kk = 0; kk < K2; ++kk) du = fmaf(w2s[c * K2 + kk], dz2s[i - kk + P2 - jlo], du);
      const long long zi = ((long long)u * C + c) * a.T + i;
      const float z = a.z1[zi], sg = sigm(z);
      dz = du * sg * (1.f + z * (1.f - sg));
      a.dz1[zi] = dz;
    }
    if (a.dzp != nullptr) {
      // the 32 lanes of a warp share c (kTile = 64): one shared atomic per warp for db1
      float sum = dz;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if ((tid & 31) == 0) atomicAdd_block(&db1s[c], sum);
      dzt[t % kTile][c] = dz;
    }
  }
  if (a.dzp != nullptr) {
    // dz1 as bf16 hi and lo planes [unit][T][32], 16-byte chunks of 64-byte rows
    // (the tensor-core dx and dw1 passes read them)
    __syncthreads();
    if (tid < C) atomicAdd(a.db1 + h * C + tid, db1s[tid]);
    const long long plane = (long long)a.B * a.Hkv * a.T * C;
    for (int e = tid; e < 2 * kTile * 4; e += kThreads) {
      const int g = e & 3, r = (e >> 2) % kTile, pl = e / (kTile * 4);
      const int i = p0 + r;
      if (i >= a.T) continue;
      uint32_t w[4];
#pragma unroll
      for (int f = 0; f < 4; ++f) {
        float v2[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float x = dzt[r][g * 8 + 2 * f + q];
          const __nv_bfloat16 hi = __float2bfloat16_rn(x);
          v2[q] = pl == 0 ? __bfloat162float(hi) : x - __bfloat162float(hi);
        }
        __nv_bfloat162 b2 = __floats2bfloat162_rn(v2[0], v2[1]);
        w[f] = *reinterpret_cast<uint32_t*>(&b2);
      }
      *reinterpret_cast<uint4*>(a.dzp + pl * plane + ((long long)u * a.T + i) * C + g * 8) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  for (int t = tid; t < C * K2; t += kThreads) {
    const int c = t / K2, kk = t % K2;
    float acc = 0.f;
    for (int e = 0; e < kTile; ++e) {
      const int j = p0 + e;
      if (j >= a.T) break;
      acc = fmaf(dz2s[j - jlo], us[c][j + kk - P2 - ulo], acc);
    }
    atomicAdd(a.dw2 + (long long)h * C * K2 + t, acc);
  }
  if (tid == 0) {
    float acc = 0.f;
    for (int e = 0; e < kTile && p0 + e < a.T; ++e) acc += dz2s[p0 + e - jlo];
    atomicAdd(a.db2 + h, acc);
  }
}

// ---------------------------------------------------------------- dx
__global__ void __launch_bounds__(kThreads) cnnb_dx_kernel(const Args a) {
  __shared__ float dzs[kMaxHid][kTile + kMaxK];  // dz1 over [p0 - (k1-1-past1), p0 + 64 + past1)
  extern __shared__ float ws[];                  // [c_hid][32][k1] weights of a channel chunk
  const int u = blockIdx.y, b = u / a.Hkv, h = u % a.Hkv, tid = threadIdx.x;
  const int p0 = blockIdx.x * kTile;
  const int C = a.c_hid, K1 = a.k1, P1 = a.past1, F1 = K1 - 1 - P1;
  const int lo = p0 - F1, width = kTile + K1 - 1;
  for (int t = tid; t < C * width; t += kThreads) {
    const int c = t / width, i = lo + t % width;
    dzs[c][t % width] = (i >= 0 && i < a.T) ? a.dz1[((long long)u * C + c) * a.T + i] : 0.f;
  }
  // thread: input channel ch0 + tid / 8, positions (tid % 8) * 8 .. + 8
  const int chl = tid >> 3, i0 = (tid & 7) * 8;
  for (int ch0 = 0; ch0 < 2 * a.D; ch0 += kChanChunk) {
    __syncthreads();
    for (int t = tid; t < C * kChanChunk * K1; t += kThreads) {
      const int c = t / (kChanChunk * K1), r = t % (kChanChunk * K1);
      ws[t] = a.w1[(((long long)h * C + c) * 2 * a.D + ch0 + r / K1) * K1 + r % K1];
    }
    __syncthreads();
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int c = 0; c < C; ++c) {
      // dz1 at m - kk + past1, m = p0 + i0 + e  ->  index i0 + e + (k1 - 1 - kk)
      float zr[8 + kMaxK - 1];
#pragma unroll
      for (int t = 0; t < 8 + kMaxK - 1; ++t) zr[t] = t < 8 + K1 - 1 ? dzs[c][i0 + t] : 0.f;
#pragma unroll
      for (int rk = 0; rk < kMaxK; ++rk) {             // rk = k1 - 1 - kk
        if (rk >= K1) break;
        const float w = ws[(c * kChanChunk + chl) * K1 + (K1 - 1 - rk)];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, zr[e + rk], acc[e]);
      }
    }
    const int ch = ch0 + chl;
    const bool is_v = ch >= a.D;
    float* dst = is_v ? a.dv : a.dk;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int m = p0 + i0 + e;
      if (m >= a.T) break;
      dst[(((long long)b * a.T + m) * a.Hkv + h) * a.D + (is_v ? ch - a.D : ch)] += acc[e];
    }
  }
}

// ---------------------------------------------------------------- dw1, db1
// CTA: KV head h (blockIdx.y), input channels [32 * blockIdx.z, + 32), and
// positions [p0, p0 + 2048) of sequence b (blockIdx.x = b * chunks + chunk).
__global__ void __launch_bounds__(kThreads) cnnb_dw1_kernel(const Args a) {
  constexpr int kSub = kDwSub;                     // positions staged at once
  extern __shared__ float dyn[];
  float (*dzs)[kSub] = reinterpret_cast<float (*)[kSub]>(dyn);                 // [c_hid][kSub]
  float (*xs)[kSub + kMaxK] = reinterpret_cast<float (*)[kSub + kMaxK]>(dyn + a.c_hid * kSub);
  const int h = blockIdx.y, ch0 = blockIdx.z * kChanChunk, tid = threadIdx.x;
  const int chunks = (a.T + kDwChunk - 1) / kDwChunk;
  const int b = blockIdx.x / chunks, pc = (blockIdx.x % chunks) * kDwChunk;
  const int u = b * a.Hkv + h;
  const int C = a.c_hid, K1 = a.k1, P1 = a.past1;
  // thread: hidden channel c = tid / 8 (+ 32), input channels (tid % 8) * 4 .. + 4, all taps
  const int c0 = tid >> 3, cl0 = (tid & 7) * 4;
  float acc[2][4][kMaxK];
#pragma unroll
  for (int q = 0; q < 2; ++q)
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
      for (int kk = 0; kk < kMaxK; ++kk) acc[q][e][kk] = 0.f;
  float dbacc[2] = {0.f, 0.f};
  const int pend = min(a.T, pc + kDwChunk);
  for (int p0 = pc; p0 < pend; p0 += kSub) {
    __syncthreads();
    for (int t = tid; t < C * kSub; t += kThreads) {
      const int c = t / kSub, i = p0 + t % kSub;
      dzs[c][t % kSub] = i < a.T ? a.dz1[((long long)u * C + c) * a.T + i] : 0.f;
    }
    const int width = kSub + K1 - 1;
    for (int t = tid; t < kChanChunk * width; t += kThreads) {
      const int ch = t / width, i = t % width;
      xs[ch][i] = load_x(a, b, h, ch0 + ch, p0 + i - P1);
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int c = c0 + q * 32;
      if (c >= C) continue;
      for (int i = 0; i < kSub; ++i) {
        const float d = dzs[c][i];
        if ((tid & 7) == 0) dbacc[q] += d;
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int kk = 0; kk < kMaxK; ++kk)
            if (kk < K1) acc[q][e][kk] = fmaf(d, xs[cl0 + e][i + kk], acc[q][e][kk]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int c = c0 + q * 32;
    if (c >= C) continue;
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
      for (int kk = 0; kk < kMaxK; ++kk)
        if (kk < K1)
          atomicAdd(a.dw1 + (((long long)h * C + c) * 2 * a.D + ch0 + cl0 + e) * K1 + kk, acc[q][e][kk]);
    if ((tid & 7) == 0 && blockIdx.z == 0) atomicAdd(a.db1 + h * C + c, dbacc[q]);
  }
}

}  // namespace cnnb

size_t score_backward_scratch_bytes(const lte_dims* d, const lte_cnn* cnn) {
  size_t n = 2 * (size_t)d->B * d->Hkv * cnn->c_hid * d->T * sizeof(float);
  if (score_backward_tc_supported(d, cnn))                 // dz1 planes for the tensor-core dw1
    n += 2 * (size_t)d->B * d->Hkv * d->T * cnn->c_hid * sizeof(__nv_bfloat16);
  return n;
}

cudaError_t score_backward(const lte_dims* d, const lte_cnn* cnn, const void* k, const void* v,
                           Strides4 s, int n_scored, const float* dr, float* dk, float* dv,
                           float* dw1, float* db1, float* dw2, float* db2, void* scratch,
                           DevError* err, cudaStream_t stream) {
  cnnb::Args a{};
  a.B = d->B; a.T = d->T; a.Hkv = d->Hkv; a.D = d->D;
  a.c_hid = cnn->c_hid; a.k1 = cnn->k1; a.past1 = cnn->past1; a.k2 = cnn->k2; a.past2 = cnn->past2;
  a.n_scored = n_scored; a.elt = d->dtype == LTE_BF16 ? 2 : 4; a.s = s;
  a.k = (const char*)k; a.v = (const char*)v;
  a.w1 = cnn->w1; a.b1 = cnn->b1; a.w2 = cnn->w2; a.b2 = cnn->b2; a.dr = dr;
  a.dk = dk; a.dv = dv; a.dw1 = dw1; a.db1 = db1; a.dw2 = dw2; a.db2 = db2;
  a.z1 = reinterpret_cast<float*>(scratch);
  a.dz1 = a.z1 + (size_t)d->B * d->Hkv * cnn->c_hid * d->T;
  const bool tc = score_backward_tc_supported(d, cnn);
  a.dzp = tc ? reinterpret_cast<__nv_bfloat16*>(a.dz1 + (size_t)d->B * d->Hkv * cnn->c_hid * d->T)
             : nullptr;
  const size_t C = cnn->c_hid;
  cudaError_t e;
  if ((e = cudaMemsetAsync(dw1, 0, d->Hkv * C * 2 * d->D * cnn->k1 * sizeof(float), stream)) != cudaSuccess ||
      (e = cudaMemsetAsync(db1, 0, d->Hkv * C * sizeof(float), stream)) != cudaSuccess ||
      (e = cudaMemsetAsync(dw2, 0, d->Hkv * C * cnn->k2 * sizeof(float), stream)) != cudaSuccess ||
      (e = cudaMemsetAsync(db2, 0, d->Hkv * sizeof(float), stream)) != cudaSuccess)
    return e;
  const size_t ws_smem = C * cnnb::kChanChunk * cnn->k1 * sizeof(float);
  const size_t dw_smem = (C * cnnb::kDwSub + cnnb::kChanChunk * (cnnb::kDwSub + cnnb::kMaxK)) * sizeof(float);
  if ((e = cudaFuncSetAttribute(cnnb::cnnb_z1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)ws_smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(cnnb::cnnb_dx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)ws_smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(cnnb::cnnb_dw1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)dw_smem)) != cudaSuccess)
    return e;
  const dim3 grid((d->T + cnnb::kTile - 1) / cnnb::kTile, d->B * d->Hkv);
  if (tc && score_tcgen05_supported(d, cnn, s)) {
    // the layer-1 recompute on tensor cores: the forward scorer writing z1
    if ((e = score_tcgen05(d, cnn, k, v, s, 0, d->T, nullptr, nullptr, stream, a.z1)) != cudaSuccess)
      return e;
  } else {
    cnnb::cnnb_z1_kernel<<<grid, cnnb::kThreads, ws_smem, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  cnnb::cnnb_dz_kernel<<<grid, cnnb::kThreads, 0, stream>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (tc && score_backward_dx_tc_supported(d, cnn)) {
    if ((e = score_backward_dx_tc(d, cnn, a.dzp, dk, dv, err, stream)) != cudaSuccess) return e;
  } else {
    cnnb::cnnb_dx_kernel<<<grid, cnnb::kThreads, ws_smem, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (tc) return score_backward_dw1_tc(d, cnn, k, v, s, a.dzp, dw1, err, stream);
  const int chunks = (d->T + cnnb::kDwChunk - 1) / cnnb::kDwChunk;
  const dim3 gw(d->B * chunks, d->Hkv, (2 * d->D) / cnnb::kChanChunk);
  cnnb::cnnb_dw1_kernel<<<gw, cnnb::kThreads, dw_smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace lte
