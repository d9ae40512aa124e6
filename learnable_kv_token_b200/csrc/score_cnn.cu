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
// it.  bf16 inputs with c_hid * k1 <= 160 use the tensor-core tile of
// score_tc.cuh (layer 1 as one GEMM, weights split bf16 hi + lo); other
// shapes and fp32 inputs use this SIMT tile.  The tile code (score_cnn.cuh) serves lte_score (tokens addressed in a
// [B,T,H,D] tensor, this file) and the decode step's deferred scoring (tokens
// addressed in the circular window segment of the cache, decode.cu).
#include "lte_common.cuh"
#include "lte_internal.h"
#include "score_cnn.cuh"
#include "score_tc.cuh"

namespace lte {

template <typename T, typename KV>
__global__ void __launch_bounds__(kScoreThreads)
score_cnn_kernel(ScoreParams p, KV kv) {
  extern __shared__ float smem[];
  const int jb = p.j_begin + blockIdx.x * kScoreNT;
  if (jb >= p.j_end) return;
  score_tile<T, KV>(p, kv, blockIdx.z, blockIdx.y, jb, p.j_end, p.T_avail, smem);
}

template <typename KV>
__global__ void __launch_bounds__(kTcThreads)
score_cnn_tc_kernel(ScoreParams p, KV kv) {
  extern __shared__ __align__(128) uint8_t smem_tc[];
  const int jb = p.j_begin + blockIdx.x * kScoreNT;
  if (jb >= p.j_end) return;
  score_tile_tc<KV>(p, kv, blockIdx.z, blockIdx.y, jb, p.j_end, p.T_avail, smem_tc);
}

// ---------------------------------------------------------------------------
// Persistent tensor-core scoring for lte_score (bf16, c_hid * k1 <= 160).
// Each CTA keeps one KV head's layer-1 weights resident in shared memory as
// bf16 hi + lo (all 2D input channels, 160 KiB at D = 128), converted once,
// and walks that head's token tiles of all sequences: 48 x rows per tile
// (42 scored tokens with a 5- and a 3-tap layer), 12 warps = 3 row tiles x 4
// column quarters of 40.  Two buffers alternate: one holds a tile's x rows,
// then (once the GEMM has read them) its Z; the next tile's x rows are copied
// into the other buffer (cp.async) while this tile's MMAs run.  Every accumulator receives exactly the MMA
// sequence of score_tile_tc (input-channel chunks of 64, steps of 16, hi then
// lo), and the tap sum, SiLU and layer 2 are the same code path, so each score
// is bit-identical to the decode step's.
constexpr int kPRows = 48;
constexpr int kPWarps = 12;
constexpr int kPThreads = 32 * kPWarps;
constexpr int kPXVec = 4;          // x-row 16-byte vectors per thread and tile at D <= 128

// one x/Z buffer: x [48][2D] bf16, later Z [160][48] fp32
__host__ __device__ inline size_t score_persist_buf_bytes(int D) {
  const size_t x = (size_t)kPRows * 2 * D * 2, z = (size_t)kPRows * kTcN * 4;
  return x > z ? x : z;
}
__host__ __device__ inline size_t score_persist_smem_bytes(int D, int c_hid, int k1, int k2) {
  const int NT = kPRows - (k1 + k2 - 2);
  return 2 * (size_t)kTcN * 2 * D * 2                 // W hi, lo: [2D/64 chunks][160][64] bf16
         + 2 * score_persist_buf_bytes(D)             // two x / Z buffers
         + (size_t)c_hid * (NT + k2 - 1) * 4          // u: [c_hid][NU] fp32
         + (size_t)c_hid * (k2 + 1) * 4;              // w2, b1 of the head
}

// 16-byte async copy global -> shared; src_bytes = 0 writes zeros
__device__ __forceinline__ void cp16_zfill(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void ldsm2_p(uint32_t a, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r0), "=r"(r1)
               : "r"(a));
}

__global__ void __launch_bounds__(kPThreads, 1)
score_persist_tc_kernel(ScoreParams p, LinearKV<__nv_bfloat16> kv, int B) {
  using stc::sw;
  extern __shared__ __align__(128) uint8_t smem_p[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int twoD = 2 * p.D, xrow_b = twoD * 2, cpr = xrow_b / 16;
  const int n_chunks = twoD / kTcKC;
  const int NT = kPRows - (p.k1 + p.k2 - 2), NU = NT + p.k2 - 1;
  const int ncol = p.c_hid * p.k1;
  const size_t wchunk = (size_t)kTcN * kTcKC * 2;              // bytes of one [160][64] chunk
  uint8_t* whi = smem_p;
  uint8_t* wlo = whi + n_chunks * wchunk;
  const size_t bufb = score_persist_buf_bytes(p.D);
  uint8_t* buf0 = wlo + n_chunks * wchunk;                     // x of even tiles, then their Z
  float* us = reinterpret_cast<float*>(buf0 + 2 * bufb);       // [c_hid][NU]
  float* wsm = us + p.c_hid * NU;                              // w2, b1 of head h

  const int h = blockIdx.x % p.Hkv;
  const int slot = blockIdx.x / p.Hkv, n_slots = gridDim.x / p.Hkv;
  const int n_tok = p.j_end - p.j_begin;
  const int tiles_per_unit = (n_tok + NT - 1) / NT;
  const int n_tiles = B * tiles_per_unit;
  if (slot >= n_slots || slot >= n_tiles) return;

  // ---- the head's layer-1 weights, once: W[c*k1 + kk][ch] as bf16 hi + lo
  const float* w1h = p.w1 + (long long)h * p.c_hid * twoD * p.k1;
  for (int i = tid; i < n_chunks * (kTcN - ncol) * kTcKC; i += kPThreads) {
    const int ck = i / ((kTcN - ncol) * kTcKC), rem = i % ((kTcN - ncol) * kTcKC);
    const int n = ncol + rem / kTcKC, k = rem % kTcKC;
    const uint32_t off = ck * wchunk + sw(n, k >> 3, kTcKC * 2) + (k & 7) * 2;
    *reinterpret_cast<__nv_bfloat16*>(whi + off) = __float2bfloat16_rn(0.f);
    *reinterpret_cast<__nv_bfloat16*>(wlo + off) = __float2bfloat16_rn(0.f);
  }
  const int per_c = twoD * p.k1;
  for (int i = tid; i < p.c_hid * per_c; i += kPThreads) {
    const int c = i / per_c, rem = i % per_c, ch = rem / p.k1, kk = rem % p.k1;
    const float w = w1h[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
    const int ck = ch / kTcKC, k = ch % kTcKC;
    const uint32_t off = ck * wchunk + sw(c * p.k1 + kk, k >> 3, kTcKC * 2) + (k & 7) * 2;
    *reinterpret_cast<__nv_bfloat16*>(whi + off) = hi;
    *reinterpret_cast<__nv_bfloat16*>(wlo + off) = lo;
  }

  score_stage_w2(p, h, wsm);                                   // once; visible after the first barrier

  // x rows of tile `t` into buffer `xs` (async): row r holds [k; v] of token
  // x0 + r, zeros outside the tokens; one commit group per tile
  auto load_x = [&](int t, uint8_t* xs) {
    const int b = t / tiles_per_unit, jb = p.j_begin + (t % tiles_per_unit) * NT;
    const int x0 = jb - p.past2 - p.past1;
    const uint32_t xa = stc::sa(xs);
#pragma unroll
    for (int v = 0; v < kPXVec; ++v) {
      const int i = tid + v * kPThreads;
      if (i < kPRows * cpr) {
        const int r = i / cpr, c = i % cpr, xg = x0 + r;
        const bool ok = xg >= 0 && xg < p.T_avail;
        const int xc = ok ? xg : 0, e = c * 8;
        const __nv_bfloat16* src = e < p.D ? kv.krow(b, h, xc) + e : kv.vrow(b, h, xc) + (e - p.D);
        cp16_zfill(xa + sw(r, c, xrow_b), src, ok ? 16 : 0);
      }
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
  };

  const int mt = warp % 3, nq = warp / 3;                      // rows 16*mt, columns 40*nq
  load_x(slot, buf0);
  int par = 0;
#pragma unroll 1
  for (int t = slot; t < n_tiles; t += n_slots, par ^= 1) {
    const int b = t / tiles_per_unit, jb = p.j_begin + (t % tiles_per_unit) * NT;
    const int j_last = min(jb + NT, p.j_end);
    uint8_t* xs = buf0 + par * bufb;                           // this tile's x, then its Z
    float* zs = reinterpret_cast<float*>(xs);                  // [160][48]
    // the other buffer held the previous tile's Z, which its tail has finished reading
    if (t + n_slots < n_tiles) load_x(t + n_slots, buf0 + (par ^ 1) * bufb);
    else asm volatile("cp.async.commit_group;\n" ::: "memory");
    asm volatile("cp.async.wait_group 1;\n" ::: "memory");   // this tile's x has landed
    __syncthreads();                                           // x (and, first time, W) ready

    // ---- Z = X (48 x 2D) . W (2D x 160), weights split hi/lo
    float acc[5][4];
#pragma unroll
    for (int i = 0; i < 5; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
    for (int ck = 0; ck < n_chunks; ++ck) {
      const uint8_t* wh = whi + ck * wchunk;
      const uint8_t* wl = wlo + ck * wchunk;
#pragma unroll
      for (int ks = 0; ks < kTcKC; ks += 16) {
        uint32_t fa[4];
        {
          const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int col = (ck * kTcKC + ks) / 8 + (lane >> 4);
          stc::ldsm4(stc::sa(xs + sw(row, col, xrow_b)), fa);
        }
#pragma unroll
        for (int np = 0; np < 2; ++np) {                       // pairs of n8 tiles
          const int row = nq * 40 + np * 16 + (lane & 7) + (lane >> 4) * 8;
          const int col = ks / 8 + ((lane >> 3) & 1);
          uint32_t bh[4], bl[4];
          stc::ldsm4(stc::sa(wh + sw(row, col, kTcKC * 2)), bh);
          stc::ldsm4(stc::sa(wl + sw(row, col, kTcKC * 2)), bl);
          stc::mma(acc[2 * np], fa, bh[0], bh[1]);
          stc::mma(acc[2 * np + 1], fa, bh[2], bh[3]);
          stc::mma(acc[2 * np], fa, bl[0], bl[1]);
          stc::mma(acc[2 * np + 1], fa, bl[2], bl[3]);
        }
        {                                                      // the quarter's 5th n8 tile
          const int row = nq * 40 + 32 + (lane & 7);
          const int col = ks / 8 + ((lane >> 3) & 1);
          uint32_t h0, h1, l0, l1;
          ldsm2_p(stc::sa(wh + sw(row, col, kTcKC * 2)), h0, h1);
          ldsm2_p(stc::sa(wl + sw(row, col, kTcKC * 2)), l0, l1);
          stc::mma(acc[4], fa, h0, h1);
          stc::mma(acc[4], fa, l0, l1);
        }
      }
    }
    __syncthreads();                                           // every warp has read x: Z replaces it
#pragma unroll
    for (int nt = 0; nt < 5; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = mt * 16 + (lane >> 2) + (e >> 1) * 8;
        const int col = nq * 40 + nt * 8 + (lane & 3) * 2 + (e & 1);
        zs[col * kPRows + row] = acc[nt][e];
      }
    score_tail(p, zs, kPRows, us, wsm, NT, b, h, jb, j_last, p.T_avail);   // barriers at both ends
  }
}

static cudaError_t launch_persist(const ScoreParams& p, const LinearKV<__nv_bfloat16>& kv, int B,
                                  cudaStream_t stream) {
  const size_t smem = score_persist_smem_bytes(p.D, p.c_hid, p.k1, p.k2);
  cudaError_t e = cudaFuncSetAttribute(score_persist_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, n_sm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const int NT = kPRows - (p.k1 + p.k2 - 2);
  const long long tiles = (long long)B * ((p.j_end - p.j_begin + NT - 1) / NT);
  long long slots = n_sm / p.Hkv;
  if (slots < 1) slots = 1;
  if (slots > tiles) slots = tiles;
  score_persist_tc_kernel<<<(unsigned)(slots * p.Hkv), kPThreads, smem, stream>>>(p, kv, B);
  return cudaGetLastError();
}

// the persistent kernel's limits: x rows of a tile fit the per-thread vectors, smem fits
static bool persist_supported(const lte_dims* d, const lte_cnn* cnn) {
  return d->dtype == LTE_BF16 && (d->D == 64 || d->D == 128) &&
         score_tc_supported(cnn->c_hid, cnn->k1, cnn->k2) &&
         kPRows - (cnn->k1 + cnn->k2 - 2) >= 16 &&
         kPRows * (2 * d->D * 2 / 16) <= kPXVec * kPThreads &&
         score_persist_smem_bytes(d->D, cnn->c_hid, cnn->k1, cnn->k2) <= 227 * 1024;
}

template <typename KV>
static cudaError_t launch_tc(const ScoreParams& p, const KV& kv, int B, int tiles,
                             cudaStream_t stream) {
  const size_t smem = score_tc_smem_bytes(p.D, p.c_hid, p.k2);
  cudaError_t e = cudaFuncSetAttribute(score_cnn_tc_kernel<KV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(tiles, p.Hkv, B);
  score_cnn_tc_kernel<KV><<<grid, kTcThreads, smem, stream>>>(p, kv);
  return cudaGetLastError();
}

template <typename T, typename KV>
static cudaError_t launch(const ScoreParams& p, const KV& kv, int B, int tiles,
                          cudaStream_t stream) {
  const size_t smem = sizeof(float) * score_smem_floats(p.D, p.c_hid, p.k1, p.k2);
  cudaError_t e = cudaFuncSetAttribute(score_cnn_kernel<T, KV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(tiles, p.Hkv, B);
  score_cnn_kernel<T, KV><<<grid, kScoreThreads, smem, stream>>>(p, kv);
  return cudaGetLastError();
}

ScoreParams score_params(const lte_dims* d, const lte_cnn* cnn) {
  ScoreParams p{};
  p.Hkv = d->Hkv; p.D = d->D; p.T = d->T;
  p.c_hid = cnn->c_hid; p.k1 = cnn->k1; p.past1 = cnn->past1; p.k2 = cnn->k2; p.past2 = cnn->past2;
  p.w1 = cnn->w1; p.b1 = cnn->b1; p.w2 = cnn->w2; p.b2 = cnn->b2;
  p.sink = d->sink; p.tau = d->tau;
  return p;
}

cudaError_t score_linear(const lte_dims* d, const lte_cnn* cnn, const void* k, const void* v,
                         Strides4 s, int j_begin, int j_end, float* r, uint8_t* mask,
                         cudaStream_t stream) {
  ScoreParams p = score_params(d, cnn);
  p.j_begin = j_begin; p.j_end = j_end; p.T_avail = d->T; p.r = r; p.mask = mask;
  const int tiles = (j_end - j_begin + kScoreNT - 1) / kScoreNT;
  if (tiles == 0) return cudaSuccess;
  if (d->dtype == LTE_BF16) {
    if (score_tcgen05_supported(d, cnn, s))
      return score_tcgen05(d, cnn, k, v, s, j_begin, j_end, r, mask, stream);
    const LinearKV<__nv_bfloat16> kv{(const __nv_bfloat16*)k, (const __nv_bfloat16*)v, s};
    if (persist_supported(d, cnn)) return launch_persist(p, kv, d->B, stream);
    if (score_tc_supported(cnn->c_hid, cnn->k1, cnn->k2)) return launch_tc(p, kv, d->B, tiles, stream);
    return launch<__nv_bfloat16>(p, kv, d->B, tiles, stream);
  }
  return launch<float>(p, LinearKV<float>{(const float*)k, (const float*)v, s}, d->B, tiles,
                       stream);
}

bool score_supported(const lte_cnn* cnn) {
  return cnn->c_hid >= 1 && cnn->c_hid <= kScoreMaxC && cnn->k1 >= 1 && cnn->k1 <= kScoreMaxK &&
         cnn->k2 >= 1 && cnn->k2 <= kScoreMaxK;
}

}  // namespace lte
