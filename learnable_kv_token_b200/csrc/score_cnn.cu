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
// lte_score dispatch: bf16 inputs whose CNN fits the tcgen05 scorer
// (score_tcgen05.cu) run there.  Other bf16 shapes use the warp-MMA tile of
// score_tc.cuh (layer 1 as one GEMM, weights split bf16 hi + lo), which is also
// the decode step's deferred scorer; fp32 inputs use the SIMT tile of
// score_cnn.cuh.  In the SIMT tile one CTA scores NT consecutive tokens of one
// (batch, KV head) unit: the [k; v] rows of the tile plus its halo are staged
// once in shared memory as fp32, w1 streams through shared memory in chunks of
// 16 input channels, every layer-1 output accumulates over (channel, tap) in
// ascending order and every score over (hidden channel, tap) in ascending
// order, so a token's score is bit-identical whichever tile, launch or
// addressing mode computes it.  The tile code serves lte_score (tokens
// addressed in a [B,T,H,D] tensor, this file) and the decode step (tokens
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
