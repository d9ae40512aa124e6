// Gated linear attention, the linear-attention layer of the laLTE hybrid.
//
// "Sparse Linear Attention: Viewing SWA from the Perspective of Linear
// Attention", section "Background: Linear attention": the state is decayed,
// the value-key outer product is written, the query reads it:
//   S_t = S_{t-1} diag(a_t) + v_t k_t^T,   o_t = S_t q_t    (S: d_v x d_k).
// The hybrid that interleaves this layer with LTE is the one of "Alleviating
// Forgetfulness of Linear Attention by Hybrid Sparse Attention and
// Contextualized Learnable Token Eviction" (TL;DR, Abstract).
//
// Prefill runs on tensor cores (gla_tc.cu): chunk-wise, 64 tokens per chunk,
// the state in TMEM.  This file holds the recurrent decode step and the
// dispatch.
//
// Decode: two CTAs of four warps per (batch, head), one per half of the value
// rows, stream the 128x128 fp32 state once (read, decay, add the outer
// product, write) with 16-byte accesses and reduce the row-query dot products
// with warp shuffles.  (Twice as many, smaller CTAs spread the states evenly
// over the SMs: with one CTA per state, 3 or 4 states land on each SM.)
#include <math.h>

#include "lte_common.cuh"
#include "lte_internal.h"

namespace lte {
namespace gla {

constexpr int DK = 128, DV = 128;

// ---------------------------------------------------------------- decode
template <typename TIn>
__global__ void __launch_bounds__(128)
gla_decode_kernel(int H, const TIn* __restrict__ q, const TIn* __restrict__ k,
                  const TIn* __restrict__ v, const float* __restrict__ a, TIn* __restrict__ o,
                  float* __restrict__ state) {
  const int bh = blockIdx.x >> 1, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = (blockIdx.x & 1) * (DV / 2);       // this CTA's half of the value rows
  // Programmatic dependent launch: wait until the previous kernel in the stream
  // has completed (its outputs may be this step's inputs, and it may be the
  // previous step on this state), then let the next kernel launch, so its CTAs
  // are resident and through their prologue when this step ends.  Both are
  // no-ops when the launch did not allow programmatic serialization.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long long vb = (long long)bh * DK;
  float q4[4], k4[4], a4[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    q4[e] = to_f32(q[vb + lane * 4 + e]);
    k4[e] = to_f32(k[vb + lane * 4 + e]);
    a4[e] = a[vb + lane * 4 + e];
  }
  float* st = state + (long long)bh * DV * DK;
  constexpr int kRows = 16;                           // rows per warp (4 warps per half)
  // every row's loads first (16 x 512 B in flight per warp), then update and store
  float4 s4[kRows];
  float vi[kRows];
#pragma unroll
  for (int rr = 0; rr < kRows; ++rr) {
    const int i = row0 + warp * kRows + rr;
    s4[rr] = reinterpret_cast<const float4*>(st + (long long)i * DK)[lane];
    vi[rr] = to_f32(v[(long long)bh * DV + i]);
  }
  float d[kRows];
#pragma unroll
  for (int rr = 0; rr < kRows; ++rr) {
    const int i = row0 + warp * kRows + rr;
    float4 x = s4[rr];
    x.x = fmaf(x.x, a4[0], vi[rr] * k4[0]);
    x.y = fmaf(x.y, a4[1], vi[rr] * k4[1]);
    x.z = fmaf(x.z, a4[2], vi[rr] * k4[2]);
    x.w = fmaf(x.w, a4[3], vi[rr] * k4[3]);
    reinterpret_cast<float4*>(st + (long long)i * DK)[lane] = x;
    d[rr] = x.x * q4[0] + x.y * q4[1] + x.z * q4[2] + x.w * q4[3];
  }
  // the 16 row sums across the 32 lanes: at each step a lane keeps half of its
  // values and adds its partner's copy of them (lanes paired over bit 4, 3, 2,
  // 1, then 0 -- the same pairing tree as a plain butterfly per row)
#pragma unroll
  for (int half = kRows / 2, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
    const bool upper = (lane & bit) != 0;
#pragma unroll
    for (int jj = 0; jj < half; ++jj) {
      const float send = upper ? d[jj] : d[jj + half];
      const float keep = upper ? d[jj + half] : d[jj];
      d[jj] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
    }
  }
  d[0] += __shfl_xor_sync(0xffffffffu, d[0], 1);
  // lane -> row: bits 4, 3, 2, 1 of the lane select the row's bits 3, 2, 1, 0
  if ((lane & 1) == 0) {
    const int row = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
                    ((lane >> 1) & 1);
    o[(long long)bh * DV + row0 + warp * kRows + row] = from_f32<TIn>(d[0]);
  }
}

}  // namespace gla

cudaError_t gla_prefill(int B, int T, int H, int dk, int dv, int dtype, const void* q,
                        const void* k, const void* v, const float* a, void* o, float* state,
                        cudaStream_t stream) {
  if (dtype != LTE_BF16 || dk != gla::DK || dv != gla::DV || T % 64 != 0)
    return cudaErrorNotSupported;
  return gla_prefill_tc(B, T, H, q, k, v, a, o, state, stream);
}

cudaError_t gla_decode(int B, int H, int dk, int dv, int dtype, const void* q, const void* k,
                       const void* v, const float* a, void* o, float* state,
                       cudaStream_t stream) {
  if (dk != gla::DK || dv != gla::DV) return cudaErrorNotSupported;
  // launched with programmatic stream serialization (see the kernel's first lines)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B * H * 2);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (dtype == LTE_BF16)
    return cudaLaunchKernelEx(&cfg, gla::gla_decode_kernel<__nv_bfloat16>, H,
                              (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                              (const __nv_bfloat16*)v, a, (__nv_bfloat16*)o, state);
  return cudaLaunchKernelEx(&cfg, gla::gla_decode_kernel<float>, H, (const float*)q,
                            (const float*)k, (const float*)v, a, (float*)o, state);
}

}  // namespace lte
