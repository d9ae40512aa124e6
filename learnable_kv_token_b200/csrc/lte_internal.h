// Internal host-side launchers shared between the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "lte_api.h"
#include "lte_common.cuh"

namespace lte {

// score_cnn.cu
bool score_supported(const lte_cnn* cnn);
cudaError_t score_linear(const lte_dims* d, const lte_cnn* cnn, const void* k, const void* v,
                         Strides4 s, int j_begin, int j_end, float* r, uint8_t* mask,
                         cudaStream_t stream);

// score_tcgen05.cu
bool score_tcgen05_supported(const lte_dims* d, const lte_cnn* cnn, Strides4 s);
// z1 != NULL: write the first layer's pre-activation for tokens [j_begin, j_end)
// (any j_end <= T) into z1 [B*Hkv][c_hid][T] instead of scores (r, mask unused)
cudaError_t score_tcgen05(const lte_dims* d, const lte_cnn* cnn, const void* k, const void* v,
                          Strides4 s, int j_begin, int j_end, float* r, uint8_t* mask,
                          cudaStream_t stream, float* z1 = nullptr);

// score_backward.cu
size_t score_backward_scratch_bytes(const lte_dims* d, const lte_cnn* cnn);
cudaError_t score_backward(const lte_dims* d, const lte_cnn* cnn, const void* k, const void* v,
                           Strides4 s, int n_scored, const float* dr, float* dk, float* dv,
                           float* dw1, float* db1, float* dw2, float* db2, void* scratch,
                           DevError* err, cudaStream_t stream);
// score_backward_tc.cu: dw1 on tcgen05 (bf16, head dim 128, c_hid 32, k1 <= 8)
bool score_backward_tc_supported(const lte_dims* d, const lte_cnn* cnn);
cudaError_t score_backward_dw1_tc(const lte_dims* d, const lte_cnn* cnn, const void* k,
                                  const void* v, Strides4 s, const void* dz_planes, float* dw1,
                                  DevError* err, cudaStream_t stream);
bool score_backward_dx_tc_supported(const lte_dims* d, const lte_cnn* cnn);
cudaError_t score_backward_dx_tc(const lte_dims* d, const lte_cnn* cnn, const void* dz_planes,
                                 float* dk, float* dv, DevError* err, cudaStream_t stream);

// evict_compact.cu
cudaError_t evict_compact(const lte_dims* d, const float* r, const uint8_t* mask, int n_scored,
                          int32_t* idx, int32_t* nret, int32_t* cnt, const void* k,
                          const void* v, Strides4 s, void* k_col, void* v_col,
                          cudaStream_t stream);
cudaError_t retained_lifetimes(const lte_dims* d, const float* r, const int32_t* idx,
                               const int32_t* nret, int32_t* death, cudaStream_t stream);
// relaxed retention: bias[u][slot] = log(r[u][idx[u][slot - s]]) / scale on the
// retained slots of the column segment, 0 elsewhere (slots [0, s + T) plus 64
// zero floats of padding at the end)
size_t slot_bias_floats(const lte_dims* d);
cudaError_t slot_bias(const lte_dims* d, const float* r, const int32_t* idx, const int32_t* nret,
                      float* bias, cudaStream_t stream);
cudaError_t cache_init(const lte_dims* d, const lte_cache* c, const void* k, const void* v,
                       Strides4 s, const float* r, const int32_t* idx, const int32_t* cnt,
                       const int32_t* death, int T_prompt, int n_scored, cudaStream_t stream);

// attn_prefill_*.cu
struct PrefillArgs {
  const lte_dims* d;
  const void *q, *k, *v;
  Strides4 qs, kvs, os;
  const int32_t* cnt;
  const int32_t* death;  // retained lifetimes (LTE_CAP_LOWEST), else NULL
  const void *k_col, *v_col;
  void* o;
  float* lse;
  DevError* err;
  void* scratch;         // workspace after the error word
  size_t scratch_bytes;
  const float* bias;     // relaxed retention: logit offset per column-segment slot, else NULL
};
cudaError_t attn_prefill_simt(const PrefillArgs& a, cudaStream_t stream);
cudaError_t attn_prefill_mma(const PrefillArgs& a, cudaStream_t stream);
bool attn_prefill_tc_supported(const lte_dims* d);
bool attn_prefill_tc_layout_ok(const PrefillArgs& a);
cudaError_t attn_prefill_tc(const PrefillArgs& a, cudaStream_t stream);
size_t attn_prefill_scratch_bytes(const lte_dims* d);

// attn_backward_mma.cu
struct BackwardArgs {
  const lte_dims* d;
  const void *q, *k, *v, *o, *dO;   // contiguous [B,T,H,D] bf16
  const int32_t *cnt, *death, *idx, *nret;
  const void *k_col, *v_col;
  const float* lse;
  float *dq, *dk, *dv;
  DevError* err;                    // the workspace's error word
  void* scratch;                    // workspace after the error word
  const float* bias;                // relaxed retention: slot logit offsets, else NULL
  float* dr;                        // relaxed retention: dL/dr [B,Hkv,T], else NULL
};
size_t attn_backward_scratch_bytes(const lte_dims* d);
cudaError_t attn_backward(const BackwardArgs& a, cudaStream_t stream);
namespace bwd { struct Args; }
// attn_backward_tc.cu: dQ on tcgen05 (head dim 128, G in {1, 2, 4, 8, 16})
bool attn_backward_dq_tc_supported(const lte_dims* d);
cudaError_t attn_backward_dq_tc(const bwd::Args& a, int B, DevError* err, cudaStream_t stream);
cudaError_t attn_backward_dkdv_tc(const bwd::Args& a, int B, DevError* err, cudaStream_t stream);
size_t attn_backward_col_items_cap(const lte_dims* d);   // work items the column pass may list

// decode.cu
size_t decode_scratch_bytes(const lte_dims* d);
bool decode_supported(const lte_dims* d);
cudaError_t decode_step(const lte_dims* d, const lte_cnn* cnn, const lte_cache* c,
                        const void* q_t, const void* k_t, const void* v_t, void* o_t,
                        float* lse_t, int score_batch, DevError* err, void* scratch,
                        cudaStream_t stream);

// decode.cu: the allocation-free variant's scratch (file-scope device array)
cudaError_t noalloc_scratch(void** ptr);

// diag.cu
cudaError_t wait_probe(const int32_t* flag, int32_t expect, unsigned long long limit_ns,
                       DevError* err, cudaStream_t stream);

// gla.cu
cudaError_t gla_prefill(int B, int T, int H, int dk, int dv, int dtype, const void* q,
                        const void* k, const void* v, const float* a, void* o, float* state,
                        cudaStream_t stream);
cudaError_t gla_prefill_tc(int B, int T, int H, const void* q, const void* k, const void* v,
                           const float* a, void* o, float* state, cudaStream_t stream);
cudaError_t gla_decode(int B, int H, int dk, int dv, int dtype, const void* q, const void* k,
                       const void* v, const float* a, void* o, float* state,
                       cudaStream_t stream);

}  // namespace lte
