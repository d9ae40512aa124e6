// Shared device helpers for the LTE sm_100a kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "lte_api.h"

namespace lte {

// Device error word: the first 16 bytes of every workspace.
struct DevError {
  int32_t code;    // 0 = ok, else LTE_ERR_TIMEOUT / LTE_ERR_DEVICE
  int32_t where;   // id of the wait or check that failed
  int32_t pad[2];
};

// Error-site ids (reported through DevError::where).
enum : int32_t {
  kWhereAttnKvWait = 101,
  kWhereAttnMmaWait = 102,
  kWhereAttnTmemWait = 103,
  kWhereDecodeIndex = 201,
  kWhereDecodeMeta = 202,
};

// Bounded spin: iterations after which a device wait gives up.
constexpr long long kSpinLimit = 1ll << 26;

__device__ __forceinline__ void record_error(DevError* e, int32_t code, int32_t where) {
  if (e == nullptr) return;
  if (atomicCAS(&e->code, 0, code) == 0) atomicExch(&e->where, where);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float siluf_(float x) { return x / (1.0f + expf(-x)); }

// Element strides of a [B, T, H, D] tensor.
struct Strides4 {
  long long b, t, h;
};

}  // namespace lte
