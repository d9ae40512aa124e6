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
  kWhereWaitProbe = 301,
};

// Bounded spin: iterations after which a device wait gives up.
constexpr long long kSpinLimit = 1ll << 26;

__device__ __forceinline__ void record_error(DevError* e, int32_t code, int32_t where) {
  if (e == nullptr) return;
  if (atomicCAS(&e->code, 0, code) == 0) atomicExch(&e->where, where);
}

// Global time in nanoseconds.
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// True once phase `parity` of the shared-memory mbarrier at `bar` has completed.
__device__ __forceinline__ bool mbar_try_wait_parity(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of an mbarrier: true once the phase has
// completed; false when the CTA is aborting (*abort_flag set by another wait)
// or when limit_ns of global time have passed, in which case it records
// LTE_ERR_TIMEOUT (site `where`) in the error word and sets *abort_flag so that
// the CTA's other waits give up as well.  No wait of the library spins for ever.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  unsigned long long limit_ns,
                                                  volatile int* abort_flag, DevError* err,
                                                  int32_t where) {
  if (mbar_try_wait_parity(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try_wait_parity(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_ns() - t0 > limit_ns) {
      record_error(err, LTE_ERR_TIMEOUT, where);
      *abort_flag = 1;
      return false;
    }
  }
}

// Retained tokens a row (or the cache) holds when n have left the window with
// a keep decision: under LTE_CAP_FIRST only the first C are stored, so the
// slot range [max(0, n' - C), n') of the compacted list, n' = this value,
// covers both policies.
__host__ __device__ __forceinline__ int held_retained(int n, int cap, int policy) {
  return (policy == LTE_CAP_FIRST && n > cap) ? cap : n;
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
