// Gated linear attention (the hybrid's companion layer): placeholder until
// the chunk-wise kernels land; both entry points report "unsupported".
#include "lte_common.cuh"
#include "lte_internal.h"

namespace lte {

cudaError_t gla_prefill(int, int, int, int, int, int, const void*, const void*, const void*,
                        const float*, void*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

cudaError_t gla_decode(int, int, int, int, int, const void*, const void*, const void*,
                       const float*, void*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace lte
