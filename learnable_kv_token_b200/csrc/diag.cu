// Device-wait probe: checks on a live GPU that a bounded wait of the library
// runs out into an error status instead of hanging the device.
//
// Two threads of one CTA share an mbarrier of arrival count 1.  Thread 32
// arrives on it once the device word *flag holds `expect` (it polls for at
// most limit_ns); thread 0 waits for the barrier's phase with
// mbar_wait_bounded, the wait the fused decode kernel uses for its copies and
// hand-offs.  If nothing sets the flag, nobody arrives, the wait runs out
// after limit_ns, LTE_ERR_TIMEOUT (site kWhereWaitProbe) is recorded in the
// error word and the kernel returns: the context stays usable.
#include "lte_common.cuh"
#include "lte_internal.h"

namespace lte {

__global__ void __launch_bounds__(64) wait_probe_kernel(const int32_t* flag, int32_t expect,
                                                        unsigned long long limit_ns,
                                                        DevError* err) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  const uint32_t bar_addr = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_addr));
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 32) {
    const unsigned long long t0 = global_ns();
    while (true) {
      if (*reinterpret_cast<const volatile int32_t*>(flag) == expect) {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar_addr) : "memory");
        break;
      }
      if (global_ns() - t0 > limit_ns) break;          // gives up without arriving
      __nanosleep(1000);
    }
  } else if (threadIdx.x == 0) {
    mbar_wait_bounded(bar_addr, 0, limit_ns, &abort_flag, err, kWhereWaitProbe);
  }
  __syncthreads();
}

cudaError_t wait_probe(const int32_t* flag, int32_t expect, unsigned long long limit_ns,
                       DevError* err, cudaStream_t stream) {
  wait_probe_kernel<<<1, 64, 0, stream>>>(flag, expect, limit_ns, err);
  return cudaGetLastError();
}

}  // namespace lte
