// Self-check of the bounded-wait error path shared by every kernel of the
// library.  A forward kernel that waits on an mbarrier (a bulk copy landing, a
// tensor-core commit) polls it a bounded number of times; if the phase never
// completes it sets LB_ERR_TIMEOUT in the status word of its workspace and
// returns instead of hanging the GPU.  This kernel takes that path on purpose:
// it initialises an mbarrier that nothing arrives on and issues no copy (so no
// transfer is left in flight when it gives up), waits with the same
// try_wait.parity poll and suspend hint as the forward kernels, and after
// `polls` failed polls raises the bit.  The host then reads and clears it with
// littlebit_device_status, and the context stays usable.
#include <cuda_runtime.h>

#include "lb_internal.h"

namespace lb {
namespace {

__device__ __forceinline__ uint32_t shared_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__global__ void wait_timeout_probe_kernel(unsigned int* status, int polls) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(shared_addr(&bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  bool done = false;
  for (int i = 0; i < polls && !done; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0, 1000;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(shared_addr(&bar))
        : "memory");
    done = ok != 0;
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    if (!done) atomicOr(status, 1u << LB_ERR_TIMEOUT);
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(shared_addr(&bar)) : "memory");
  }
}

}  // namespace

cudaError_t launch_wait_timeout_probe(unsigned int* status, int polls, cudaStream_t st) {
  if (!status || polls < 1 || polls > kSpinLimit) return cudaErrorInvalidValue;
  wait_timeout_probe_kernel<<<1, 32, 0, st>>>(status, polls);
  return cudaGetLastError();
}

}  // namespace lb
