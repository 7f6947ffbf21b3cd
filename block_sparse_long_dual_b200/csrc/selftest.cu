// Self-test of the bounded-wait mechanism every kernel here relies on: a CTA
// waits on an mbarrier phase that nothing completes (or, for the positive
// case, that its own thread completes) with the same bounded try_wait loop the
// kernels use, and reports SFA_ERR_TIMEOUT when the limit runs out.  No fault,
// trap or endless loop is involved: the wait ends by itself and the context
// stays usable.
#include "common.cuh"
#include "kernels.h"

namespace sfa {

namespace {

__global__ void bounded_wait_kernel(int* status, uint64_t limit_ns, int arrive) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = (uint32_t)__cvta_generic_to_shared(&bar);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0 && arrive)
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(b) : "memory");
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    bool ok = false;
    for (;;) {
      uint32_t done;
      asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                   "selp.u32 %0, 1, 0, p;\n\t}" : "=r"(done) : "r"(b), "r"(0u) : "memory");
      if (done) { ok = true; break; }
      if (globaltimer_ns() - t0 > limit_ns) break;
    }
    *status = ok ? SFA_OK : SFA_ERR_TIMEOUT;
  }
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(int* status, uint64_t limit_ns, int arrive, cudaStream_t st) {
  bounded_wait_kernel<<<1, 32, 0, st>>>(status, limit_ns, arrive);
  return cudaGetLastError();
}

}  // namespace sfa
