// selftest.cu -- failure-detection self-test of the bounded device waits.
//
// Every mbarrier wait in the library's kernels is bounded in time; when the
// bound runs out the kernel records kDevTimeout in the context's status word
// and returns instead of hanging, and the host reports KVC_ERR_DEVICE_TIMEOUT
// at its next synchronising call.  This kernel exercises that path on
// purpose and harmlessly: one thread initialises an mbarrier that expects one
// arrival, never arrives on it, and waits for its phase with the given limit.
#include "kvc_internal.h"
#include "tc_ptx.cuh"

namespace kvc {
namespace {

__global__ void wait_timeout_probe_kernel(int32_t *status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(&bar, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const uint64_t t0 = global_ns();
  while (!mbar_try(&bar, 0)) {  // phase 0 never completes: nothing arrives
    if (global_ns() - t0 > limit_ns) {
      atomicCAS(status, kDevOk, kDevTimeout);
      return;
    }
  }
}

}  // namespace

cudaError_t launch_wait_timeout_probe(int32_t *status, uint32_t limit_ms, cudaStream_t s) {
  wait_timeout_probe_kernel<<<1, 1, 0, s>>>(status, (uint64_t)limit_ms * 1000000ull);
  return cudaGetLastError();
}

}  // namespace kvc
