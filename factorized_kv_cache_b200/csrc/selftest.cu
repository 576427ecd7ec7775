// Self-test of the bounded pipeline waits (tpa_selftest_wait_timeout in include/tpa.h).
//
// The tensor-core kernels wait on shared-memory barriers (mbarrier phases) that other roles of
// the same CTA complete; every such wait gives up after a time limit, records
// TPA_DEVERR_TIMEOUT in the device error word and lets the kernel return, so that a broken
// pipeline ends as an error status, not as a GPU that no longer answers.  This kernel runs that
// exact wait on a barrier that nothing ever arrives at, with a caller-chosen limit, so the
// timeout path can be exercised on purpose without a fault: the kernel returns after the limit
// and the context stays usable.
#include "ptx_sm100.cuh"
#include "tpa_internal.h"

namespace tpa {
namespace {

__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns, unsigned int* err) {
  __shared__ alignas(8) uint64_t bar;
  const uint32_t a = ptx::smem_u32(&bar);
  if (threadIdx.x == 0) {
    ptx::mbar_init(a, 1);  // one arrival completes phase 0; none is ever made
    ptx::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !ptx::mbar_wait_bounded(a, 0, limit_ns)) atomicOr(err, TPA_DEVERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(uint64_t limit_ns, unsigned int* err, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, err);
  return cudaGetLastError();
}

}  // namespace tpa
