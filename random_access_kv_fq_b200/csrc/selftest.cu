// Failure-path self test: a kernel whose one bounded wait is on an mbarrier phase that nothing
// completes.  It gives up after a fixed number of polls exactly as the real kernels do (counts
// one timed-out wait and returns), so the host-side report of bounded-wait failures can be
// tested without faulting or hanging a GPU.
#include "fq_internal.h"
#include "sm100_ptx.cuh"

namespace fq {
namespace {

__device__ unsigned int g_selftest_wait_timeouts = 0;

__global__ void wait_on_a_phase_nothing_completes(uint32_t polls) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);  // expects one arrival; no thread ever arrives
    ptx::fence_mbar_init();
  }
  __syncthreads();
  bool done = false;
  for (uint32_t i = 0; i < polls && !done; ++i) done = ptx::mbar_try(&bar, 0u);
  if (threadIdx.x == 0 && !done) atomicAdd(&g_selftest_wait_timeouts, 1u);
}

}  // namespace

cudaError_t wait_timeouts_selftest(bool clear, unsigned* count) {
  return read_wait_counter(g_selftest_wait_timeouts, clear, count);
}

cudaError_t launch_selftest_wait(uint32_t polls, cudaStream_t st) {
  wait_on_a_phase_nothing_completes<<<1, 32, 0, st>>>(polls);
  return cudaGetLastError();
}

}  // namespace fq
