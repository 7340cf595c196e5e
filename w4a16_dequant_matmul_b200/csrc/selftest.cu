// Self-test of the failure-detection path shared by the pipelined kernels: every mbarrier
// wait in them is bounded, and a wait that gives up records kStTimeout in the device status
// word and lets its kernel return, so the context stays usable. This kernel makes one such
// wait run out on purpose: one thread waits on a freshly initialised mbarrier that nothing
// ever arrives at, with the kernels' own bounded waits (the spinning or the suspending one),
// and records the timeout when the limit passes. No fault, trap or unbounded wait.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace wq {
namespace {

__global__ void bounded_wait_selftest(uint64_t limit_ns, int spin, unsigned* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // phase 0 of `bar` never completes (no arrivals), so the parity-0 wait must give up
    const bool ok = spin ? mbar_wait_spin_bounded(&bar, 0u, limit_ns)
                         : mbar_wait_bounded(&bar, 0u, limit_ns);
    if (!ok) set_status(status, kStTimeout);
  }
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, bool spin, unsigned* status,
                                         cudaStream_t st) {
  bounded_wait_selftest<<<1, 32, 0, st>>>(limit_ns, spin ? 1 : 0, status);
  return cudaGetLastError();
}

}  // namespace wq
