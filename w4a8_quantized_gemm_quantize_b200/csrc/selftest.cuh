// Self-test of the failure path shared by every kernel of the library: a
// bounded mbarrier wait that nothing completes must give up by itself after
// its time limit, record its code in the device error word and let the
// kernel return, leaving the CUDA context usable.
#pragma once
#include "ptx.cuh"

namespace w4a8 {

// One warp; thread 0 waits on a fresh mbarrier (one pending arrival that
// never comes) with the given limit.
__global__ void bounded_wait_selftest_kernel(int* err, uint64_t limit_ns, int code) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) (void)mbar_wait_limit(&bar, 0, nullptr, DevErr{err}, code, limit_ns);
}

}  // namespace w4a8
