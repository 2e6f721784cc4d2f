// Self-test of the bounded-wait path: one warp waits on a shared-memory
// barrier that is completed first (arrive) or never (the wait gives up after
// the limit and records the timeout in the library's device flag, as every
// kernel of the layer does when an upstream fault leaves it waiting).
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace csa {

namespace {

__global__ void __launch_bounds__(32) selftest_wait_kernel(uint64_t limit_ns, int arrive,
                                                            unsigned int* __restrict__ err) {
  using namespace sm100;
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (arrive && threadIdx.x == 0) mbar_arrive(&bar);
  __syncwarp();
  mbar_wait_limit(&bar, 0, err, limit_ns);
}

}  // namespace

cudaError_t launch_selftest_wait(uint32_t limit_us, bool arrive, unsigned int* err,
                                 cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>((uint64_t)limit_us * 1000u, arrive ? 1 : 0, err);
  return cudaGetLastError();
}

}  // namespace csa
