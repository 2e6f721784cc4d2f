// Device helpers shared by the tcgen05 attention kernels.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace csa {

// Bounded barrier among the 4 warps that share `bar` (one arrive per warp).
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& phase, unsigned int* err) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) sm100::mbar_arrive(bar);
  const bool ok = sm100::mbar_wait(bar, phase & 1, err);
  ++phase;
  return ok;
}

// Lane i ends with the reduction (max or sum) of element i over the 32 lanes.
template <bool kMax>
__device__ __forceinline__ float transpose_reduce(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1) {
    const bool upper = (lane & half) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, half);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  return v[0];
}

}  // namespace csa
