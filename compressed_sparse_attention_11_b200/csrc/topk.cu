// Prefill top-k: one block per query row selects the k best of its V(t)
// visible index scores (section 4.2 step 4 of "DeepSeek-V4: million-token
// context"; ties to the smaller entry index; indices ascending, -1 padded).
#include "launch.h"
#include "topk.cuh"

namespace csa {

constexpr int kSelThreads = 512;
constexpr int64_t kSelSmemKeys = 32768;  // rows up to this long are staged in shared memory
constexpr int kSelCap = 4096;            // candidates kept above the sampled threshold
constexpr int kSelSample = 2048;         // sample size of the threshold estimate

__global__ void __launch_bounds__(kSelThreads) topk_rows_kernel(
    const float* __restrict__ scores, int64_t ld, int64_t n, int m, int64_t E, int k,
    int64_t smem_keys, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelectShared<kSelThreads>& sh = *reinterpret_cast<SelectShared<kSelThreads>*>(smem_raw);
  int32_t* cand = reinterpret_cast<int32_t*>(smem_raw + sizeof(SelectShared<kSelThreads>));
  uint32_t* sample = reinterpret_cast<uint32_t*>(cand + kSelCap);
  uint32_t* keys = sample + kSelSample;
  const int64_t t = blockIdx.x, b = blockIdx.y;
  const int64_t V = min((t + 1) / m, E);
  int32_t* out = idx + (b * n + t) * k;
  if (V <= k) {
    for (int j = threadIdx.x; j < k; j += kSelThreads) out[j] = j < V ? j : -1;
    return;
  }
  const float* row = scores + (b * n + t) * ld;
  if (V <= smem_keys) {
    for (int64_t i = threadIdx.x; i < V; i += kSelThreads) keys[i] = order_key(row[i]);
    __syncthreads();
    block_select_topk_sampled<kSelThreads>(KeysInSmem{keys}, V, k, out, sh, cand, kSelCap,
                                           sample, kSelSample);
  } else {
    block_select_topk_sampled<kSelThreads>(ScoresIn{row}, V, k, out, sh, cand, kSelCap, sample,
                                           kSelSample);
  }
}

cudaError_t launch_topk_rows(const float* scores, int64_t ld, int64_t batch, int64_t n, int m,
                             int64_t E, int k, int32_t* idx, cudaStream_t s) {
  const int64_t smem_keys = E <= kSelSmemKeys ? E : 0;
  const size_t smem = sizeof(SelectShared<kSelThreads>) + (size_t)kSelCap * 4 +
                      (size_t)kSelSample * 4 + (size_t)smem_keys * sizeof(uint32_t);
  cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  dim3 grid((unsigned)n, (unsigned)batch);
  topk_rows_kernel<<<grid, kSelThreads, smem, s>>>(scores, ld, n, m, E, k, smem_keys, idx);
  return cudaGetLastError();
}

}  // namespace csa
