// csa_index_topk_noalloc: the indexer + top-k entry point for callers that
// cannot hand the library a workspace.
//
// Some callers cannot call cudaMalloc: code running inside another
// framework's memory pool (its caching allocator owns the device memory and
// a side allocation would fragment it or exceed its budget), plugin-style
// enqueue hooks that forbid allocation, and latency-critical serving paths
// where cudaMalloc's implicit device synchronisation is unacceptable.  This
// variant keeps its fp32 score scratch in a file-scope device array instead
// of a caller workspace; it then runs exactly the kernels of csa_index_topk.
//
// Limits and sharing rules:
//  - the array holds kNoAllocScoreSlots fp32 scores (8 MiB per device, held
//    by every GPU that loads the library until the process exits); a call
//    needs batch * n * floor(n/m) slots and is rejected with
//    CSA_ERR_UNSUPPORTED when that is larger;
//  - every call shares the one array: calls whose work overlaps on the GPU
//    (different streams, or concurrent threads) race on it.  Nothing in it
//    has to start at zero: each call writes every score slot it reads.
//  - the first call on a device looks up the array's device address with
//    cudaGetSymbolAddress (with that device current) and caches it; make that
//    first call before any stream capture.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace {

constexpr int64_t kNoAllocScoreSlots = int64_t(1) << 21;  // 8 MiB of fp32
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) float g_noalloc_scores[kNoAllocScoreSlots];

std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kNoAllocMaxDevices] = {};

}  // namespace

extern "C" csa_status csa_index_topk_noalloc(const void* q_i, const float* w_i, const void* k_i,
                                             int64_t batch, int64_t n, int nh_i, int c_i, int m,
                                             int k, csa_dtype dt, int32_t* idx, void* stream) {
  if (m >= 1 && batch > 0 && n > 0) {
    const size_t need = csa_index_topk_workspace(batch, n, nh_i, c_i, m, k);
    if (need > (size_t)kNoAllocScoreSlots * sizeof(float))
      return csa::set_last_error(
          CSA_ERR_UNSUPPORTED,
          "csa_index_topk_noalloc: needs %zu score bytes, the built-in scratch holds %zu "
          "(use csa_index_topk with a workspace)",
          need, (size_t)kNoAllocScoreSlots * sizeof(float));
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return csa::set_last_error(CSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return csa::set_last_error(CSA_ERR_UNSUPPORTED, "device %d beyond the %d supported", dev,
                               kNoAllocMaxDevices);
  float* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scores);
      if (e != cudaSuccess || p == nullptr)
        return csa::set_last_error(CSA_ERR_CUDA, "cudaGetSymbolAddress: %s",
                                   cudaGetErrorString(e));
      g_noalloc_ptr[dev] = static_cast<float*>(p);
    }
    scratch = g_noalloc_ptr[dev];
  }
  return csa_index_topk(q_i, w_i, k_i, batch, n, nh_i, c_i, m, k, dt, idx, scratch,
                        (size_t)kNoAllocScoreSlots * sizeof(float), stream);
}
