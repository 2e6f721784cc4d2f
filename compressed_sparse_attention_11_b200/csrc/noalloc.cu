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
//    cudaGetSymbolAddress (with that device current) and caches it.  Under
//    the CUDA runtime's lazy module loading that first lookup may load the
//    library's device code and with it this array (a device allocation made
//    by the runtime, which may synchronise the device); make that first call
//    before any stream capture.  The cached address does not survive
//    cudaDeviceReset: calls after a reset of the device are unsupported.
#include <mutex>
#include <string>

#include "common.cuh"
#include "launch.h"

namespace {

constexpr int64_t kNoAllocScoreSlots = int64_t(1) << 21;  // 8 MiB of fp32
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) float g_noalloc_scores[kNoAllocScoreSlots];

std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Score slots a call needs (batch * n * floor(n/m)), or -1 when that product
// does not fit in 64 bits.
int64_t noalloc_slots(int64_t batch, int64_t n, int m) {
  const int64_t E = n / m;
  int64_t rows = 0, slots = 0;
  if (__builtin_mul_overflow(batch, n, &rows) || __builtin_mul_overflow(rows, E, &slots))
    return -1;
  return slots;
}

}  // namespace

extern "C" csa_status csa_index_topk_noalloc(const void* q_i, const float* w_i, const void* k_i,
                                             int64_t batch, int64_t n, int nh_i, int c_i, int m,
                                             int k, csa_dtype dt, int32_t* idx, void* stream) {
  // the argument rules of csa_index_topk come first, so a bad call gets the
  // same CSA_ERR_INVALID_ARG whatever its size
  if (dt != CSA_F32 && dt != CSA_BF16)
    return csa::set_last_error(CSA_ERR_INVALID_ARG, "dt must be CSA_F32 or CSA_BF16");
  if (batch < 0 || n < 0)
    return csa::set_last_error(CSA_ERR_INVALID_ARG, "batch and n must be >= 0");
  if (nh_i < 1) return csa::set_last_error(CSA_ERR_INVALID_ARG, "nh_i must be >= 1");
  if (c_i < 8 || c_i % 8 != 0)
    return csa::set_last_error(CSA_ERR_INVALID_ARG, "c_i must be a positive multiple of 8");
  if (m < 1) return csa::set_last_error(CSA_ERR_INVALID_ARG, "m must be >= 1");
  if (k < 1) return csa::set_last_error(CSA_ERR_INVALID_ARG, "k must be >= 1");
  if (batch > 0 && n > 0) {
    const int64_t need = noalloc_slots(batch, n, m);
    if (need < 0 || need > kNoAllocScoreSlots)
      return csa::set_last_error(
          CSA_ERR_UNSUPPORTED,
          "csa_index_topk_noalloc: needs batch * n * floor(n/m) = %s score slots, the built-in "
          "scratch holds %lld (use csa_index_topk with a workspace)",
          need < 0 ? "more than 2^63" : std::to_string(need).c_str(),
          (long long)kNoAllocScoreSlots);
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
