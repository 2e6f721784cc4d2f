// Lightning-indexer scores on CUDA cores (fp32 path and shapes the tcgen05
// kernel in indexer_tc.cu does not take).
//
// I[t, s] = sum_h w[t, h] * ReLU(q_i[t, h, :] . K_i[s, :]) for s < V(t),
// V(t) = floor((t+1)/m)  (B9 indexer equation of the "Core formulas chapter";
// section 4.2 of "DeepSeek-V4: million-token context"; completion rule of
// the reader's notes, section 3).
//
// A block holds a tile of 128 keys (transposed in shared memory, one key per
// thread) and walks a tile of queries; each query's heads are staged in
// shared memory as [dim][head] so one 16-byte load feeds four heads.
#include "common.cuh"
#include "launch.h"

namespace csa {

constexpr int kIdxKeys = 128;   // keys per block (one per thread)
constexpr int kIdxQueries = 16; // queries per block
constexpr int kIdxHG = 32;      // heads accumulated at once

template <typename T>
__global__ void __launch_bounds__(kIdxKeys) index_scores_kernel(
    const T* __restrict__ q_i, const float* __restrict__ w_i, const T* __restrict__ k_i,
    int64_t n, int nh_i, int c_i, int m, int64_t E, float* __restrict__ scores, int64_t ld) {
  extern __shared__ float smem[];
  float* Ks = smem;                          // [c_i][kIdxKeys]
  float* Qs = smem + (size_t)c_i * kIdxKeys; // [c_i][nh_pad]
  const int nh_pad = (nh_i + kIdxHG - 1) / kIdxHG * kIdxHG;
  const int tid = threadIdx.x;
  const int64_t s0 = (int64_t)blockIdx.x * kIdxKeys;
  const int64_t t0 = (int64_t)blockIdx.y * kIdxQueries;
  const int64_t b = blockIdx.z;
  const int64_t t_last = min(t0 + kIdxQueries, n) - 1;
  const int64_t v_last = min((t_last + 1) / m, E);
  if (s0 >= v_last) return;  // no query of this tile sees any key of this tile

  // keys of this tile, transposed
  const int64_t s = s0 + tid;
  for (int d = 0; d < c_i; d += 8) {
    float v[8];
    if (s < E) {
      load8(k_i + (b * E + s) * c_i + d, v);
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = 0.f;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) Ks[(d + q) * kIdxKeys + tid] = v[q];
  }

  for (int64_t t = t0; t <= t_last; ++t) {
    const int64_t V = min((t + 1) / m, E);
    if (s0 >= V) continue;  // uniform over the block
    __syncthreads();        // previous query's Qs no longer in use
    // stage q_i[t] as [dim][head] (heads padded with zeros)
    const T* qt = q_i + ((b * n + t) * nh_i) * c_i;
    for (int e = tid; e < nh_pad * c_i; e += kIdxKeys) {
      const int h = e / c_i, d = e % c_i;
      Qs[d * nh_pad + h] = h < nh_i ? to_f32(qt[(int64_t)h * c_i + d]) : 0.f;
    }
    __syncthreads();
    const float* wt = w_i + (b * n + t) * nh_i;
    float score = 0.f;
    for (int hg = 0; hg < nh_pad; hg += kIdxHG) {
      float acc[kIdxHG];
#pragma unroll
      for (int h = 0; h < kIdxHG; ++h) acc[h] = 0.f;
      for (int d = 0; d < c_i; ++d) {
        const float kv = Ks[d * kIdxKeys + tid];
        const float4* qrow = reinterpret_cast<const float4*>(Qs + d * nh_pad + hg);
#pragma unroll
        for (int h4 = 0; h4 < kIdxHG / 4; ++h4) {
          const float4 qv = qrow[h4];
          acc[4 * h4 + 0] = fmaf(qv.x, kv, acc[4 * h4 + 0]);
          acc[4 * h4 + 1] = fmaf(qv.y, kv, acc[4 * h4 + 1]);
          acc[4 * h4 + 2] = fmaf(qv.z, kv, acc[4 * h4 + 2]);
          acc[4 * h4 + 3] = fmaf(qv.w, kv, acc[4 * h4 + 3]);
        }
      }
#pragma unroll
      for (int h = 0; h < kIdxHG; ++h)
        if (hg + h < nh_i) score = fmaf(wt[hg + h], fmaxf(acc[h], 0.f), score);
    }
    if (s < V) scores[(b * n + t) * ld + s] = score;
  }
}

cudaError_t launch_index_scores(const void* q_i, const float* w_i, const void* k_i,
                                int64_t batch, int64_t n, int nh_i, int c_i, int m,
                                csa_dtype dt, float* scores, int64_t ld, cudaStream_t s) {
  const int64_t E = n / m;
  if (E == 0) return cudaSuccess;
  if (index_scores_tc_supported(nh_i, c_i, dt, q_i, k_i)) {
    unsigned int* err = device_timeout_flag();
    if (err == nullptr) return cudaErrorUnknown;
    return launch_index_scores_tc(q_i, w_i, k_i, batch, n, nh_i, c_i, m, scores, false, ld, err,
                                  s);
  }
  const int nh_pad = (nh_i + kIdxHG - 1) / kIdxHG * kIdxHG;
  const size_t smem = sizeof(float) * ((size_t)c_i * kIdxKeys + (size_t)c_i * nh_pad);
  dim3 grid((unsigned)((E + kIdxKeys - 1) / kIdxKeys),
            (unsigned)((n + kIdxQueries - 1) / kIdxQueries), (unsigned)batch);
  if (dt == CSA_F32) {
    auto kern = index_scores_kernel<float>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kIdxKeys, smem, s>>>((const float*)q_i, w_i, (const float*)k_i, n, nh_i, c_i,
                                      m, E, scores, ld);
  } else {
    auto kern = index_scores_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kIdxKeys, smem, s>>>((const __nv_bfloat16*)q_i, w_i,
                                      (const __nv_bfloat16*)k_i, n, nh_i, c_i, m, E, scores,
                                      ld);
  }
  return cudaGetLastError();
}

}  // namespace csa
