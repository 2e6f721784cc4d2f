// RMSNorm + partial RoPE of whole rows (query heads, window rows, compressed
// entries), the per-row step before core attention in sections 4.5 and 7.4
// of "DeepSeek-V4: million-token context":
//   out[r, :] = RoPE_{pos(r)}(x[r, :] / sqrt(mean(x[r, :]^2) + eps) * gamma)
// with the rotation on the trailing rope_dims dims only (section 7.1).
//
// HBM-bound: one warp per row, each lane 8 consecutive dims per 256-dim
// stripe (16-byte loads of bf16), the sum of squares reduced by shuffles.
// Rows are [batch, n, heads, c]; the row of token t rotates by t * pos_mul
// (1 for queries and window rows, m for compressed entries, whose position is
// their block's first token).
#include "common.cuh"
#include "launch.h"
#include "rope.cuh"

namespace csa {

namespace {

constexpr int kWarps = 8;
constexpr int kMaxStripes = 4;  // c <= 1024

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) norm_rope_rows_kernel(
    const T* __restrict__ x, int64_t rows, int heads, int64_t n, int c, int64_t pos_mul,
    const float* __restrict__ gamma, float eps, int rope_dims, float base, T* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t t = (row / heads) % n;
  const T* src = x + row * c;
  float v[kMaxStripes][8];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxStripes; ++i) {
    const int d0 = 8 * (lane + 32 * i);
    if (d0 < c) {
      load8(src + d0, v[i]);
#pragma unroll
      for (int q = 0; q < 8; ++q) ss = fmaf(v[i][q], v[i][q], ss);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv = 1.f / sqrtf(ss / (float)c + eps);
#pragma unroll
  for (int i = 0; i < kMaxStripes; ++i) {
    const int d0 = 8 * (lane + 32 * i);
    if (d0 < c) {
      norm_rope8(v[i], d0, c, inv, gamma, t * pos_mul, rope_dims, base);
      store8(out + row * c + d0, v[i]);
    }
  }
}

}  // namespace

cudaError_t launch_norm_rope_rows(const void* x, int64_t batch, int64_t n, int heads, int c,
                                  int64_t pos_mul, const csa_norm_rope* nr, csa_dtype dt,
                                  void* out, cudaStream_t s) {
  const int64_t rows = batch * n * heads;
  if (rows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + kWarps - 1) / kWarps);
  if (dt == CSA_BF16)
    norm_rope_rows_kernel<__nv_bfloat16><<<grid, kWarps * 32, 0, s>>>(
        (const __nv_bfloat16*)x, rows, heads, n, c, pos_mul, nr->gamma, nr->eps, nr->rope_dims,
        nr->rope_base, (__nv_bfloat16*)out);
  else
    norm_rope_rows_kernel<float><<<grid, kWarps * 32, 0, s>>>(
        (const float*)x, rows, heads, n, c, pos_mul, nr->gamma, nr->eps, nr->rope_dims,
        nr->rope_base, (float*)out);
  return cudaGetLastError();
}

}  // namespace csa
