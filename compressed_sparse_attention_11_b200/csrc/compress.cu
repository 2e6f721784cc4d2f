// Token-level KV compressor (CSA overlapped, HCA single-stream).
//
// Defined by the B9 CSA/HCA compressor equations of the "Core formulas
// chapter" and sections 4.1 / 5.1 of "DeepSeek-V4: million-token context":
// entry i, dim d is a per-dimension softmax over the logits Z + B of its rows
// (CSA: m own-block rows of Za/Ca and m previous-block rows of Zb/Cb; the
// first entry has no previous block), applied as Hadamard weights to C.
//
// HBM-streaming kernel: every input row is read exactly once, 16 bytes per
// thread per row (8 dims), and the softmax is kept online in registers
// (running max, running sum, running weighted sum per dim).  The 2m (or m)
// rows of one entry are split over R adjacent lanes (R = 1 for CSA's 8 rows,
// larger for HCA's 128) and merged with warp shuffles.
#include "common.cuh"
#include "launch.h"

namespace csa {

template <typename T>
__global__ void __launch_bounds__(256) compress_kernel(
    const T* __restrict__ ca, const T* __restrict__ cb, const T* __restrict__ za,
    const T* __restrict__ zb, const float* __restrict__ ba, const float* __restrict__ bb,
    int64_t n, int c, int m, int overlap, int64_t E, int r_log2, int64_t items,
    T* __restrict__ out) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const bool valid = g < items;
  const int R = 1 << r_log2;
  const int r = (int)(g & (R - 1));
  int64_t rest = g >> r_log2;
  const int chunks = c >> 3;
  const int chunk = (int)(rest % chunks);
  rest /= chunks;
  const int64_t i = rest % E;
  const int64_t b = rest / E;
  const int d0 = chunk * 8;

  float M[8], S[8], A[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) { M[q] = kNegInf; S[q] = 0.f; A[q] = 0.f; }

  if (valid) {
    const int rows = overlap ? 2 * m : m;
    const int64_t seq = b * n;
    for (int j = r; j < rows; j += R) {
      const T* cp;
      const T* zp;
      const float* bp;
      if (j < m) {
        const int64_t row = seq + i * m + j;
        cp = ca + row * c + d0;
        zp = za + row * c + d0;
        bp = ba + (int64_t)j * c + d0;
      } else {
        if (i == 0) continue;  // previous block of entry 0: logits -inf, rows 0
        const int64_t row = seq + (i - 1) * m + (j - m);
        cp = cb + row * c + d0;
        zp = zb + row * c + d0;
        bp = bb + (int64_t)(j - m) * c + d0;
      }
      float cv[8], zv[8], bv[8];
      load8(cp, cv);
      load8(zp, zv);
      load8(bp, bv);
#pragma unroll
      for (int q = 0; q < 8; ++q) osm_update(M[q], S[q], A[q], zv[q] + bv[q], cv[q]);
    }
  }
  // merge the R partial states of this entry's rows
  for (int off = 1; off < R; off <<= 1) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float m2 = __shfl_xor_sync(0xffffffffu, M[q], off);
      const float s2 = __shfl_xor_sync(0xffffffffu, S[q], off);
      const float a2 = __shfl_xor_sync(0xffffffffu, A[q], off);
      osm_merge(M[q], S[q], A[q], m2, s2, a2);
    }
  }
  if (valid && r == 0) {
    float o[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) o[q] = A[q] / S[q];
    store8(out + (b * E + i) * c + d0, o);
  }
}

template <typename T>
static cudaError_t launch_compress_t(const void* ca, const void* cb, const void* za,
                                     const void* zb, const float* ba, const float* bb,
                                     int64_t batch, int64_t n, int c, int m, int overlap,
                                     void* out, cudaStream_t s) {
  const int64_t E = n / m;
  const int rows = overlap ? 2 * m : m;
  // lanes per entry-chunk: about 8 rows per lane, at most 32
  int r_log2 = 0;
  while ((1 << r_log2) < 32 && (rows >> r_log2) > 8) ++r_log2;
  const int64_t items = batch * E * (c / 8) << r_log2;
  const int64_t blocks = (items + 255) / 256;
  compress_kernel<T><<<(unsigned)blocks, 256, 0, s>>>(
      (const T*)ca, (const T*)cb, (const T*)za, (const T*)zb, ba, bb, n, c, m, overlap, E,
      r_log2, items, (T*)out);
  return cudaGetLastError();
}

cudaError_t launch_compress(const void* ca, const void* cb, const void* za, const void* zb,
                            const float* ba, const float* bb, int64_t batch, int64_t n, int c,
                            int m, int overlap, csa_dtype dt, void* out, cudaStream_t s) {
  if (dt == CSA_F32)
    return launch_compress_t<float>(ca, cb, za, zb, ba, bb, batch, n, c, m, overlap, out, s);
  return launch_compress_t<__nv_bfloat16>(ca, cb, za, zb, ba, bb, batch, n, c, m, overlap,
                                          out, s);
}

}  // namespace csa
