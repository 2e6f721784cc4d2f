// Query / KV-entry RMSNorm and partial RoPE helpers ("DeepSeek-V4:
// million-token context" sections 4.5 "other details", 7.1 Partial RoPE and
// 7.4 Query/KV Entry Normalization: every query head and KV entry is
// RMSNorm-ed before core attention, and the trailing rope_dims dims of
// queries, entries and the attention output are rotated).
//
// Rotation: pair j (dims c - R + 2j, c - R + 2j + 1) turns by angle
// pos * base^(-2j/R).  The angle is formed and reduced modulo 2 pi in double
// precision, so that positions up to millions keep a float-accurate sine and
// cosine, which are then taken in single precision on [-pi, pi].
#pragma once

#include "common.cuh"

namespace csa {

__device__ __forceinline__ void rope_cos_sin(int64_t pos, int j, int rope_dims, float base,
                                             float& c, float& s) {
  const double theta = exp2(-2.0 * (double)j / (double)rope_dims * log2((double)base));
  double a = (double)pos * theta;
  const double two_pi = 6.283185307179586476925286766559;
  a -= two_pi * rint(a / two_pi);
  sincosf((float)a, &s, &c);
}

// (x, y) turned by the angle whose cosine and sine are (c, s).
__device__ __forceinline__ void rope_turn(float& x, float& y, float c, float s) {
  const float xr = x * c - y * s;
  const float yr = x * s + y * c;
  x = xr;
  y = yr;
}

}  // namespace csa

namespace csa {

// Eight consecutive dims d0 .. d0 + 7 (d0 a multiple of 8) of one row whose
// reciprocal RMS is `inv`: scaled by inv * gamma[d], then, if they lie in the
// trailing rope_dims dims, turned pairwise for position `pos`.
__device__ __forceinline__ void norm_rope8(float v[8], int d0, int c, float inv,
                                           const float* __restrict__ gamma, int64_t pos,
                                           int rope_dims, float base) {
#pragma unroll
  for (int q = 0; q < 8; ++q) v[q] = v[q] * inv * __ldg(gamma + d0 + q);
  if (d0 >= c - rope_dims) {
    const int j0 = (d0 - (c - rope_dims)) >> 1;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      float cs, sn;
      rope_cos_sin(pos, j0 + p, rope_dims, base, cs, sn);
      rope_turn(v[2 * p], v[2 * p + 1], cs, sn);
    }
  }
}

}  // namespace csa
