// Shared device helpers for the CSA/HCA kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

constexpr float kLog2e = 1.4426950408889634f;
#define kNegInf (-__int_as_float(0x7f800000))

// 2^x on the SFU (PTX ex2.approx); exp(x) is ex2(x * log2(e)).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- 8-element vector loads/stores (16 B of bf16, 32 B of fp32) ----------
__device__ __forceinline__ void load8(const float* p, float v[8]) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float v[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
// plain (coherent) variant for data written earlier in the same kernel
__device__ __forceinline__ void load8_cg(const __nv_bfloat16* p, float v[8]) {
  uint4 u;
  asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "l"(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void store8(float* p, const float v[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float v[8]) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = u;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f32(float& d, float x) { d = x; }
__device__ __forceinline__ void from_f32(__nv_bfloat16& d, float x) { d = __float2bfloat16_rn(x); }

// Float -> uint32 key whose unsigned order is the float order (NaN aside).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of order_key.
__device__ __forceinline__ float key_to_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// E4M3 code of x, round to nearest even, saturating to +-448 (cvt.rn.satfinite).
__device__ __forceinline__ uint8_t e4m3_code(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}
__device__ __forceinline__ float e4m3_value(uint8_t code) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(code, __NV_E4M3);
  return __half2float(*reinterpret_cast<__half*>(&h));
}

// Online-softmax update of one dim: state (M, S, A) takes logit l, value c.
__device__ __forceinline__ void osm_update(float& M, float& S, float& A, float l, float c) {
  if (l > M) {
    const float f = ex2((M - l) * kLog2e);
    S = S * f + 1.f;
    A = A * f + c;
    M = l;
  } else {
    const float w = ex2((l - M) * kLog2e);
    S += w;
    A = fmaf(w, c, A);
  }
}

// Online-softmax state merge: (m, s, a) <- (m, s, a) (+) (m2, s2, a2).
__device__ __forceinline__ void osm_merge(float& m, float& s, float& a, float m2, float s2,
                                          float a2) {
  float mn = fmaxf(m, m2);
  if (mn == kNegInf) return;
  float f1 = ex2((m - mn) * kLog2e), f2 = ex2((m2 - mn) * kLog2e);
  s = s * f1 + s2 * f2;
  a = a * f1 + a2 * f2;
  m = mn;
}

}  // namespace csa
