// Decode indexer on the tcgen05 tensor cores, streaming the FP8 index keys.
//
// For one decode token per sequence b at position t:
//   I[s] = sum_h w[h] * ReLU(q_i[h, :] . k_s),  k_s = scale_s * code_s,
// for the V = floor((t+1)/m) visible entries (B9 indexer equation of the
// "Core formulas chapter"; keys stored in FP8 as in section 7.3 of the
// "DeepSeek paper-feature analysis").  scale_s > 0, so
// ReLU(scale_s x) = scale_s ReLU(x) and the scale is applied per key after
// the contraction.
//
// The keys dominate the bytes of a decode step, so this kernel is an HBM
// stream: TMA brings 128-key FP8 tiles (16 KB, 128-byte swizzle) into a
// 3-stage ring; converter warps turn each byte pair into fp16 with the
// hardware e4m3->f16 conversion (exact: every E4M3 value is a normal fp16)
// and write the MMA's K-major A tile; one lane issues
// M=128 keys x N=H heads x K=128 MMAs (fp16 in, fp32 accumulation) with the
// query's heads (bf16 -> fp16) as B; the same warps read D back from TMEM and
// reduce over heads.  Scores go to a per-sequence fp32 array (L2-resident at
// these sizes) for the selection kernel.
//
// q_i enters as bf16 and is rounded to fp16 for the MMA: exact for every
// value with magnitude in [2^-17, 65504] (bf16 keeps 8 significant bits);
// smaller magnitudes lose low bits (absolute error below 2^-25).
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kKeys = 128;                // keys per tile (MMA M)
constexpr int kCI = 128;                  // index-key dim (bytes per FP8 key)
constexpr int kRawStages = 3;
constexpr int kRawBytes = kKeys * kCI;    // 16 KB
constexpr int kASlab = kKeys * 128;       // 16 KB: 64 fp16 dims x 128 keys
constexpr int kABytes = 2 * kASlab;       // 32 KB
constexpr int kChunk = 2048;              // keys per CTA
constexpr int kThreads = 256;             // warp 0 TMA, warp 1 MMA, warps 4-7 convert + reduce

struct __align__(8) DecIdxBars {
  uint64_t raw_full[kRawStages], raw_empty[kRawStages], a_full, a_empty, d_full[2], d_empty[2],
      drain;
  uint32_t tmem_base;
};

template <int H>
struct DecIdxCfg {
  static constexpr int B_SLAB = H * 128;
  static constexpr int OFF_RAW = 0;
  static constexpr int OFF_A = OFF_RAW + kRawStages * kRawBytes;
  static constexpr int OFF_B = OFF_A + kABytes;
  static constexpr int OFF_W = OFF_B + 2 * B_SLAB;
  static constexpr int OFF_BAR = OFF_W + H * 4;
  static constexpr int SMEM = OFF_BAR + (int)sizeof(DecIdxBars) + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * H < 32 ? 32 : 2 * H;
};

template <int H>
__global__ void __launch_bounds__(kThreads, 2) decode_index_tc_kernel(
    const __grid_constant__ CUtensorMap tm_keys, const float* __restrict__ key_scale,
    const __nv_bfloat16* __restrict__ q_i, const float* __restrict__ w_i,
    const int64_t* __restrict__ pos, int64_t cap, int m, float* __restrict__ scores,
    unsigned int* __restrict__ err) {
  using C = DecIdxCfg<H>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sRaw = smem + C::OFF_RAW;
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sB = smem + C::OFF_B;
  float* sW = reinterpret_cast<float*>(smem + C::OFF_W);
  DecIdxBars* bar = reinterpret_cast<DecIdxBars*>(smem + C::OFF_BAR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t b = blockIdx.y;
  const int64_t t = pos[b];
  const int64_t V = t < 0 ? 0 : min((t + 1) / m, cap);
  const int64_t c0 = (int64_t)blockIdx.x * kChunk;
  const int64_t Vc = max((int64_t)0, min((int64_t)kChunk, V - c0));
  const int ntiles = (int)((Vc + kKeys - 1) / kKeys);
  if (ntiles == 0) return;
  if (flag_value(err) != 0) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRawStages; ++s) {
      mbar_init(&bar->raw_full[s], 1);
      mbar_init(&bar->raw_empty[s], 4);
    }
    mbar_init(&bar->a_full, 4);
    mbar_init(&bar->a_empty, 1);
    for (int p = 0; p < 2; ++p) {
      mbar_init(&bar->d_full[p], 1);
      mbar_init(&bar->d_empty[p], 4);
    }
    mbar_init(&bar->drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  // B operand: the sequence's H query heads, fp16, K-major, 128-byte swizzle
  for (int e = threadIdx.x; e < H * 16; e += kThreads) {
    const int h = e >> 4, ch = e & 15;  // 16 chunks of 8 dims
    float v[8];
    load8(q_i + (b * H + h) * kCI + ch * 8, v);
    uint4 u;
    __half2 p0 = __floats2half2_rn(v[0], v[1]), p1 = __floats2half2_rn(v[2], v[3]);
    __half2 p2 = __floats2half2_rn(v[4], v[5]), p3 = __floats2half2_rn(v[6], v[7]);
    u.x = *reinterpret_cast<uint32_t*>(&p0);
    u.y = *reinterpret_cast<uint32_t*>(&p1);
    u.z = *reinterpret_cast<uint32_t*>(&p2);
    u.w = *reinterpret_cast<uint32_t*>(&p3);
    const int slab = ch >> 3, c8 = ch & 7;
    *reinterpret_cast<uint4*>(sB + slab * C::B_SLAB + h * 128 + ((c8 ^ (h & 7)) * 16)) = u;
  }
  for (int h = threadIdx.x; h < H; h += kThreads) sW[h] = w_i[b * H + h];
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 0) {
    // ------------------------------- TMA producer --------------------------------
    int issued[kRawStages] = {0, 0, 0};
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % kRawStages, u = j / kRawStages;
      if (j >= kRawStages && !mbar_wait(&bar->raw_empty[s], (uint32_t)((u - 1) & 1), err)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar->raw_full[s], kRawBytes);
        tma_load_3d(sRaw + s * kRawBytes, &tm_keys, &bar->raw_full[s], 0,
                    (int)(c0 + (int64_t)j * kKeys), (int)b);
      }
      __syncwarp();
      ++issued[s];
    }
    for (int s = 0; s < kRawStages; ++s)
      if (issued[s] > 0) mbar_wait(&bar->raw_full[s], (uint32_t)((issued[s] - 1) & 1), err, false);
  } else if (warp == 1) {
    // ------------------------------- MMA issuer ----------------------------------
    // kind::f16 with fp16 A and B: format fields 0
    constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(H >> 3) << 17) | ((uint32_t)(kKeys >> 4) << 24);
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    for (int j = 0; j < ntiles; ++j) {
      const int p = j & 1;
      if (!mbar_wait(&bar->a_full, (uint32_t)(j & 1), err)) break;
      if (j >= 2 && !mbar_wait(&bar->d_empty[p], (uint32_t)(((j >> 1) - 1) & 1), err)) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < kCI / 16; ++kk) {
          const uint32_t koff = (uint32_t)((kk & 3) * 32);
          mma_bf16(tmem + p * H, desc_sw128(a0 + (kk >> 2) * kASlab + koff),
                   desc_sw128(b0 + (kk >> 2) * C::B_SLAB + koff), kIdesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar->d_full[p]);
        mma_commit(&bar->a_empty);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(&bar->drain);
    __syncwarp();
    mbar_wait(&bar->drain, 0, err, false);
  } else if (warp >= 4) {
    // ------------------- convert FP8 -> fp16, then reduce over heads --------------
    const int row = (warp - 4) * 32 + lane;  // key row within a tile = TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    for (int j = 0; j <= ntiles; ++j) {
      if (j < ntiles) {
        const int s = j % kRawStages, u = j / kRawStages;
        if (!mbar_wait(&bar->raw_full[s], (uint32_t)(u & 1), err)) break;
        if (j >= 1 && !mbar_wait(&bar->a_empty, (uint32_t)((j - 1) & 1), err)) break;
        const uint8_t* rr = sRaw + s * kRawBytes + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // 16 keys bytes -> 2 fp16 chunks
          const uint4 raw = *reinterpret_cast<const uint4*>(rr + ((c ^ (row & 7)) * 16));
          const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t h[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(
                (__nv_fp8x2_storage_t)(w4[q] & 0xffffu), __NV_E4M3);
            const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(
                (__nv_fp8x2_storage_t)(w4[q] >> 16), __NV_E4M3);
            h[2 * q] = (uint32_t)lo.x | ((uint32_t)lo.y << 16);
            h[2 * q + 1] = (uint32_t)hi.x | ((uint32_t)hi.y << 16);
          }
          // dims 16c .. 16c+15 -> fp16 chunks 2c, 2c+1 of the 128-dim row
          const int slab = c >> 2;
          const int ca = (2 * c) & 7, cb = (2 * c + 1) & 7;
          uint8_t* arow = sA + slab * kASlab + row * 128;
          *reinterpret_cast<uint4*>(arow + ((ca ^ (row & 7)) * 16)) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4*>(arow + ((cb ^ (row & 7)) * 16)) = make_uint4(h[4], h[5], h[6], h[7]);
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bar->raw_empty[s]);
          mbar_arrive(&bar->a_full);
        }
      }
      if (j >= 1) {
        const int jj = j - 1, p = jj & 1;
        if (!mbar_wait(&bar->d_full[p], (uint32_t)((jj >> 1) & 1), err)) break;
        tc_fence_after();
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < H / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(lane_addr + p * H + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            acc = fmaf(sW[c * 32 + i], fmaxf(__uint_as_float(r[i]), 0.f), acc);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->d_empty[p]);
        const int64_t s = c0 + (int64_t)jj * kKeys + row;
        if (s < V) scores[b * cap + s] = acc * key_scale[b * cap + s];
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int H>
cudaError_t launch_h(const csa_cache_desc& d, const CacheView& cv, const int64_t* pos,
                     const void* q_i, const float* w_i, float* scores, unsigned int* err,
                     cudaStream_t s) {
  using C = DecIdxCfg<H>;
  CUtensorMap tk;
  if (!make_tmap_3d(&tk, cv.ikey_fp8, 1, kCI, (uint64_t)d.capacity, (uint64_t)d.batch, kCI,
                    (uint64_t)d.capacity * kCI, kCI, kKeys))
    return cudaErrorInvalidValue;
  auto kern = decode_index_tc_kernel<H>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((d.capacity + kChunk - 1) / kChunk), (unsigned)d.batch);
  kern<<<grid, kThreads, C::SMEM, s>>>(tk, cv.ikey_scale, (const __nv_bfloat16*)q_i, w_i, pos,
                                       d.capacity, d.m, scores, err);
  return cudaGetLastError();
}

}  // namespace

bool decode_index_tc_supported(const csa_cache_desc& d) {
  return !d.is_hca && d.c_i == kCI &&
         (d.nh_i == 16 || d.nh_i == 32 || d.nh_i == 64 || d.nh_i == 128);
}

cudaError_t launch_decode_index_tc(const csa_cache_desc& d, const CacheView& cv,
                                   const int64_t* pos, const void* q_i, const float* w_i,
                                   float* scores, unsigned int* err, cudaStream_t s) {
  switch (d.nh_i) {
    case 16: return launch_h<16>(d, cv, pos, q_i, w_i, scores, err, s);
    case 32: return launch_h<32>(d, cv, pos, q_i, w_i, scores, err, s);
    case 64: return launch_h<64>(d, cv, pos, q_i, w_i, scores, err, s);
    case 128: return launch_h<128>(d, cv, pos, q_i, w_i, scores, err, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace csa
