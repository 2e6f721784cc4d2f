// Decode indexer on the tcgen05 tensor cores, FP8 x FP8.
//
// For one decode token per sequence b at position t:
//   I[s] = sum_h w[h] * ReLU(q_i[h, :] . k_s),  k_s = scale_s * code_s,
// for the V = floor((t+1)/m) visible entries (B9 indexer equation of the
// "Core formulas chapter"; the index keys are FP8 as the indexer path of the
// "DeepSeek paper-feature analysis" section 7.3 keeps them).  scale_s > 0,
// so ReLU(scale_s x) = scale_s ReLU(x) and the key scale is applied after
// the contraction.
//
// The keys dominate the bytes of a decode step, so this kernel is an HBM
// stream with the FP8 tiles fed to the tensor core as they arrive: TMA brings
// 128-key tiles (16 KB, 128-byte swizzle) into a 12-stage ring and one lane
// issues M=128 keys x N=2H x K=128 kind::f8f6f4 MMAs straight from the ring.
// The B operand holds each query head twice: hi = E4M3(q/s_h) and
// lo = E4M3(q/s_h - hi), s_h a power of two with max|q_h|/s_h <= 448, so
// s_h (hi + lo) reproduces the bf16 query exactly except for elements below
// 2^-6 s_h in magnitude (absolute error below 2^-10 s_h there).  Two groups
// of four epilogue warps (alternate tiles, up to four accumulators in TMEM)
// add the two halves, apply ReLU, the head weights (with s_h folded in) and
// the key scale; scores go to a per-sequence fp32 array
// (L2-resident at these sizes) for the selection kernel, with the largest
// and smallest score order keys of each sequence (atomicMax / atomicMin into
// `range`, which must hold 0 / ~0 on entry).  One CTA per SM keeps 12 tiles
// (192 KB) in flight.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kKeys = 128;             // keys per tile (MMA M)
constexpr int kCI = 128;               // index-key dim = bytes per FP8 key
constexpr int kStages = 12;              // 192 KB of key tiles in flight per SM
constexpr int kTileBytes = kKeys * kCI;  // 16 KB
constexpr int kChunk = 2048;           // keys per CTA
constexpr int kThreads = 384;          // warp 0 TMA, warp 1 MMA, warps 4-11 epilogue

constexpr int kDBufs = 4;              // TMEM accumulators (tiles in flight past the MMA)

struct __align__(8) DecIdxBars {
  uint64_t full[kStages], empty[kStages], d_full[kDBufs], d_empty[kDBufs], drain;
  uint32_t tmem_base;
};

template <int H>
struct DecIdxCfg {
  static constexpr int N = 2 * H;                  // hi and lo rows per head
  static constexpr int OFF_RAW = 0;
  static constexpr int OFF_B = OFF_RAW + kStages * kTileBytes;
  static constexpr int OFF_W = OFF_B + N * 128;
  static constexpr int OFF_BAR = OFF_W + H * 4;
  static constexpr int SMEM = OFF_BAR + (int)sizeof(DecIdxBars) + 1024;
  static constexpr uint32_t TMEM_COLS = kDBufs * N <= 512 ? kDBufs * N : 512;
  static constexpr int DBUFS = (int)(TMEM_COLS / N);  // 4 for H = 64, 2 for H = 128
};

template <int H>
__global__ void __launch_bounds__(kThreads, 1) decode_index_tc_kernel(
    const __grid_constant__ CUtensorMap tm_keys, const float* __restrict__ key_scale,
    const __nv_bfloat16* __restrict__ q_i, const float* __restrict__ w_i,
    const int64_t* __restrict__ pos, int64_t cap, int m, float* __restrict__ scores,
    unsigned int* __restrict__ range, unsigned int* __restrict__ err) {
  using C = DecIdxCfg<H>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sRaw = smem + C::OFF_RAW;
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
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->full[s], 1);
      mbar_init(&bar->empty[s], 1);
    }
    for (int p = 0; p < kDBufs; ++p) {
      mbar_init(&bar->d_full[p], 1);
      mbar_init(&bar->d_empty[p], 4);
    }
    mbar_init(&bar->drain, 1);
    fence_mbar_init();
    // the key tiles do not depend on the query: start streaming at once
    for (int j = 0; j < ntiles && j < kStages; ++j) {
      mbar_arrive_expect_tx(&bar->full[j], kTileBytes);
      tma_load_3d(sRaw + j * kTileBytes, &tm_keys, &bar->full[j], 0,
                  (int)(c0 + (int64_t)j * kKeys), (int)b);
    }
  }
  if (warp == 1) {
    tmem_alloc(&bar->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  // B operand: per head a power-of-two scale and the hi / lo E4M3 split
  constexpr int kWarps = kThreads / 32, kHPW = (H + kWarps - 1) / kWarps;
  uint2 qraw[kHPW];
#pragma unroll
  for (int i = 0; i < kHPW; ++i) {  // all of this warp's loads in flight at once
    const int h = warp + i * kWarps;
    if (h < H) qraw[i] = *reinterpret_cast<const uint2*>(q_i + (b * H + h) * kCI + lane * 4);
  }
#pragma unroll
  for (int i = 0; i < kHPW; ++i) {
    const int h = warp + i * kWarps;
    if (h >= H) break;
    float v[4];
    {
      const uint2 raw = qraw[i];
      v[0] = __uint_as_float(raw.x << 16);
      v[1] = __uint_as_float(raw.x & 0xffff0000u);
      v[2] = __uint_as_float(raw.y << 16);
      v[3] = __uint_as_float(raw.y & 0xffff0000u);
    }
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    float sc = 1.f;
    if (amax > 0.f) {  // smallest power of two >= amax / 448
      const uint32_t u = __float_as_uint(amax / 448.f);
      sc = (u & 0x007fffffu) == 0 ? __uint_as_float(u) : __uint_as_float((u & 0x7f800000u) + 0x00800000u);
    }
    uint32_t hi4 = 0, lo4 = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x = v[e] / sc;  // exact: sc is a power of two
      const uint8_t hc = e4m3_code(x);
      const uint8_t lc = e4m3_code(x - e4m3_value(hc));
      hi4 |= (uint32_t)hc << (8 * e);
      lo4 |= (uint32_t)lc << (8 * e);
    }
    const int d = lane * 4, ch = d >> 4;
    const int rh = h, rl = H + h;
    *reinterpret_cast<uint32_t*>(sB + rh * 128 + ((ch ^ (rh & 7)) * 16) + (d & 15)) = hi4;
    *reinterpret_cast<uint32_t*>(sB + rl * 128 + ((ch ^ (rl & 7)) * 16) + (d & 15)) = lo4;
    if (lane == 0) sW[h] = w_i[b * H + h] * sc;
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 0) {
    // ------------------------------- TMA producer --------------------------------
    int issued[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) issued[s] = s < ntiles ? 1 : 0;  // prefetched above
    for (int j = kStages; j < ntiles; ++j) {
      const int s = j % kStages, u = j / kStages;
      if (!mbar_wait(&bar->empty[s], (uint32_t)((u - 1) & 1), err)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar->full[s], kTileBytes);
        tma_load_3d(sRaw + s * kTileBytes, &tm_keys, &bar->full[s], 0,
                    (int)(c0 + (int64_t)j * kKeys), (int)b);
      }
      __syncwarp();
      ++issued[s];
    }
    for (int s = 0; s < kStages; ++s)
      if (issued[s] > 0) mbar_wait(&bar->full[s], (uint32_t)((issued[s] - 1) & 1), err, false);
  } else if (warp == 1) {
    // ------------------------------- MMA issuer ----------------------------------
    constexpr uint32_t kIdesc = idesc_e4m3(kKeys, C::N);
    const uint32_t a0 = smem_u32(sRaw), b0 = smem_u32(sB);
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % kStages, u = j / kStages, p = j % C::DBUFS, v = j / C::DBUFS;
      if (!mbar_wait(&bar->full[s], (uint32_t)(u & 1), err)) break;
      if (v >= 1 && !mbar_wait(&bar->d_empty[p], (uint32_t)((v - 1) & 1), err)) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < kCI / 32; ++kk)  // K = 32 bytes per instruction
          mma_f8(tmem + p * C::N, desc_sw128(a0 + s * kTileBytes + kk * 32),
                 desc_sw128(b0 + kk * 32), kIdesc, kk > 0 ? 1u : 0u);
        mma_commit(&bar->d_full[p]);
        mma_commit(&bar->empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(&bar->drain);
    __syncwarp();
    mbar_wait(&bar->drain, 0, err, false);
  } else if (warp >= 4) {
    // ----------- epilogue: hi + lo, ReLU, head weights, key scale ----------------
    // two groups of four warps take alternate tiles, each warp 32 key rows x
    // all heads
    const int quad = warp & 3, grp = (warp - 4) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    uint32_t kmax = 0u, kmin = 0xffffffffu;  // order keys of this thread's scores
    // the key scales do not depend on the MMA: all of this thread's loads go
    // out at once, so one DRAM latency is paid instead of one per tile
    constexpr int kMine = kChunk / kKeys / 2;
    float kscale[kMine];
#pragma unroll
    for (int i = 0; i < kMine; ++i) {
      const int64_t s = c0 + (int64_t)(grp + 2 * i) * kKeys + row;
      kscale[i] = s < V ? __ldcs(key_scale + b * cap + s) : 0.f;
    }
#pragma unroll 1
    for (int i = 0; i < kMine; ++i) {
      const int j = grp + 2 * i;
      if (j >= ntiles) break;
      const int p = j % C::DBUFS, v = j / C::DBUFS;
      const int64_t s = c0 + (int64_t)j * kKeys + row;
      const float ks = kscale[0];  // shift the queue (registers, not a local array)
#pragma unroll
      for (int q = 0; q + 1 < kMine; ++q) kscale[q] = kscale[q + 1];
      if (!mbar_wait(&bar->d_full[p], (uint32_t)(v & 1), err)) break;
      tc_fence_after();
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < H / 32; ++c) {
        uint32_t hi[32], lo[32];
        tmem_ld32(lane_addr + p * C::N + c * 32, hi);
        tmem_ld32(lane_addr + p * C::N + H + c * 32, lo);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          acc = fmaf(sW[c * 32 + i],
                     fmaxf(__uint_as_float(hi[i]) + __uint_as_float(lo[i]), 0.f), acc);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->d_empty[p]);
      if (s < V) {
        const float sc = acc * ks;
        scores[b * cap + s] = sc;
        const uint32_t ky = order_key(sc);
        kmax = max(kmax, ky);
        kmin = min(kmin, ky);
      }
    }
    // the sequence's score range, for the selection kernel
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
      kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
    }
    if (lane == 0) {
      atomicMax(&range[b * 2 + 0], kmax);
      atomicMin(&range[b * 2 + 1], kmin);
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
                     const void* q_i, const float* w_i, float* scores, unsigned int* range,
                     unsigned int* err, cudaStream_t s) {
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
                                       d.capacity, d.m, scores, range, err);
  return cudaGetLastError();
}

}  // namespace

bool decode_index_tc_supported(const csa_cache_desc& d) {
  return !d.is_hca && d.c_i == kCI && (d.nh_i == 64 || d.nh_i == 128);
}

cudaError_t launch_decode_index_tc(const csa_cache_desc& d, const CacheView& cv,
                                   const int64_t* pos, const void* q_i, const float* w_i,
                                   float* scores, unsigned int* range, unsigned int* err,
                                   cudaStream_t s) {
  switch (d.nh_i) {
    case 64: return launch_h<64>(d, cv, pos, q_i, w_i, scores, range, err, s);
    case 128: return launch_h<128>(d, cv, pos, q_i, w_i, scores, range, err, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace csa
