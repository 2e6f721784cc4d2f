// Low-precision lightning indexer: FP8 query x FP8 key on the tcgen05 tensor
// cores, and index scores stored in bf16 ("DeepSeek paper-feature analysis",
// "Lightning Indexer": a few heads and FP8 make the indexer cheap, and the
// ReLU suits FP8; "FP4 Quantization-Aware Training": index scores in BF16
// instead of FP32).
//
// FP8 form: every query head vector q_i[t, h, :] and every index key k_i[s, :]
// (128 dims) is quantised to E4M3 with one fp32 scale, scale = amax / 448
// (1 when amax = 0), code = E4M3(x / scale) round-to-nearest-even with
// saturation.  Then
//   I[t, s] = s_k[s] * sum_h (w[t, h] s_q[t, h]) ReLU(sum_d q8[t, h, d] k8[s, d])
// since both scales are positive.  The FP8 products are exact in the fp32
// accumulator, so the kernel computes the indexer formula on the dequantised
// vectors up to fp32 summation order.
//
// The scoring kernel has the form of the bf16 one (indexer_tc.cu): 128 keys
// on the MMA's M side, 256 (query, head) columns per accumulator, two
// accumulators in tensor memory, a TMA ring of key tiles; an FP8 row of 128
// dims is one 128-byte swizzled row, so a K = 128 contraction is four
// kind::f8f6f4 MMAs (K = 32 each) per half, half the instructions of bf16,
// and the CTA's 512 query rows take 64 KB of shared memory instead of 128.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kKT = 128;        // keys per tile (MMA M)
constexpr int kHalfCols = 256;  // MMA N
constexpr int kCI = 128;        // index dim = bytes per FP8 row
constexpr int kStages = 4;
constexpr int kThreads = 320;   // warps 0-7 epilogue, 8 TMA, 9 MMA

struct __align__(8) F8Bars {
  uint64_t a_full[kStages], a_empty[kStages], b_full, d_full[2], d_empty[2], drain;
  uint32_t tmem_base;
};

template <int H>
struct F8Cfg {
  static constexpr int TQ = 512 / H;  // queries per CTA
  static constexpr int HQ = TQ / 2;   // queries per accumulator half
  static constexpr int QW = 128 / H;  // queries per epilogue warp per half
  static constexpr int B_BYTES = 512 * kCI;  // 64 KB
  static constexpr int A_BYTES = kKT * kCI;  // 16 KB
  static constexpr int OFF_A = B_BYTES;
  static constexpr int OFF_W = OFF_A + kStages * A_BYTES;
  static constexpr int OFF_BAR = OFF_W + TQ * H * 4;
  static constexpr int SMEM = OFF_BAR + (int)sizeof(F8Bars) + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
};

__device__ __forceinline__ void store_score(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_score(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

// E4M3 codes and fp32 scale of rows of 128 bf16 values: one warp per row,
// four dims per lane.
__global__ void __launch_bounds__(256) quantize_rows_fp8_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t rows, uint8_t* __restrict__ codes,
    float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const uint2 u = __ldcs(reinterpret_cast<const uint2*>(x + r * kCI) + lane);
  const float v[4] = {__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                      __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u)};
  float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float sc = amax > 0.f ? amax / 448.f : 1.f;
  uint32_t packed = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) packed |= (uint32_t)e4m3_code(v[q] / sc) << (8 * q);
  reinterpret_cast<uint32_t*>(codes + r * kCI)[lane] = packed;
  if (lane == 0) scales[r] = sc;
}

template <int H, typename ST>
__global__ void __launch_bounds__(kThreads, 1) index_scores_f8_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const float* __restrict__ q_scale, const float* __restrict__ k_scale,
    const float* __restrict__ w_i, int64_t n, int m, int64_t E, ST* __restrict__ scores,
    int64_t ld, unsigned int* __restrict__ err) {
  using C = F8Cfg<H>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sB = smem;
  uint8_t* sA = smem + C::OFF_A;
  float* sW = reinterpret_cast<float*>(smem + C::OFF_W);
  F8Bars* bar = reinterpret_cast<F8Bars*>(smem + C::OFF_BAR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t qt = (int64_t)gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int64_t b = blockIdx.y;
  const int64_t t0 = qt * C::TQ;
  const int64_t t_last = min(t0 + C::TQ, n) - 1;
  const int64_t vmax = min((t_last + 1) / m, E);
  const int nkt = (int)((vmax + kKT - 1) / kKT);
  if (nkt == 0) return;               // uniform: no key visible to any query of the tile
  if (flag_value(err) != 0) return;   // an earlier launch gave up a wait: outputs are void

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->a_full[s], 1);
      mbar_init(&bar->a_empty[s], 1);
    }
    mbar_init(&bar->b_full, 1);
    for (int p = 0; p < 2; ++p) {
      mbar_init(&bar->d_full[p], 1);
      mbar_init(&bar->d_empty[p], 8);
    }
    mbar_init(&bar->drain, 1);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  // head weights times the query heads' FP8 scales
  for (int e = threadIdx.x; e < C::TQ * H; e += kThreads) {
    const int64_t t = t0 + e / H;
    const int64_t r = (b * n + t) * H + (e % H);
    sW[e] = t < n ? w_i[r] * q_scale[r] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 8) {
    // ---------------- TMA producer -------------------------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      mbar_arrive_expect_tx(&bar->b_full, C::B_BYTES);
      for (int box = 0; box < 2; ++box)
        tma_load_3d(sB + box * 256 * kCI, &tm_q, &bar->b_full, 0, (int)(t0 * H) + box * 256,
                    (int)b);
    }
    __syncwarp();
    int issued[kStages] = {0, 0, 0, 0};
    for (int j = 0; j < nkt; ++j) {
      const int s = j % kStages, u = j / kStages;
      if (j >= kStages && !mbar_wait(&bar->a_empty[s], (u - 1) & 1, err)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar->a_full[s], C::A_BYTES);
        tma_load_3d(sA + s * C::A_BYTES, &tm_k, &bar->a_full[s], 0, j * kKT, (int)b);
      }
      __syncwarp();
      ++issued[s];
    }
    // drain: every load issued has landed before the CTA may exit
    mbar_wait(&bar->b_full, 0, err, false);
    for (int s = 0; s < kStages; ++s)
      if (issued[s] > 0) mbar_wait(&bar->a_full[s], (issued[s] - 1) & 1, err, false);
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------------------------------------------
    constexpr uint32_t kIdesc = idesc_e4m3(kKT, kHalfCols);
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    bool ok = mbar_wait(&bar->b_full, 0, err);
    for (int j = 0; j < nkt && ok; ++j) {
      const int s = j % kStages, u = j / kStages;
      if (!mbar_wait(&bar->a_full[s], u & 1, err)) break;
      tc_fence_after();
      for (int p = 0; p < 2; ++p) {
        if (j >= 1 && !mbar_wait(&bar->d_empty[p], (j - 1) & 1, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < kCI / 32; ++kk)  // K = 32 bytes per instruction
            mma_f8(tmem + p * kHalfCols, desc_sw128(a0 + s * C::A_BYTES + kk * 32),
                   desc_sw128(b0 + p * (kHalfCols * kCI) + kk * 32), kIdesc, kk > 0 ? 1u : 0u);
          mma_commit(&bar->d_full[p]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) mma_commit(&bar->a_empty[s]);
      __syncwarp();
    }
    // drain: all MMAs issued by this warp complete before TMEM is released
    if (lane == 0) mma_commit(&bar->drain);
    __syncwarp();
    mbar_wait(&bar->drain, 0, err, false);
  } else {
    // ---------------- epilogue: ReLU, weights, reduction over heads, key scale -------
    const int quad = warp & 3;      // TMEM lanes 32 quad .. 32 quad + 31 = this thread's key
    const int colhalf = warp >> 2;  // which 128 of the 256 columns
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    for (int j = 0; j < nkt; ++j) {
      bool ok = true;
      const int64_t s = (int64_t)j * kKT + quad * 32 + lane;
      const float ks = s < E ? __ldg(k_scale + b * E + s) : 0.f;
      for (int p = 0; p < 2; ++p) {
        if (!mbar_wait(&bar->d_full[p], j & 1, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float acc[C::QW];
#pragma unroll
        for (int qq = 0; qq < C::QW; ++qq) acc[qq] = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(lane_addr + p * kHalfCols + colhalf * 128 + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const int col = c * 32 + i;           // within this warp's 128 columns
            const int qq = col / H, h = col % H;  // query within warp, head
            const int q_local = p * C::HQ + colhalf * C::QW + qq;
            const float4 wv = *reinterpret_cast<const float4*>(sW + q_local * H + h);
            float a = acc[qq];
            a = fmaf(wv.x, fmaxf(__uint_as_float(r[i + 0]), 0.f), a);
            a = fmaf(wv.y, fmaxf(__uint_as_float(r[i + 1]), 0.f), a);
            a = fmaf(wv.z, fmaxf(__uint_as_float(r[i + 2]), 0.f), a);
            a = fmaf(wv.w, fmaxf(__uint_as_float(r[i + 3]), 0.f), a);
            acc[qq] = a;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->d_empty[p]);
#pragma unroll
        for (int qq = 0; qq < C::QW; ++qq) {
          const int64_t t = t0 + p * C::HQ + colhalf * C::QW + qq;
          if (t < n && s < min((t + 1) / m, E))
            store_score(scores + (b * n + t) * ld + s, acc[qq] * ks);
        }
      }
      if (!ok) break;
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int H, typename ST>
cudaError_t launch_f8_scores(const uint8_t* q8, const float* qs, const uint8_t* k8,
                             const float* ks, const float* w_i, int64_t batch, int64_t n, int m,
                             ST* scores, int64_t ld, unsigned int* err, cudaStream_t s) {
  using C = F8Cfg<H>;
  const int64_t E = n / m;
  CUtensorMap tq, tk;
  if (!make_tmap_3d(&tq, q8, 1, kCI, (uint64_t)n * H, (uint64_t)batch, kCI,
                    (uint64_t)n * H * kCI, kCI, 256) ||
      !make_tmap_3d(&tk, k8, 1, kCI, (uint64_t)E, (uint64_t)batch, kCI, (uint64_t)E * kCI, kCI,
                    kKT))
    return cudaErrorInvalidValue;
  auto kern = index_scores_f8_kernel<H, ST>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((n + C::TQ - 1) / C::TQ), (unsigned)batch);
  kern<<<grid, kThreads, C::SMEM, s>>>(tq, tk, qs, ks, w_i, n, m, E, scores, ld, err);
  return cudaGetLastError();
}

}  // namespace

bool index_fp8_supported(int nh_i, int c_i) {
  return c_i == kCI && (nh_i == 16 || nh_i == 32 || nh_i == 64 || nh_i == 128);
}

cudaError_t launch_quantize_rows_fp8(const void* x, int64_t rows, uint8_t* codes, float* scales,
                                     cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  quantize_rows_fp8_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(
      (const __nv_bfloat16*)x, rows, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_index_scores_fp8(const uint8_t* q8, const float* qs, const uint8_t* k8,
                                    const float* ks, const float* w_i, int64_t batch, int64_t n,
                                    int nh_i, int m, void* scores, bool bf16_scores, int64_t ld,
                                    unsigned int* err, cudaStream_t s) {
#define CSA_F8_CASE(HH)                                                                        \
  if (nh_i == HH)                                                                              \
    return bf16_scores ? launch_f8_scores<HH, __nv_bfloat16>(q8, qs, k8, ks, w_i, batch, n, m, \
                                                             (__nv_bfloat16*)scores, ld, err, s) \
                       : launch_f8_scores<HH, float>(q8, qs, k8, ks, w_i, batch, n, m,         \
                                                     (float*)scores, ld, err, s);
  CSA_F8_CASE(64) CSA_F8_CASE(32) CSA_F8_CASE(16) CSA_F8_CASE(128)
#undef CSA_F8_CASE
  return cudaErrorInvalidValue;
}

}  // namespace csa
