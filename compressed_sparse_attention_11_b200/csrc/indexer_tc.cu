// Lightning-indexer scores on the tcgen05 tensor cores (bf16 in, fp32 out).
//
// I[t, s] = sum_h w[t, h] * ReLU(q_i[t, h, :] . K_i[s, :]) for s < V(t) =
// floor((t+1)/m) (B9 indexer equation of the "Core formulas chapter";
// section 4.2 of "DeepSeek-V4: million-token context").
//
// The contraction runs "swapped": the MMA's M side is 128 compressed keys
// and its N side is 256 (query, head) columns, so D[s, (t, h)] lands in TMEM
// with one key per lane and the head-weighted ReLU reduction over h is a
// per-thread loop in the epilogue (no cross-lane reduction).
//
// One CTA owns 512 (query, head) rows -- 512/H queries -- resident in shared
// memory (loaded once by TMA) and streams the causally visible key tiles
// through a 2-stage TMA ring.  Each key tile feeds two MMAs of N = 256 into
// two TMEM accumulators (256 columns each), so the epilogue of one half
// overlaps the MMA of the other.  Warp roles: warps 0-7 epilogue, warp 8 TMA
// producer, warp 9 MMA issuer (one elected lane).
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kKT = 128;       // keys per tile (MMA M)
constexpr int kHalfCols = 256; // MMA N
constexpr int kStages = 2;
constexpr int kThreads = 320;

struct __align__(8) IdxBars {
  uint64_t a_full[kStages], a_empty[kStages], b_full, d_full[2], d_empty[2], drain;
  uint32_t tmem_base;
};

template <int H, int CI>
struct IdxCfg {
  static constexpr int TQ = 512 / H;     // queries per CTA
  static constexpr int HQ = TQ / 2;      // queries per accumulator half
  static constexpr int QW = 128 / H;     // queries per epilogue warp per half
  static constexpr int SLABS = CI / 64;  // 64-dim (128-byte) K slabs
  static constexpr int B_SLAB = 512 * 128;
  static constexpr int B_BYTES = SLABS * B_SLAB;
  static constexpr int A_SLAB = kKT * 128;
  static constexpr int A_BYTES = SLABS * A_SLAB;
  static constexpr int OFF_A = B_BYTES;
  static constexpr int OFF_W = OFF_A + kStages * A_BYTES;
  static constexpr int OFF_BAR = OFF_W + TQ * H * 4;
  static constexpr int SMEM = OFF_BAR + (int)sizeof(IdxBars) + 1024;  // + base alignment
  static_assert(SMEM <= 232448, "shared memory budget");
};

__device__ __forceinline__ void put_score(float* p, float v) { *p = v; }
__device__ __forceinline__ void put_score(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

// ST: the stored score type (fp32, or bf16 for the bf16-score selection).
template <int H, int CI, typename ST>
__global__ void __launch_bounds__(kThreads, 1) index_scores_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const float* __restrict__ w_i, int64_t n, int m, int64_t E, ST* __restrict__ scores,
    int64_t ld, unsigned int* __restrict__ err) {
  using C = IdxCfg<H, CI>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sB = smem;
  uint8_t* sA = smem + C::OFF_A;
  float* sW = reinterpret_cast<float*>(smem + C::OFF_W);
  IdxBars* bar = reinterpret_cast<IdxBars*>(smem + C::OFF_BAR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t qt = (int64_t)gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int64_t b = blockIdx.y;
  const int64_t t0 = qt * C::TQ;
  const int64_t t_last = min(t0 + C::TQ, n) - 1;
  const int64_t vmax = min((t_last + 1) / m, E);
  const int nkt = (int)((vmax + kKT - 1) / kKT);
  if (nkt == 0) return;  // uniform: no key visible to any query of the tile
  if (flag_value(err) != 0) return;  // an earlier launch gave up a wait: outputs are void

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&bar->a_full[s], 1); mbar_init(&bar->a_empty[s], 1); }
    mbar_init(&bar->b_full, 1);
    for (int p = 0; p < 2; ++p) { mbar_init(&bar->d_full[p], 1); mbar_init(&bar->d_empty[p], 8); }
    mbar_init(&bar->drain, 1);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  for (int e = threadIdx.x; e < C::TQ * H; e += kThreads) {
    const int64_t t = t0 + e / H;
    sW[e] = t < n ? w_i[(b * n + t) * H + (e % H)] : 0.f;
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
      for (int sl = 0; sl < C::SLABS; ++sl)
        for (int box = 0; box < 2; ++box)
          tma_load_3d(sB + sl * C::B_SLAB + box * 256 * 128, &tm_q, &bar->b_full, sl * 64,
                      (int)(t0 * H) + box * 256, (int)b);
    }
    __syncwarp();
    int issued[kStages] = {0, 0};
    bool ok = true;
    for (int j = 0; j < nkt && ok; ++j) {
      const int s = j % kStages, u = j / kStages;
      if (j >= kStages && !mbar_wait(&bar->a_empty[s], (u - 1) & 1, err)) { ok = false; break; }
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar->a_full[s], C::A_BYTES);
        for (int sl = 0; sl < C::SLABS; ++sl)
          tma_load_3d(sA + s * C::A_BYTES + sl * C::A_SLAB, &tm_k, &bar->a_full[s], sl * 64,
                      j * kKT, (int)b);
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
    constexpr uint32_t kIdesc = idesc_bf16(kKT, kHalfCols);
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    bool ok = mbar_wait(&bar->b_full, 0, err);
    for (int j = 0; j < nkt && ok; ++j) {
      const int s = j % kStages, u = j / kStages;
      if (!mbar_wait(&bar->a_full[s], u & 1, err)) break;
      tc_fence_after();
      for (int p = 0; p < 2; ++p) {
        if (j >= 1 && !mbar_wait(&bar->d_empty[p], (j - 1) & 1, err)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < CI / 16; ++kk) {
            const uint32_t koff = (uint32_t)((kk & 3) * 32);
            const uint32_t a_addr = a0 + s * C::A_BYTES + (kk >> 2) * C::A_SLAB + koff;
            const uint32_t b_addr = b0 + (kk >> 2) * C::B_SLAB + p * (kHalfCols * 128) + koff;
            mma_bf16(tmem + p * kHalfCols, desc_sw128(a_addr), desc_sw128(b_addr), kIdesc,
                     kk > 0 ? 1u : 0u);
          }
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
    // ---------------- epilogue: ReLU, head weights, reduction over heads --------------
    const int quad = warp & 3;       // TMEM lanes 32*quad .. 32*quad+31
    const int colhalf = warp >> 2;   // which 128 of the 256 columns
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    for (int j = 0; j < nkt; ++j) {
      bool ok = true;
      for (int p = 0; p < 2; ++p) {
        if (!mbar_wait(&bar->d_full[p], j & 1, err)) { ok = false; break; }
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
            const int col = c * 32 + i;             // within this warp's 128 columns
            const int qq = col / H, h = col % H;    // query within warp, head
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
        const int64_t s = (int64_t)j * kKT + quad * 32 + lane;
#pragma unroll
        for (int qq = 0; qq < C::QW; ++qq) {
          const int64_t t = t0 + p * C::HQ + colhalf * C::QW + qq;
          if (t < n && s < min((t + 1) / m, E)) put_score(scores + (b * n + t) * ld + s, acc[qq]);
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

template <int H, int CI, typename ST>
cudaError_t launch_tc(const void* q_i, const float* w_i, const void* k_i, int64_t batch,
                      int64_t n, int m, ST* scores, int64_t ld, unsigned int* err,
                      cudaStream_t s) {
  using C = IdxCfg<H, CI>;
  const int64_t E = n / m;
  CUtensorMap tq, tk;
  if (!make_tmap_bf16_3d(&tq, q_i, CI, (uint64_t)n * H, batch, CI * 2ull,
                         (uint64_t)n * H * CI * 2, 64, 256) ||
      !make_tmap_bf16_3d(&tk, k_i, CI, E, batch, CI * 2ull, (uint64_t)E * CI * 2, 64, kKT))
    return cudaErrorInvalidValue;
  auto kern = index_scores_tc_kernel<H, CI, ST>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((n + C::TQ - 1) / C::TQ), (unsigned)batch);
  kern<<<grid, kThreads, C::SMEM, s>>>(tq, tk, w_i, n, m, E, scores, ld, err);
  return cudaGetLastError();
}

}  // namespace

bool index_scores_tc_supported(int nh_i, int c_i, csa_dtype dt, const void* q_i,
                               const void* k_i) {
  if (dt != CSA_BF16) return false;
  if (!(c_i == 64 || c_i == 128)) return false;
  if (!(nh_i == 16 || nh_i == 32 || nh_i == 64 || nh_i == 128)) return false;
  return ((reinterpret_cast<uintptr_t>(q_i) | reinterpret_cast<uintptr_t>(k_i)) & 15) == 0;
}

cudaError_t launch_index_scores_tc(const void* q_i, const float* w_i, const void* k_i,
                                   int64_t batch, int64_t n, int nh_i, int c_i, int m,
                                   void* scores, bool bf16_scores, int64_t ld, unsigned int* err,
                                   cudaStream_t s) {
#define CSA_IDX_CASE(HH, CC)                                                                   \
  if (nh_i == HH && c_i == CC)                                                                 \
    return bf16_scores                                                                         \
               ? launch_tc<HH, CC, __nv_bfloat16>(q_i, w_i, k_i, batch, n, m,                  \
                                                  (__nv_bfloat16*)scores, ld, err, s)          \
               : launch_tc<HH, CC, float>(q_i, w_i, k_i, batch, n, m, (float*)scores, ld, err, s);
  CSA_IDX_CASE(64, 128) CSA_IDX_CASE(64, 64) CSA_IDX_CASE(32, 128) CSA_IDX_CASE(32, 64)
  CSA_IDX_CASE(16, 128) CSA_IDX_CASE(16, 64) CSA_IDX_CASE(128, 128) CSA_IDX_CASE(128, 64)
#undef CSA_IDX_CASE
  return cudaErrorInvalidValue;
}

}  // namespace csa
