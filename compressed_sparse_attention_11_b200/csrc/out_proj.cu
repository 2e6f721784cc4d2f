// Grouped output projection on the tcgen05 tensor cores ("DeepSeek-V4:
// million-token context" section 4.4; V4-Flash shapes in B9 of the "Core
// formulas chapter": n_h = 64 heads of c = 512 in g = 8 groups, d_g = 1024,
// d = 4096).  The heads of group g are consecutive in o [n, n_h, c], so
//   stage 1: z[:, g d_g + j] = sum_k o[:, g (n_h/g) c + k] W1[g, j, k]
//   stage 2: y[:, j]         = sum_k z[:, k] W2[j, k]
// are both "C = A B^T" products with K-major operands: stage 1 is one launch
// over (group, row block, column block) tiles, stage 2 the same kernel with
// one group.  z is kept in bf16 between the stages.
//
// Persistent CTAs (one per SM) walk 128 x 256 output tiles; a 4-stage TMA
// ring brings 64-wide K slabs of A (128 rows, 16 KB) and B (256 rows,
// 32 KB) in the 128-byte swizzle; one lane issues four M = 128, N = 256,
// K = 16 MMAs per slab into one of two TMEM accumulators, so the epilogue of
// a tile (tensor memory -> bf16 -> global, one row per thread) overlaps the
// MMAs of the next.  Warp roles: 0 TMA, 1 MMA, 4-7 epilogue.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int kStages = 4;
constexpr int kThreads = 256;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;

struct __align__(8) GemmBars {
  uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
};
constexpr int OFF_BAR = kStages * STAGE_BYTES;
constexpr int SMEM = OFF_BAR + (int)sizeof(GemmBars) + 1024;
static_assert(SMEM <= 232448, "shared memory budget");

// tile -> (group, row block, column block), column blocks fastest so that
// neighbouring CTAs share the A tile (re-read from L2)
struct TileMap {
  int64_t mblocks;
  int nblocks;
  __device__ void of(int64_t tile, int& g, int64_t& mb, int& nb) const {
    nb = (int)(tile % nblocks);
    const int64_t r = tile / nblocks;
    mb = r % mblocks;
    g = (int)(r / mblocks);
  }
};

__global__ void __launch_bounds__(kThreads, 1) gemm_tn_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
    __nv_bfloat16* __restrict__ c, int64_t ldc, int64_t M, int n_per_group, int K,
    int a_col_step, int64_t tiles, TileMap map, unsigned int* __restrict__ err) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  GemmBars* bar = reinterpret_cast<GemmBars*>(smem + OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (flag_value(err) != 0) return;  // an earlier launch gave up a wait: outputs are void

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->full[s], 1);
      mbar_init(&bar->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bar->acc_full[a], 1);
      mbar_init(&bar->acc_empty[a], 4);  // the four epilogue warps
    }
    mbar_init(&bar->drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const int ksteps = K / BK;

  if (warp == 0) {
    // ---------------- TMA producer -------------------------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
    }
    int64_t it = 0;  // slabs issued
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
      int g, nb;
      int64_t mb;
      map.of(tile, g, mb, nb);
      for (int kk = 0; kk < ksteps; ++kk, ++it) {
        const int s = (int)(it % kStages);
        if (it >= kStages && !mbar_wait(&bar->empty[s], (uint32_t)(((it / kStages) - 1) & 1), err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* st = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&bar->full[s], STAGE_BYTES);
          tma_load_3d(st, &tm_a, &bar->full[s], g * a_col_step + kk * BK, (int)(mb * BM), 0);
          tma_load_3d(st + A_BYTES, &tm_b, &bar->full[s], kk * BK,
                      g * n_per_group + nb * BN, 0);
        }
        __syncwarp();
      }
    }
    // every issued slab has landed before the CTA exits
    for (int64_t r = it > kStages ? it - kStages : 0; r < it; ++r)
      mbar_wait(&bar->full[r % kStages], (uint32_t)((r / kStages) & 1), err, false);
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------------------------------------------
    constexpr uint32_t kIdesc = idesc_bf16(BM, BN);
    const uint32_t s0 = smem_u32(smem);
    int64_t it = 0;
    int local = 0;  // tiles of this CTA
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++local) {
      const int a = local & 1;
      // the accumulator is free once the epilogue read it (two tiles ago)
      if (local >= 2 && !mbar_wait(&bar->acc_empty[a], (uint32_t)(((local >> 1) - 1) & 1), err))
        break;
      tc_fence_after();
      for (int kk = 0; kk < ksteps; ++kk, ++it) {
        const int s = (int)(it % kStages);
        if (!(ok = mbar_wait(&bar->full[s], (uint32_t)((it / kStages) & 1), err))) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t ab = s0 + s * STAGE_BYTES, bb = ab + A_BYTES;
#pragma unroll
          for (int k4 = 0; k4 < BK / 16; ++k4)
            mma_bf16(tmem + a * BN, desc_sw128(ab + k4 * 32), desc_sw128(bb + k4 * 32), kIdesc,
                     (kk | k4) != 0 ? 1u : 0u);
          mma_commit(&bar->empty[s]);
          if (kk == ksteps - 1) mma_commit(&bar->acc_full[a]);
        }
        __syncwarp();
      }
    }
    if (lane == 0) mma_commit(&bar->drain);
    __syncwarp();
    mbar_wait(&bar->drain, 0, err, false);
  } else if (warp >= 4) {
    // ---------------- epilogue: one output row per thread -----------------------------
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
    int local = 0;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++local) {
      int g, nb;
      int64_t mb;
      map.of(tile, g, mb, nb);
      const int a = local & 1;
      if (!mbar_wait(&bar->acc_full[a], (uint32_t)((local >> 1) & 1), err)) break;
      tc_fence_after();
      const int64_t m = mb * BM + row;
      __nv_bfloat16* crow = c + m * ldc + (int64_t)g * n_per_group + nb * BN;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(lane_addr + a * BN + ch * 32, r);
        tmem_ld_wait();
        if (m < M) {
#pragma unroll
          for (int v = 0; v < 4; ++v)
            *reinterpret_cast<uint4*>(crow + ch * 32 + v * 8) = make_uint4(
                pack_bf16x2(__uint_as_float(r[8 * v]), __uint_as_float(r[8 * v + 1])),
                pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3])),
                pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5])),
                pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->acc_empty[a]);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// C[M, G * n_per_group] (row stride ldc) = per group g: A[:, g * a_col_step ..
// + K] (row stride lda) times B[g * n_per_group .. + n_per_group, 0 .. K]^T.
cudaError_t launch_gemm_tn(const void* A, int64_t lda, int64_t a_cols, const void* B, int64_t b_rows,
                           int K, void* C, int64_t ldc, int64_t M, int n_per_group, int G,
                           int a_col_step, unsigned int* err, cudaStream_t s) {
  CUtensorMap ta, tb;
  if (!make_tmap_bf16_3d(&ta, A, (uint64_t)a_cols, (uint64_t)M, 1, (uint64_t)lda * 2,
                         (uint64_t)lda * 2 * M, BK, BM) ||
      !make_tmap_bf16_3d(&tb, B, (uint64_t)K, (uint64_t)b_rows, 1, (uint64_t)K * 2,
                         (uint64_t)K * 2 * b_rows, BK, BN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gemm_tn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM);
  if (e != cudaSuccess) return e;
  TileMap map{(M + BM - 1) / BM, n_per_group / BN};
  const int64_t tiles = (int64_t)G * map.mblocks * map.nblocks;
  const unsigned grid = (unsigned)std::min<int64_t>(tiles, sm_count());
  gemm_tn_kernel<<<grid, kThreads, SMEM, s>>>(ta, tb, (__nv_bfloat16*)C, ldc, M, n_per_group, K,
                                              a_col_step, tiles, map, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_grouped_out_proj(const void* o, int64_t rows, int nh, int c, int G, int dg,
                                    int d, const void* w1, const void* w2, void* z, void* y,
                                    cudaStream_t s) {
  unsigned int* err = device_timeout_flag();
  if (err == nullptr) return cudaErrorUnknown;
  const int kin = nh / G * c;
  cudaError_t e = launch_gemm_tn(o, (int64_t)nh * c, (int64_t)nh * c, w1, (int64_t)G * dg, kin, z,
                                 (int64_t)G * dg, rows, dg, G, kin, err, s);
  if (e != cudaSuccess) return e;
  return launch_gemm_tn(z, (int64_t)G * dg, (int64_t)G * dg, w2, d, G * dg, y, d, rows, d, 1, 0,
                        err, s);
}

}  // namespace csa
