// Decode attention on the tcgen05 tensor cores over the FP8/bf16 cache: one
// 128-entry tile of one sequence's entry set per CTA.
//
// For the decode token of sequence b at position t, E_t is (CSA) the selected
// entries sel[b, :] with 0 <= s < V = floor((t+1)/m), or (HCA) every visible
// entry, followed by the window rows max(0, t-W+1) .. t from the ring
// (sections 4.3 / 4.5 of "DeepSeek-V4: million-token context"; entries stored
// as FP8 codes with one fp32 scale plus bf16 RoPE dims, section 7.3 of the
// "DeepSeek paper-feature analysis").  Each CTA takes tile j of E_t:
//   1. all 384 threads gather the tile -- FP8 codes dequantised to bf16
//      (code * scale), RoPE dims and window rows copied -- into the same
//      128-byte-swizzled slab layout as the prefill kernel, with many loads
//      in flight per thread (a decode step has few queries, so the gather's
//      memory parallelism decides the time);
//   2. S^T = K Q^T (M = 128 entries, N = 64 heads) on the tensor core;
//   3. softmax statistics of the tile (max, then exp2 and row sums);
//   4. O^T = V^T P^T (four M = 128 dim chunks);
//   5. the tile's unnormalised O, max and sum go to the partial buffers, and
//      a combine kernel merges the tiles of each sequence with the sink.
// With a single tile per sequence the CTA writes the final output itself.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"
#include "tc_attn_util.cuh"

namespace csa {

namespace {

constexpr int kNH = 64, kC = 512, kTE = 128;
constexpr int kSlabs = kC / 64;
constexpr int kSlabBytes = kTE * 128;
constexpr int kQSlabBytes = kNH * 128;
constexpr int kThreads = 384;  // gather: all; then warps 0-7 softmax/epilogue, warp 8 MMA
constexpr int kMmaWarp = 8;
constexpr int kMaxSelDec = 1024;

struct __align__(8) DecAttnBars {
  uint64_t q_full, s_full, p_full, o_full, grp[2];
  uint32_t tmem_base;
  int nsel;
};

constexpr int OFF_Q = 0;
constexpr int OFF_KV = OFF_Q + kSlabs * kQSlabBytes;
constexpr int OFF_P = OFF_KV + kSlabs * kSlabBytes;
constexpr int OFF_LIST = OFF_P + kTE * 128;
constexpr int OFF_RED = OFF_LIST + kMaxSelDec * 4;      // [2 (max,sum)][2 hh][4 quad][32]
constexpr int OFF_SCAN = OFF_RED + 2 * 2 * 4 * 32 * 4;  // [12] warp counts
constexpr int OFF_BAR = OFF_SCAN + 64;
constexpr int SMEM = OFF_BAR + (int)sizeof(DecAttnBars) + 1024;
static_assert(SMEM <= 232448, "shared memory budget");

constexpr uint32_t kColS = 0, kColO = 64;

__global__ void __launch_bounds__(kThreads, 1) decode_attn_tile_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CacheView cv,
    const int64_t* __restrict__ pos, const int32_t* __restrict__ sel, int k, int window, int m,
    int64_t cap, int rope, const float* __restrict__ sink, float scale, int ntile_max,
    float* __restrict__ part_o, float* __restrict__ part_ms, __nv_bfloat16* __restrict__ out,
    unsigned int* __restrict__ err) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem + OFF_Q;
  uint8_t* sKV = smem + OFF_KV;
  uint8_t* sP = smem + OFF_P;
  int32_t* list = reinterpret_cast<int32_t*>(smem + OFF_LIST);
  float* red = reinterpret_cast<float*>(smem + OFF_RED);
  int* wcount = reinterpret_cast<int*>(smem + OFF_SCAN);
  DecAttnBars* bar = reinterpret_cast<DecAttnBars*>(smem + OFF_BAR);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  const int64_t b = blockIdx.y;
  const int64_t t = pos[b];
  const int64_t V = t < 0 ? 0 : min((t + 1) / m, cap);
  const int64_t w0 = max((int64_t)0, t - window + 1);
  const int nwin = t < 0 ? 0 : (int)(t - w0 + 1);
  const bool direct = ntile_max == 1;
  const int64_t pbase = (b * ntile_max + tile) * kNH;
  if (flag_value(err) != 0) return;

  // -------- the entry list: valid selections in order (CSA) or 0..V-1 (HCA) ----
  int nsel;
  if (sel != nullptr) {
    const int32_t* row = sel + b * k;
    const int per = (k + kThreads - 1) / kThreads;
    const int lo = min(k, tid * per), hi = min(k, lo + per);
    int cnt = 0;
    for (int j = lo; j < hi; ++j) cnt += (row[j] >= 0 && row[j] < V) ? 1 : 0;
    int inc = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += v;
    }
    if (lane == 31) wcount[warp] = inc;
    __syncthreads();
    int base = 0;
    nsel = 0;
    for (int w = 0; w < kThreads / 32; ++w) {
      if (w < warp) base += wcount[w];
      nsel += wcount[w];
    }
    int p = base + inc - cnt;
    for (int j = lo; j < hi; ++j)
      if (row[j] >= 0 && row[j] < V) list[p++] = row[j];
    __syncthreads();
  } else {
    nsel = (int)V;
  }
  const int N = nsel + nwin;
  const int T = (N + kTE - 1) / kTE;
  if (tile >= T) {  // an empty tile: contributes nothing to the combine
    if (!direct && tid < kNH) {
      part_ms[(pbase + tid) * 2 + 0] = kNegInf;
      part_ms[(pbase + tid) * 2 + 1] = 0.f;
    }
    return;
  }

  if (tid == 0) {
    mbar_init(&bar->q_full, 1);
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->p_full, 8);
    mbar_init(&bar->o_full, 1);
    mbar_init(&bar->grp[0], 4);
    mbar_init(&bar->grp[1], 4);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  if (tid == 0) {
    mbar_arrive_expect_tx(&bar->q_full, kSlabs * kQSlabBytes);
    for (int s = 0; s < kSlabs; ++s)
      tma_load_3d(sQ + s * kQSlabBytes, &tm_q, &bar->q_full, s * 64, 0, (int)b);
  }

  // -------- gather: 128 rows x 64 chunks of 8 dims, 8 loads in flight/thread ----
  const int body = kC - rope;
  constexpr int kUnroll = 8;
  for (int e0 = tid; e0 < kTE * 64; e0 += kThreads * kUnroll) {
    uint4 v[kUnroll];
    float sc[kUnroll];
    bool fp8[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int e = e0 + u * kThreads;
      v[u] = make_uint4(0, 0, 0, 0);
      sc[u] = 0.f;
      fp8[u] = false;
      if (e >= kTE * 64) continue;
      const int r = e >> 6, c = e & 63, d0 = c * 8;
      const int slot = tile * kTE + r;
      if (slot < nsel) {
        const int64_t es = b * cap + (sel != nullptr ? (int64_t)list[slot] : (int64_t)slot);
        if (d0 < body) {
          const uint2 c8 = *reinterpret_cast<const uint2*>(cv.entry_fp8 + es * body + d0);
          v[u].x = c8.x;
          v[u].y = c8.y;
          sc[u] = cv.entry_scale[es];
          fp8[u] = true;
        } else {
          v[u] = *reinterpret_cast<const uint4*>(cv.entry_rope + es * rope + (d0 - body));
        }
      } else if (slot < N) {
        const int64_t u_pos = w0 + (slot - nsel);
        v[u] = *reinterpret_cast<const uint4*>(cv.window + (b * window + u_pos % window) * kC +
                                               d0);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int e = e0 + u * kThreads;
      if (e >= kTE * 64) continue;
      const int r = e >> 6, c = e & 63;
      uint4 o = v[u];
      if (fp8[u]) {
        const uint32_t w2[2] = {v[u].x, v[u].y};
        uint32_t q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t pair = (w2[i >> 1] >> ((i & 1) * 16)) & 0xffffu;
          q[i] = pack_bf16x2(e4m3_value((uint8_t)(pair & 0xff)) * sc[u],
                             e4m3_value((uint8_t)(pair >> 8)) * sc[u]);
        }
        o = make_uint4(q[0], q[1], q[2], q[3]);
      }
      const int slab = c >> 3, cs = c & 7;
      *reinterpret_cast<uint4*>(sKV + slab * kSlabBytes + r * 128 + ((cs ^ (r & 7)) * 16)) = o;
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == kMmaWarp) {
    // -------------------------------- MMA ----------------------------------------
    constexpr uint32_t kIdQK = idesc_bf16(kTE, kNH, 0, 0);
    constexpr uint32_t kIdPV = idesc_bf16(128, kNH, 1, 1);
    const uint32_t kv0 = smem_u32(sKV), q0 = smem_u32(sQ), p0 = smem_u32(sP);
    if (mbar_wait(&bar->q_full, 0, err)) {
      tc_fence_after();
      if (lane == 0) {
        for (int s = 0; s < kSlabs; ++s)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + kColS, desc_sw128(kv0 + s * kSlabBytes + kk * 32),
                     desc_sw128(q0 + s * kQSlabBytes + kk * 32), kIdQK, (s | kk) != 0 ? 1u : 0u);
        mma_commit(&bar->s_full);
      }
      __syncwarp();
      if (mbar_wait(&bar->p_full, 0, err)) {
        tc_fence_after();
        if (lane == 0) {
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int kk = 0; kk < kTE / 16; ++kk)
              mma_bf16(tmem + kColO + c * kNH,
                       desc_sw128_mn(kv0 + 2 * c * kSlabBytes + kk * 2048, kSlabBytes, 1024),
                       desc_sw128_mn(p0 + kk * 2048, 1024, 1024), kIdPV, kk > 0 ? 1u : 0u);
          mma_commit(&bar->o_full);
        }
        __syncwarp();
        mbar_wait(&bar->o_full, 0, err, false);  // drain before TMEM is released
      }
    } else {
      mbar_wait(&bar->q_full, 0, err, false);
    }
  } else if (warp < 8) {
    // ------------------------- softmax and epilogue --------------------------------
    const int quad = warp & 3, hh = warp >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const float qscale = scale * kLog2e;
    uint32_t gphase = 0;
    bool ok = mbar_wait(&bar->s_full, 0, err);
    float m_h = kNegInf, psum[32];
    if (ok) {
      tc_fence_after();
      const bool valid = tile * kTE + row < N;
      uint32_t r[32];
      tmem_ld32(lane_base + kColS + hh * 32, r);
      tmem_ld_wait();
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = valid ? __uint_as_float(r[i]) * qscale : kNegInf;
      float* rmax = red + (hh * 4) * 32;
      rmax[quad * 32 + lane] = transpose_reduce<true>(v);
      ok = group_sync(&bar->grp[hh], gphase, err);
      if (ok) {
        m_h = fmaxf(fmaxf(rmax[lane], rmax[32 + lane]), fmaxf(rmax[64 + lane], rmax[96 + lane]));
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float ma = __shfl_sync(0xffffffffu, m_h, i), mb = __shfl_sync(0xffffffffu, m_h, i + 1);
          ma = ma == kNegInf ? 0.f : ma;
          mb = mb == kNegInf ? 0.f : mb;
          const float la = valid ? __uint_as_float(r[i]) * qscale : kNegInf;
          const float lb = valid ? __uint_as_float(r[i + 1]) * qscale : kNegInf;
          const float pa = ex2(la - ma), pb = ex2(lb - mb);
          psum[i] = pa;
          psum[i + 1] = pb;
          pk[i >> 1] = pack_bf16x2(pa, pb);
        }
        uint8_t* prow = sP + row * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(prow + (((hh * 4 + j) ^ (row & 7)) * 16)) =
              make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        fence_proxy_async();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->p_full);
      }
    }
    if (ok) ok = mbar_wait(&bar->o_full, 0, err);
    if (ok) {
      tc_fence_after();
      float* rsum = red + (2 * 4 + hh * 4) * 32;
      rsum[quad * 32 + lane] = transpose_reduce<false>(psum);
      ok = group_sync(&bar->grp[hh], gphase, err);
      if (ok) {
        const int h = hh * 32 + lane;
        const float tot = rsum[lane] + rsum[32 + lane] + rsum[64 + lane] + rsum[96 + lane];
        float inv = 1.f;
        if (direct) {
          const float mref = m_h == kNegInf ? 0.f : m_h;
          const float z = sink != nullptr ? sink[h] * kLog2e : kNegInf;
          inv = 1.f / (tot + (z == kNegInf ? 0.f : ex2(z - mref)));
        } else if (quad == 0) {
          part_ms[(pbase + h) * 2 + 0] = m_h;
          part_ms[(pbase + h) * 2 + 1] = tot;
        }
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColO + c * kNH + hh * 32, o);
          tmem_ld_wait();
          const int d = c * 128 + row;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int hd = hh * 32 + i;
            if (direct)
              out[(b * kNH + hd) * kC + d] =
                  __float2bfloat16_rn(__uint_as_float(o[i]) * __shfl_sync(0xffffffffu, inv, i));
            else
              part_o[(pbase + hd) * kC + d] = __uint_as_float(o[i]);
          }
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merges the tiles of each sequence: o = sum_i 2^(m_i - M) O_i /
// (sum_i 2^(m_i - M) l_i + 2^(sink - M)).  One CTA per (sequence, head).
__global__ void __launch_bounds__(128) decode_combine_kernel(
    const float* __restrict__ part_o, const float* __restrict__ part_ms,
    const float* __restrict__ sink, int ntile, __nv_bfloat16* __restrict__ out) {
  const int64_t b = blockIdx.y;
  const int h = blockIdx.x;
  const float z = sink != nullptr ? sink[h] * kLog2e : kNegInf;
  float M = z;
  for (int i = 0; i < ntile; ++i) M = fmaxf(M, part_ms[((b * ntile + i) * kNH + h) * 2]);
  float den = z == kNegInf ? 0.f : ex2(z - M);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const int d0 = threadIdx.x * 4;
  for (int i = 0; i < ntile; ++i) {
    const int64_t base = (b * ntile + i) * kNH + h;
    const float mi = part_ms[base * 2];
    if (mi == kNegInf) continue;
    const float wgt = ex2(mi - M);
    den = fmaf(wgt, part_ms[base * 2 + 1], den);
    const float4 o = *reinterpret_cast<const float4*>(part_o + base * kC + d0);
    acc[0] = fmaf(wgt, o.x, acc[0]);
    acc[1] = fmaf(wgt, o.y, acc[1]);
    acc[2] = fmaf(wgt, o.z, acc[2]);
    acc[3] = fmaf(wgt, o.w, acc[3]);
  }
  const float inv = 1.f / den;
  __nv_bfloat16* o = out + (b * kNH + h) * kC + d0;
  *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv),
                                            pack_bf16x2(acc[2] * inv, acc[3] * inv));
}

}  // namespace

bool decode_attn_tc_supported(const csa_cache_desc& d) {
  return d.nh == kNH && d.c == kC && (d.is_hca || d.k <= kMaxSelDec) && d.rope_dims % 8 == 0;
}

int decode_attn_splits(const csa_cache_desc& d) {
  const int64_t slots = (d.is_hca ? d.capacity : (int64_t)d.k) + d.window;
  return (int)((slots + kTE - 1) / kTE);
}

cudaError_t launch_decode_attn_tc(const csa_cache_desc& d, const CacheView& cv,
                                  const int64_t* pos, const void* q, const int32_t* sel,
                                  const float* sink, float scale, int ntile, void* out,
                                  float* part_o, float* part_ms, unsigned int* err,
                                  cudaStream_t s) {
  CUtensorMap tq;
  if (!make_tmap_bf16_3d(&tq, q, kC, kNH, d.batch, kC * 2ull, (uint64_t)kNH * kC * 2, 64, kNH))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(decode_attn_tile_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  decode_attn_tile_kernel<<<dim3((unsigned)ntile, (unsigned)d.batch), kThreads, SMEM, s>>>(
      tq, cv, pos, d.is_hca ? nullptr : sel, d.k, d.window, d.m, d.capacity, d.rope_dims, sink,
      scale, ntile, part_o, part_ms, (__nv_bfloat16*)out, err);
  if ((e = cudaGetLastError()) != cudaSuccess || ntile == 1) return e;
  decode_combine_kernel<<<dim3(kNH, (unsigned)d.batch), kC / 4, 0, s>>>(part_o, part_ms, sink,
                                                                        ntile,
                                                                        (__nv_bfloat16*)out);
  return cudaGetLastError();
}

}  // namespace csa
