// Core attention on the tcgen05 tensor cores: shared-KV MQA over a per-query
// entry set with the attention sink in the softmax denominator (bf16 in/out,
// fp32 accumulation), for 64 query heads of dim 512.
//
// E_t is (CSA) the selected compressed entries idx[t, :] with 0 <= s < V(t)
// or (HCA) every visible compressed entry, followed by the raw window rows
// max(0, t-W+1) .. t; each entry is both key and value, and
//   o_h = sum_j exp(l_hj) e_j / (exp(sink_h) + sum_j exp(l_hj)),
// l_hj = scale q_h . e_j  (sections 4.3 and 4.5 of "DeepSeek-V4: million-token
// context"; B9 of the "Core formulas chapter"; one softmax shared by the
// window, the compressed entries and the sink).
//
// Heads on TMEM lanes, 64 rows (M = 64): the 64 heads of one query take the
// M side of both products and the N side is as wide as the operands allow:
//   S[h, e]  = Q[h, :] . K[e, :]           M = 64 heads, N = 128 entries
//   O[h, d] += sum_e P[h, e] V[e, d]        M = 64 heads, N = 256 dims (x2)
// -- 48 MMAs per 128-entry tile.  An M = 64 operand or accumulator fills 16
// lanes of each TMEM lane quarter.  The low 16 lanes hold the query itself
// (the A operand of Q.K, read from tensor memory: 512 bf16 = 256 columns)
// and the two 128-column S buffers; the high 16 lanes hold O (512 columns).
// One warp per quarter owns the scores and the output of its 16 heads, two
// threads per head; the softmax is per thread with one partner shuffle; the
// running max moves (and the head's O row is rescaled in TMEM) only when a
// tile's max exceeds it by 2^8.
//
// With the query out of shared memory, the entry tiles (128 entries x 512
// dims, stored once as eight 64-dim 128-byte-swizzled slabs: the K-major B
// operand of Q.K and the MN-major B operand (V) of P.V) live in a ring of
// three 64 KB groups of four slabs; tile g takes groups 2g and 2g + 1 (mod 3).
// The MMA warp issues Q.K(g) over its first group, then P.V(g - 1) (whose
// first half frees the group that Q.K(g) needs next), then Q.K(g) over its
// second group: the gather and the first half of Q.K of the next tile run
// while the softmax of this one does.  Persistent CTAs (one per SM) walk the
// queries.
//
// Query boundaries are kept off the tensor pipe's path: the next query's
// selection row is bulk-copied into shared memory while this one runs; the
// query reaches tensor memory in two halves (dims 0-255, then 256-511), each
// written as soon as the previous query's Q.K half that read it is done, from
// registers loaded at the top of the query; the last P.V of a query is issued
// before anything of the next query is awaited; and the epilogue passes each
// warp's rows through the idle P buffer so that its global stores are whole
// 256-byte row pieces.
//
// Every wait is bounded (including the warp-group exchanges, which use
// mbarriers rather than named barriers), so a fault upstream ends the kernel
// with the timeout flag set instead of a hang.  Warp roles: warps 0-3
// softmax + epilogue; warps 4-10 gather (cp.async, zero-filled past the end
// of E_t; they also compact the query's valid selected indices), and warps
// 4-7 write each query into tensor memory; warp 11 issues the MMAs.
#include "common.cuh"
#include "launch.h"
#include "rope.cuh"
#include "sm100.cuh"
#include "tc_attn_util.cuh"

#include <algorithm>

namespace csa {

namespace {

constexpr int kNH = 64;                  // query heads (MMA M)
constexpr int kC = 512;                  // entry dim
constexpr int kTE = 128;                 // entries per tile (QK N)
constexpr int kSlabs = kC / 64;          // 64-dim slabs
constexpr int kSlabBytes = kTE * 128;    // 16 KB
constexpr int kGroupBytes = 4 * kSlabBytes;  // 64 KB: half a tile
constexpr int kGroups = 3;               // the ring
static_assert(kSlabs == 8, "a tile is two groups of four slabs");
constexpr int kPSlabBytes = kNH * 128;   // 8 KB: 64 heads x 64 entries
constexpr int kSoftWarps = 4, kProdWarps = 7;
constexpr int kProdThreads = kProdWarps * 32;
constexpr int kMmaWarp = kSoftWarps + kProdWarps;
constexpr int kThreads = (kMmaWarp + 1) * 32;  // 384
constexpr int kRowsPerPass = kProdThreads / 8;  // 28 rows x 8 16-byte chunks per pass
constexpr int kPasses = (kTE + kRowsPerPass - 1) / kRowsPerPass;  // 5
constexpr int kMaxSel = 2048;                  // selected entries per query
constexpr int kMeta = 4;                       // queries in flight between the roles
constexpr float kRescaleLog2 = 8.f;            // move the running max only past 2^8

constexpr uint32_t kColQ = 256;         // Q: the low 16 lanes, columns 256-511
constexpr uint32_t kColS = 0;           // S buffers: the low 16 lanes, columns 0 and 128
constexpr uint32_t kLaneO = 16u << 16;  // O: the high 16 lanes, columns 0-511

struct __align__(16) AttnMeta {
  int ntiles, nrows;
  int64_t t, b;
};

struct __align__(8) AttnBars {
  uint64_t grp_full[kGroups];  // a group's four slabs are stored
  uint64_t grp_free[kGroups];  // the P.V half that reads a group is done
  uint64_t s_full[2], s_empty[2], p_full, p_free, o_empty, meta_full[kMeta];
  // the query's dims 0-255 (lo) and 256-511 (hi) in tensor memory: written /
  // no longer read by the Q.K halves
  uint64_t q_full_lo, q_full_hi, q_empty_lo, q_empty_hi;
  uint64_t idx_full;  // the next query's selection row is in shared memory
  uint64_t drain;
  uint64_t grp_prod;  // bounded group barrier of the producer warps (one arrive per warp)
  uint64_t qinv_full[kMeta];  // (query norm) the query's per-head 1/RMS is in qinv
  uint32_t tmem_base;
};

constexpr int OFF_KV = 0;
constexpr int OFF_P = OFF_KV + kGroups * kGroupBytes;      // 196608
constexpr int OFF_LIST = OFF_P + 2 * kPSlabBytes;           // 212992
constexpr int OFF_IDXN = OFF_LIST + kMaxSel * 4;             // the next query's row
constexpr int OFF_META = OFF_IDXN + kMaxSel * 4;
constexpr int OFF_SCAN = OFF_META + kMeta * (int)sizeof(AttnMeta);
constexpr int OFF_QINV = OFF_SCAN + 64;                       // [kMeta][64] fp32
constexpr int OFF_BAR = OFF_QINV + kMeta * kNH * 4;
constexpr int SMEM = OFF_BAR + (int)sizeof(AttnBars) + 1024;
static_assert(SMEM <= 232448, "shared memory budget");

// One 128-dim round of a query row for tensor memory: the 64 dims of this
// thread's half, two per 32-bit column.
__device__ __forceinline__ void load_q_round(const uint4* src, uint32_t (&r)[32]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint4 v = __ldcs(src + j);
    r[4 * j] = v.x;
    r[4 * j + 1] = v.y;
    r[4 * j + 2] = v.z;
    r[4 * j + 3] = v.w;
  }
}

// Query norm: a 64-dim round r (dims d0 .. d0 + 63, two per word) multiplied
// by gamma, its raw squares added to ss.  The 1/RMS factor itself is applied
// to the logits (it is one scalar per head).
__device__ __forceinline__ void q_round_gamma(uint32_t (&r)[32], int d0,
                                              const float* __restrict__ gamma, float& ss) {
#pragma unroll
  for (int w = 0; w < 32; w += 2) {
    const float4 g = __ldg(reinterpret_cast<const float4*>(gamma + d0 + 2 * w));
    const float x0 = __uint_as_float(r[w] << 16), x1 = __uint_as_float(r[w] & 0xffff0000u);
    const float x2 = __uint_as_float(r[w + 1] << 16), x3 = __uint_as_float(r[w + 1] & 0xffff0000u);
    ss = fmaf(x0, x0, fmaf(x1, x1, fmaf(x2, x2, fmaf(x3, x3, ss))));
    r[w] = pack_bf16x2(x0 * g.x, x1 * g.y);
    r[w + 1] = pack_bf16x2(x2 * g.z, x3 * g.w);
  }
}

// The last round's pairs that lie in the trailing rope_dims dims (word p =
// pair p of dims 448 .. 511), turned by the angles of pairs p - (64 - R) / 2
// whose cosine and sine lane j of the warp holds for pair j.  Every lane of
// the warp calls it (the shuffles); only `mine` lanes change their words.
__device__ __forceinline__ void q_round_rope(uint32_t (&r)[32], bool mine, int rope_dims,
                                             float cs_lane, float sn_lane) {
  const int p0 = 32 - rope_dims / 2;
#pragma unroll
  for (int p = 0; p < 32; ++p) {
    const float cs = __shfl_sync(0xffffffffu, cs_lane, p >= p0 ? p - p0 : 0);
    const float sn = __shfl_sync(0xffffffffu, sn_lane, p >= p0 ? p - p0 : 0);
    if (mine && p >= p0) {
      float x = __uint_as_float(r[p] << 16), y = __uint_as_float(r[p] & 0xffff0000u);
      rope_turn(x, y, cs, sn);
      r[p] = pack_bf16x2(x, y);
    }
  }
}

// kQNorm: the query RMSNorm + rotation in the prologue and the output
// rotation in the epilogue (a separate instantiation, so that the plain
// kernel carries none of its registers).
template <bool kQNorm>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kv_comp,
    const int32_t* __restrict__ idx, int k, const __nv_bfloat16* __restrict__ kv_win,
    int window, const float* __restrict__ sink, float scale, int64_t n, int m, int64_t E,
    int64_t total, QNormRope qn, __nv_bfloat16* __restrict__ out, unsigned int* __restrict__ err) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sKV = smem + OFF_KV;
  uint8_t* sP = smem + OFF_P;
  int32_t* list = reinterpret_cast<int32_t*>(smem + OFF_LIST);
  int32_t* idxn = reinterpret_cast<int32_t*>(smem + OFF_IDXN);
  AttnMeta* meta = reinterpret_cast<AttnMeta*>(smem + OFF_META);
  int* pscan = reinterpret_cast<int*>(smem + OFF_SCAN);
  float* qinv = reinterpret_cast<float*>(smem + OFF_QINV);
  AttnBars* bar = reinterpret_cast<AttnBars*>(smem + OFF_BAR);
  constexpr bool qnorm = kQNorm;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if ((int64_t)blockIdx.x >= total) return;
  if (flag_value(err) != 0) return;

  if (threadIdx.x == 0) {
    for (int u = 0; u < kGroups; ++u) {
      mbar_init(&bar->grp_full[u], kProdThreads);
      mbar_init(&bar->grp_free[u], 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&bar->s_full[u], 1);
      mbar_init(&bar->s_empty[u], kSoftWarps);
    }
    for (int u = 0; u < kMeta; ++u) {
      mbar_init(&bar->meta_full[u], 1);
      mbar_init(&bar->qinv_full[u], 4);  // the four warps that write the query
    }
    mbar_init(&bar->p_full, kSoftWarps);
    mbar_init(&bar->p_free, 1);
    mbar_init(&bar->q_full_lo, 4);  // the four warps that write the query
    mbar_init(&bar->q_full_hi, 4);
    mbar_init(&bar->q_empty_lo, 1);
    mbar_init(&bar->q_empty_hi, 1);
    mbar_init(&bar->idx_full, 1);
    mbar_init(&bar->o_empty, kSoftWarps);
    mbar_init(&bar->drain, 1);
    mbar_init(&bar->grp_prod, kProdWarps);
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

  if (warp >= kSoftWarps && warp < kMmaWarp) {
    // ======================= gather producer (224 threads) =====================
    const int ptid = threadIdx.x - kSoftWarps * 32;
    const int pw = ptid >> 5;
    const int chunk = ptid & 7;
    int g = 0;
    uint32_t gphase = 0;
    bool ok = true;
    // the entries and window rows are re-read by many queries: keep them in L2
    const uint64_t pol_kv = l2_policy_evict_last();
    // the selection rows move into shared memory one query ahead (one bulk
    // copy) when they are whole 16-byte units; otherwise they are read in place
    const bool stage = idx != nullptr && k > 0 && (k & 3) == 0 &&
                       (reinterpret_cast<uintptr_t>(idx) & 15) == 0;
    int idx_issued = 0;  // bulk copies issued (thread 0) / consumed
    auto stage_row = [&](int64_t qn) {
      fence_proxy_async();
      mbar_arrive_expect_tx(&bar->idx_full, (uint32_t)k * 4u);
      bulk_load(idxn, idx + qn * k, (uint32_t)k * 4u, &bar->idx_full);
      ++idx_issued;
    };
    if (stage && ptid == 0) stage_row(blockIdx.x);
    for (int64_t kq = 0; ok; ++kq) {
      const int64_t qi = blockIdx.x + kq * gridDim.x;
      if (qi >= total) break;
      const int64_t b = qi / n, t = qi % n;
      const int64_t V = min((t + 1) / m, E);
      const int64_t w0 = max((int64_t)0, t - window + 1);
      const int nwin = (int)(t - w0 + 1);
      // the next query of this CTA (64 KB, contiguous) starts moving into L2
      if (ptid == 0 && qi + gridDim.x < total)
        bulk_prefetch_l2(q + (qi + gridDim.x) * (kNH * kC), kNH * kC * 2);
      // warps 0-3: the first two of the four 128-dim rounds of this query
      // (thread (r, half): head 16 pw + r, the 64 dims 128 c + 64 half ..) start
      // loading now, under the list compaction and the first half-tile's
      // gather (read once: evict first)
      const uint4* qsrc = reinterpret_cast<const uint4*>(
          q + ((b * n + t) * kNH + pw * 16 + (lane & 15)) * kC + 64 * (lane >> 4));
      uint32_t ra[32], rb[32];
      if (pw < 4) {
        load_q_round(qsrc, ra);
        load_q_round(qsrc + 16, rb);
      }
      // the previous query's list is no longer read
      if (!group_sync(&bar->grp_prod, gphase, err)) break;
      int nsel;
      if (idx != nullptr) {
        // compact the valid selections, keeping their order
        const int per = (k + kProdThreads - 1) / kProdThreads;
        const int lo = min(k, ptid * per), hi = min(k, lo + per);
        const int32_t* row = idx + (b * n + t) * k;
        if (stage) {
          if (!mbar_wait(&bar->idx_full, (uint32_t)(kq & 1), err)) break;
          row = idxn;
        }
        int cnt = 0;
        for (int j = lo; j < hi; ++j) {
          const int s = row[j];
          cnt += (s >= 0 && s < V) ? 1 : 0;
        }
        int inc = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, inc, off);
          if (lane >= off) inc += v;
        }
        if (lane == 31) pscan[pw] = inc;
        if (!group_sync(&bar->grp_prod, gphase, err)) break;
        int base = 0;
        nsel = 0;
        for (int w = 0; w < kProdWarps; ++w) {
          if (w < pw) base += pscan[w];
          nsel += pscan[w];
        }
        int pos = base + inc - cnt;
        for (int j = lo; j < hi; ++j) {
          const int s = row[j];
          if (s >= 0 && s < V) list[pos++] = s;
        }
        if (!group_sync(&bar->grp_prod, gphase, err)) break;
        // every thread is done with the staged row: the next query's comes in
        if (stage && ptid == 0 && qi + gridDim.x < total) stage_row(qi + gridDim.x);
      } else {
        nsel = (int)V;
      }
      const int N = nsel + nwin;
      const int T = (N + kTE - 1) / kTE;
      if (ptid == 0) {
        AttnMeta& mt = meta[kq % kMeta];
        mt.ntiles = T;
        mt.nrows = N;
        mt.t = t;
        mt.b = b;
        mbar_arrive(&bar->meta_full[kq % kMeta]);
      }
      // ---- the query into tensor memory, warps pw < 4 (lanes 32 pw + r; each
      // 32-bit column two consecutive dims): dims 0-255 once the first
      // half-tile's gather is under way and the old query's first Q.K half is
      // done (rounds 2-3 then load), dims 256-511 after the second half-tile ----
      const uint32_t qaddr = tmem + ((uint32_t)(pw * 32) << 16) + kColQ;
      // (query norm) this thread's dims of rounds 0-1 start at 64 half, of
      // rounds 2-3 at 256 + 64 half; raw squares summed over all four rounds
      const int qhalf = lane >> 4;
      float qss = 0.f;
      auto write_q_lo = [&]() -> bool {
        if (qnorm) {
          q_round_gamma(ra, 64 * qhalf, qn.gamma, qss);
          q_round_gamma(rb, 128 + 64 * qhalf, qn.gamma, qss);
        }
        if (kq >= 1 && !mbar_wait(&bar->q_empty_lo, (uint32_t)((kq - 1) & 1), err)) return false;
        tc_fence_after();
        tmem_st16x64(qaddr, ra);
        tmem_st16x64(qaddr + 64, rb);
        load_q_round(qsrc + 32, ra);
        load_q_round(qsrc + 48, rb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->q_full_lo);
        return true;
      };
      auto write_q_hi = [&]() -> bool {
        if (qnorm) {
          q_round_gamma(ra, 256 + 64 * qhalf, qn.gamma, qss);
          q_round_gamma(rb, 384 + 64 * qhalf, qn.gamma, qss);
          if (qn.rope_dims > 0) {  // dims 448 .. 511 sit in round 3 of the upper half
            float cs = 1.f, sn = 0.f;
            if (lane < qn.rope_dims / 2) rope_cos_sin(t, lane, qn.rope_dims, qn.base, cs, sn);
            q_round_rope(rb, qhalf == 1, qn.rope_dims, cs, sn);
          }
          const float tot = qss + __shfl_xor_sync(0xffffffffu, qss, 16);
          if (lane < 16) qinv[(kq % kMeta) * kNH + pw * 16 + lane] = 1.f / sqrtf(tot / kC + qn.eps);
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar->qinv_full[kq % kMeta]);
        }
        if (kq >= 1 && !mbar_wait(&bar->q_empty_hi, (uint32_t)((kq - 1) & 1), err)) return false;
        tc_fence_after();
        tmem_st16x64(qaddr + 128, ra);
        tmem_st16x64(qaddr + 192, rb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->q_full_hi);
        return true;
      };
      for (int tt = 0; tt < T && ok; ++tt, ++g) {
        for (int h = 0; h < 2 && ok; ++h) {
          // this thread's rows of the tile: global row pointers (nullptr = zero fill)
          const __nv_bfloat16* src[kPasses];
#pragma unroll
          for (int rr = 0; rr < kPasses; ++rr) {
            const int slot = tt * kTE + (ptid >> 3) + kRowsPerPass * rr;
            const __nv_bfloat16* p = nullptr;
            if (slot < nsel) {
              const int64_t e = idx != nullptr ? (int64_t)list[slot] : (int64_t)slot;
              p = kv_comp + (b * E + e) * kC;
            } else if (slot < N) {
              p = kv_win + (b * n + w0 + (slot - nsel)) * kC;
            }
            src[rr] = p;
          }
          // half h of tile g: group u = 2 g + h of the ring, free once the P.V
          // half that read it three groups ago is done
          const int u = 2 * g + h, gp = u % kGroups;
          if (u >= kGroups &&
              !mbar_wait(&bar->grp_free[gp], (uint32_t)(((u / kGroups) - 1) & 1), err)) {
            ok = false;
            break;
          }
          uint8_t* dst0 = sKV + gp * kGroupBytes;
          for (int j = 0; j < 4; ++j) {
            const int s = 4 * h + j;
            uint8_t* dst = dst0 + j * kSlabBytes;
#pragma unroll
            for (int rr = 0; rr < kPasses; ++rr) {
              const int row = (ptid >> 3) + kRowsPerPass * rr;
              if (row >= kTE) continue;
              const __nv_bfloat16* p = src[rr] != nullptr ? src[rr] + s * 64 + chunk * 8 : kv_win;
              cp_async_16_hint(dst + row * 128 + ((chunk ^ (row & 7)) * 16), p,
                               src[rr] != nullptr ? 16u : 0u, pol_kv);
            }
          }
          cp_async_arrive_noinc(&bar->grp_full[gp]);
          if (tt == 0 && pw < 4 && !(h == 0 ? write_q_lo() : write_q_hi())) {
            ok = false;
            break;
          }
        }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    // a staged row that an early exit left unread has landed before the exit
    if (ptid == 0 && idx_issued > 0)
      mbar_wait(&bar->idx_full, (uint32_t)((idx_issued - 1) & 1), err, false);
  } else if (warp == kMmaWarp) {
    // ======================= MMA issuer (one lane) =============================
    constexpr uint32_t kIdQK = idesc_bf16(kNH, kTE, 0, 0);   // Q K-major, K K-major
    constexpr uint32_t kIdPV = idesc_bf16(kNH, 256, 0, 1);   // P K-major, V MN-major
    const uint32_t kv0 = smem_u32(sKV), p0 = smem_u32(sP);
    int g = 0;
    bool ok = true;
    // the tile whose P.V is still to be issued: index, first of its query, query
    int pend = -1;
    bool pend_first = false;
    int64_t pend_kq = 0;
    auto issue_pv = [&]() -> bool {
      if (!mbar_wait(&bar->p_full, (uint32_t)(pend & 1), err)) return false;
      // the first P.V of a query overwrites O: the previous epilogue has read it
      if (pend_first && pend_kq >= 1 &&
          !mbar_wait(&bar->o_empty, (uint32_t)((pend_kq - 1) & 1), err))
        return false;
      tc_fence_after();
      if (lane == 0) {
        for (int hf = 0; hf < 2; ++hf) {  // dims 256 hf .. 256 hf + 255: group 2 pend + hf
          const int gp = (2 * pend + hf) % kGroups;
#pragma unroll
          for (int kk = 0; kk < kTE / 16; ++kk)
            mma_bf16(tmem + kLaneO + hf * 256,
                     desc_sw128(p0 + (kk >> 2) * kPSlabBytes + (kk & 3) * 32),
                     desc_sw128_mn(kv0 + gp * kGroupBytes + kk * 2048, kSlabBytes, 1024),
                     kIdPV, (pend_first && kk == 0) ? 0u : 1u);
          mma_commit(&bar->grp_free[gp]);
        }
        mma_commit(&bar->p_free);
      }
      __syncwarp();
      pend = -1;
      return true;
    };
    // Q.K over group u (slabs 4 h .. 4 h + 3 of tile g, h = u - 2 g)
    auto issue_qk_half = [&](int h, int sb) -> bool {
      const int u = 2 * g + h, gp = u % kGroups;
      if (!mbar_wait(&bar->grp_full[gp], (uint32_t)((u / kGroups) & 1), err)) return false;
      fence_proxy_async();
      tc_fence_after();
      if (lane == 0) {
        for (int j = 0; j < 4; ++j) {
          const int s = 4 * h + j;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // 16 dims = 8 columns of the query per step
            mma_bf16_ts(tmem + kColS + sb * kTE, tmem + kColQ + s * 32 + kk * 8,
                        desc_sw128(kv0 + gp * kGroupBytes + j * kSlabBytes + kk * 32), kIdQK,
                        (s | kk) != 0 ? 1u : 0u);
        }
      }
      __syncwarp();
      return true;
    };
    for (int64_t kq = 0; ok; ++kq) {
      const int64_t qi = blockIdx.x + kq * gridDim.x;
      if (qi >= total) break;
      // the previous query's last P.V first: neither its epilogue nor the ring
      // waits for this query's list
      if (pend >= 0 && !issue_pv()) break;
      if (!mbar_wait(&bar->meta_full[kq % kMeta], (uint32_t)((kq / kMeta) & 1), err)) break;
      const int T = meta[kq % kMeta].ntiles;
      if (!mbar_wait(&bar->q_full_lo, (uint32_t)(kq & 1), err)) break;
      tc_fence_after();
      for (int tt = 0; tt < T; ++tt, ++g) {
        const int sb = g & 1;
        // S buffer sb is free once the softmax has read it (tile g - 2)
        if (g >= 2 && !mbar_wait(&bar->s_empty[sb], (uint32_t)(((g >> 1) - 1) & 1), err)) {
          ok = false;
          break;
        }
        if (!(ok = issue_qk_half(0, sb))) break;
        if (tt == T - 1 && lane == 0) mma_commit(&bar->q_empty_lo);
        // P.V of the previous tile: its first half frees the group of this
        // tile's second half
        if (pend >= 0 && !(ok = issue_pv())) break;
        if (tt == 0) {
          if (!(ok = mbar_wait(&bar->q_full_hi, (uint32_t)(kq & 1), err))) break;
          tc_fence_after();
        }
        if (!(ok = issue_qk_half(1, sb))) break;
        if (lane == 0) {
          mma_commit(&bar->s_full[sb]);
          if (tt == T - 1) mma_commit(&bar->q_empty_hi);
        }
        __syncwarp();
        pend = g;
        pend_first = tt == 0;
        pend_kq = kq;
      }
    }
    if (ok && pend >= 0) issue_pv();
    if (lane == 0) mma_commit(&bar->drain);
    __syncwarp();
    mbar_wait(&bar->drain, 0, err, false);
  } else {
    // ======================= softmax + epilogue (4 warps) ======================
    // warp q: TMEM lane quarter q = heads 16 q .. 16 q + 15; thread (hl, ch):
    // head 16 q + hl, columns 32 ch .. 32 ch + 31 of every 64-column load
    const int hl = lane & 15, ch = lane >> 4;
    const int hd = warp * 16 + hl;
    const uint32_t o_lane = tmem + ((uint32_t)(warp * 32) << 16) + kLaneO;
    const uint32_t s_lane = tmem + ((uint32_t)(warp * 32) << 16) + kColS;
    const float qscale = scale * kLog2e;
    // the sink of head hd (log2 units), the same for every query
    const float z = sink != nullptr ? sink[hd] * kLog2e : kNegInf;
    int g = 0;
    for (int64_t kq = 0;; ++kq) {
      const int64_t qi = blockIdx.x + kq * gridDim.x;
      if (qi >= total) break;
      if (!mbar_wait(&bar->meta_full[kq % kMeta], (uint32_t)((kq / kMeta) & 1), err)) break;
      const AttnMeta mt = meta[kq % kMeta];
      // (query norm) this head's 1/RMS scales its logits
      float qscale_h = qscale;
      if (qnorm) {
        if (!mbar_wait(&bar->qinv_full[kq % kMeta], (uint32_t)((kq / kMeta) & 1), err)) break;
        qscale_h = qscale * qinv[(kq % kMeta) * kNH + hd];
      }
      float m_run = kNegInf;  // running max (log2 units) of head hd
      float l_run = 0.f;      // this thread's share of the head's sum
      bool ok = true;
      for (int tt = 0; tt < mt.ntiles; ++tt, ++g) {
        const int sb = g & 1;
        if (!mbar_wait(&bar->s_full[sb], (uint32_t)((g >> 1) & 1), err)) { ok = false; break; }
        tc_fence_after();
        float lg[64];  // logits of columns 64 c + 32 ch + i, c = 0, 1
        {
          uint32_t r[32];
          const int nv = mt.nrows - tt * kTE;  // valid columns of this tile
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            tmem_ld16x64(s_lane + sb * kTE + c * 64, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              lg[c * 32 + i] = 64 * c + 32 * ch + i < nv ? __uint_as_float(r[i]) * qscale_h : kNegInf;
          }
        }
        // the S buffer is free for the Q.K of tile g + 2
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->s_empty[sb]);
        float mx = kNegInf;
#pragma unroll
        for (int i = 0; i < 64; ++i) mx = fmaxf(mx, lg[i]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));  // the head's other half
        float f = 1.f;
        bool resc = false;
        if (tt == 0) {
          m_run = mx;
        } else if (mx > m_run + kRescaleLog2) {
          resc = true;
          f = ex2(m_run - mx);
          m_run = mx;
        }
        // P (and, for a rescale, O) is free once the previous P.V is done
        if (g >= 1 && !mbar_wait(&bar->p_free, (uint32_t)((g - 1) & 1), err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
          l_run *= f;
          for (int c = 0; c < kC / 64; ++c) {
            uint32_t o[32];
            tmem_ld16x64(o_lane + c * 64, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st16x64(o_lane + c * 64, o);
          }
          tmem_st_wait();
        }
        const float mref = m_run == kNegInf ? 0.f : m_run;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float pa = ex2(lg[c * 32 + i] - mref), pb = ex2(lg[c * 32 + i + 1] - mref);
            l_run += pa + pb;
            pk[i >> 1] = pack_bf16x2(pa, pb);
          }
          uint8_t* prow = sP + c * kPSlabBytes + hd * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(prow + (((4 * ch + j) ^ (hd & 7)) * 16)) =
                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->p_full);
      }
      if (!ok) break;
      // ---- epilogue: o = O / (sum_j p_j + 2^(sink - m)) -------------------------
      // O is complete once the P.V of the query's last tile (g - 1) is done
      if (!mbar_wait(&bar->p_free, (uint32_t)((g - 1) & 1), err)) break;
      tc_fence_after();
      const float l = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
      const float mref = m_run == kNegInf ? 0.f : m_run;
      const float inv = 1.f / (l + (z == kNegInf ? 0.f : ex2(z - mref)));
      // 128 dims a pass: the warp's 16 head rows (256 bytes each) go through
      // its own 4 KB of the P buffer (free until the warp writes the next P),
      // 16-byte chunks XOR-swizzled by row, so that every global store writes
      // two whole 256-byte row pieces; thread (hl, ch) loads dims
      // 128 pp + 64 ch .. + 63 of head hl
      uint8_t* ebuf = sP + (hl >> 3) * kPSlabBytes + warp * 2048 + (hl & 7) * 256;
      __nv_bfloat16* ow = out + ((mt.b * n + mt.t) * kNH + warp * 16) * kC;
      // (query norm) the output's trailing dims turn back by position -t: lane j
      // holds the angle of pair j
      float ocs = 1.f, osn = 0.f;
      if (qnorm && qn.rope_dims > 0 && lane < qn.rope_dims / 2)
        rope_cos_sin(-mt.t, lane, qn.rope_dims, qn.base, ocs, osn);
#pragma unroll 1
      for (int pp = 0; pp < kC / 128; ++pp) {
        uint32_t o[64];
        tmem_ld16x128(o_lane + pp * 128, o);
        tmem_ld_wait();
        if (qnorm && qn.rope_dims > 0 && pp == kC / 128 - 1) {  // dims 448 .. 511: ch == 1
          const int p0 = 32 - qn.rope_dims / 2;
#pragma unroll
          for (int p = 0; p < 32; ++p) {
            const float cs = __shfl_sync(0xffffffffu, ocs, p >= p0 ? p - p0 : 0);
            const float sn = __shfl_sync(0xffffffffu, osn, p >= p0 ? p - p0 : 0);
            if (ch == 1 && p >= p0) {
              float x = __uint_as_float(o[2 * p]), y = __uint_as_float(o[2 * p + 1]);
              rope_turn(x, y, cs, sn);
              o[2 * p] = __float_as_uint(x);
              o[2 * p + 1] = __float_as_uint(y);
            }
          }
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          uint32_t pk[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(o[8 * jj + 2 * i]) * inv,
                                __uint_as_float(o[8 * jj + 2 * i + 1]) * inv);
          *reinterpret_cast<uint4*>(ebuf + (((8 * ch + jj) ^ (hl & 7)) * 16)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 2 * i + (lane >> 4), x = lane & 15;
          const uint4 v = *reinterpret_cast<const uint4*>(
              sP + (r >> 3) * kPSlabBytes + warp * 2048 + (r & 7) * 256 + ((x ^ (r & 7)) * 16));
          __stcs(reinterpret_cast<uint4*>(ow + r * kC + 128 * pp + 8 * x), v);
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->o_empty);
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

}  // namespace

bool attn_tc_supported(int nh, int c, int k, csa_dtype dt, const void* q, const void* kv_comp,
                       const void* kv_win, int rope_dims) {
  if (dt != CSA_BF16 || nh != kNH || c != kC || k > kMaxSel || rope_dims > 64) return false;
  return ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(kv_comp) |
           reinterpret_cast<uintptr_t>(kv_win)) & 15) == 0;
}

cudaError_t launch_attn_tc(const void* q, const void* kv_comp, const int32_t* idx, int k,
                           const void* kv_win, int window, const float* sink, float scale,
                           int64_t batch, int64_t n, int m, const QNormRope& qn, void* out,
                           unsigned int* err, cudaStream_t s) {
  auto kern = qn.gamma != nullptr ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  const int64_t total = batch * n;
  const int64_t grid = std::min<int64_t>(total, sm_count());
  kern<<<(unsigned)grid, kThreads, SMEM, s>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)kv_comp, idx, k,
      (const __nv_bfloat16*)kv_win, window, sink, scale, n, m, n / m, total, qn,
      (__nv_bfloat16*)out, err);
  return cudaGetLastError();
}

}  // namespace csa
