// Decode indexer on the tcgen05 tensor cores, FP8 x FP8, persistent.
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
// stream with the FP8 tiles fed to the tensor core as they arrive.  All
// sequences' 128-key tiles form one list, cut into equal contiguous ranges,
// one per CTA (one CTA per SM); each CTA keeps a single TMA ring of 16 KB
// tiles (128-byte swizzle) full across sequence boundaries, so the stream
// never drains between sequences.  One lane issues M = 128 keys x N = 2H x
// K = 128 kind::f8f6f4 MMAs straight from the ring: the B operand holds each
// query head twice, hi = E4M3(q/s_h) and lo = E4M3(q/s_h - hi) with s_h a
// power of two, which together reproduce the bf16 query (the append step
// builds this operand once per sequence; here one bulk copy per sequence
// brings it in, two operand slots each freed by the MMAs of its sequence's
// last tile, and the head weights w_h s_h into a 16-deep ring freed by the
// epilogue, which trails the MMAs by at most ten tiles, so no phase of its
// barriers can alias).  Two warpgroups of epilogue warps take alternate
// tiles (four accumulators in TMEM for H = 64), add the hi and lo halves and
// apply ReLU, the head weights and the key scale; scores go to a
// per-sequence fp32 array (L2-resident at these sizes) for the selection
// kernel.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kKeys = 128;               // keys per tile (MMA M)
constexpr int kCI = 128;                 // index-key dim = bytes per FP8 key
constexpr int kTileBytes = kKeys * kCI;  // 16 KB
constexpr int kThreads = 384;  // warp 0 TMA, 1 MMA, 2 operand copies, 4-7 / 8-11 epilogue
constexpr int kBSlots = 2;               // query operands (sequences) in flight
constexpr int kWSlots = 16;              // head-weight vectors (sequences) in flight
constexpr int kSmemLimit = 232448;
// Per-sequence histogram of the scores' order keys (their top 12 bits): the
// selection step reads it to find the bin holding the k-th largest score
// without another pass over the scores.  Two slots, since the two epilogue
// groups can be on neighbouring sequences at a boundary.
constexpr int kHistBins = 4096;
constexpr int kHistShift = 20;
constexpr int kHistBytes = 2 * kHistBins * 4;
constexpr int kEpiThreads = 256;  // warps 4-11

template <int S>
struct __align__(8) DecIdxBars {
  uint64_t full[S], empty[S], d_full[2], d_empty[2], b_full[kBSlots], b_empty[kBSlots], drain;
  uint64_t w_full[kWSlots], w_empty[kWSlots];
  uint32_t tmem_base;
  int j0, count;  // the CTA's first tile (within sequence b0) and its number of tiles
  int64_t b0;
  unsigned int abort;  // the timeout flag as read once for the whole CTA
};

// Tiles travel in groups of TPP ("pairs"): one ring stage, one TMEM
// accumulator set, and one commit each.  A tcgen05 commit or MMA costs the
// issuing thread about as much as a 128-key MMA of the tensor core, so
// committing once per two tiles is what keeps the MMA warp ahead of HBM.
template <int H>
struct DecIdxCfg {
  static constexpr int N = 2 * H;                  // hi and lo rows per head
  static constexpr int B_BYTES = N * 128;          // one query operand
  static constexpr int TPP = 512 / N / 2;          // tiles per pair: 2 (H = 64), 1 (H = 128)
  static constexpr int STAGE_BYTES = TPP * kTileBytes;
  static constexpr int STAGES =
      (kSmemLimit - 1024 - kBSlots * B_BYTES - kWSlots * H * 4 - kHistBytes - 768) / STAGE_BYTES;
  static constexpr int OFF_RAW = 0;
  static constexpr int OFF_B = OFF_RAW + STAGES * STAGE_BYTES;
  static constexpr int OFF_W = OFF_B + kBSlots * B_BYTES;
  static constexpr int OFF_HIST = OFF_W + kWSlots * H * 4;
  static constexpr int OFF_BAR = OFF_HIST + kHistBytes;
  static constexpr int SMEM = OFF_BAR + (int)sizeof(DecIdxBars<STAGES>) + 1024;
  static_assert(SMEM <= kSmemLimit, "shared memory budget");
  static_assert(TPP >= 1 && 2 * TPP * N <= 512, "two accumulator sets in TMEM");
};

// Adds histogram slot `slot` of this CTA into sequence b's global histogram
// and clears it.  Called by the 256 epilogue threads once every score of the
// sequence in this CTA's range has been counted (after a barrier over them).
__device__ __forceinline__ void flush_hist(uint32_t* hist, int slot, uint32_t* ghist, int64_t b,
                                           int etid) {
  uint32_t* hs = hist + slot * kHistBins;
  uint32_t* gh = ghist + b * kHistBins;
  for (int j = etid; j < kHistBins; j += kEpiThreads) {
    const uint32_t c = hs[j];
    if (c != 0u) {
      atomicAdd(gh + j, c);
      hs[j] = 0u;
    }
  }
}

__device__ __forceinline__ void hist_add(uint32_t* hist, int slot, float score) {
  atomicAdd(hist + slot * kHistBins + (order_key(score) >> kHistShift), 1u);
}

// Paged classical cache: entry s of sequence b in block btab[b][s >> shift]
// of the pool (btab == NULL: the contiguous [batch][capacity] form).  A key
// tile is then brought in as boxes of `box` rows, one per block piece.
struct PagedKeys {
  const int32_t* btab;
  int64_t stride, nblocks;
  int shift, box;
};

__device__ __forceinline__ int64_t paged_row(const PagedKeys& pk, int64_t b, int64_t s,
                                             int64_t cap) {
  if (pk.btab == nullptr) return b * cap + s;
  const int64_t blk = pk.btab[b * pk.stride + (s >> pk.shift)];
  if (blk < 0 || blk >= pk.nblocks) return -1;
  return (blk << pk.shift) + (s & ((int64_t(1) << pk.shift) - 1));
}

// Rows (or -1) of the boxes of keys s0 .. s0 + tk - 1 below V; returns the
// bytes the present ones bring.
__device__ __forceinline__ uint32_t paged_tile_rows(const PagedKeys& pk, int64_t b, int64_t s0,
                                                    int tk, int64_t V, int64_t cap,
                                                    int64_t (&rows)[8]) {
  uint32_t bytes = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    rows[q] = -1;
    const int64_t sq = s0 + (int64_t)q * pk.box;
    if (q * pk.box < tk && sq < V) rows[q] = paged_row(pk, b, sq, cap);
    if (rows[q] >= 0) bytes += (uint32_t)pk.box * 128u;
  }
  return bytes;
}

__device__ __forceinline__ void paged_tile_load(const CUtensorMap* tm, uint64_t* bar,
                                                uint8_t* dst, const PagedKeys& pk,
                                                const int64_t (&rows)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    if (rows[q] >= 0) sm100::tma_load_3d(dst + q * pk.box * 128, tm, bar, 0, (int)rows[q], 0);
}

// Tiles of tk keys of sequence b.
__device__ __forceinline__ int tiles_of(const int64_t* pos, int64_t b, int m, int64_t cap,
                                        int tk) {
  const int64_t t = pos[b];
  const int64_t V = t < 0 ? 0 : min((t + 1) / m, cap);
  return (int)((V + tk - 1) / tk);
}

// Walks the CTA's tiles in order: sequence b, tile j of nt.
struct TileWalk {
  int64_t b;
  int j, nt, tk;
  __device__ void start(const int64_t* pos, int64_t b0, int j0, int m, int64_t cap, int tk_) {
    tk = tk_;
    b = b0;
    j = j0;
    nt = tiles_of(pos, b0, m, cap, tk);
  }
  __device__ void next(const int64_t* pos, int64_t batch, int m, int64_t cap) {
    if (++j < nt) return;
    j = 0;
    do {
      ++b;
      nt = b < batch ? tiles_of(pos, b, m, cap, tk) : 1;
    } while (nt == 0);
  }
};

// Warp 0: this CTA's contiguous share [g0, g1) of the flattened tile list
// and the sequence / tile where it starts.
__device__ void locate_range(const int64_t* pos, int64_t batch, int m, int64_t cap, int tk,
                             int64_t& b0, int& j0, int& count) {
  const int lane = threadIdx.x & 31;
  int64_t total = 0;
  for (int64_t base = 0; base < batch; base += 32) {
    int64_t nt = base + lane < batch ? tiles_of(pos, base + lane, m, cap, tk) : 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) nt += __shfl_xor_sync(0xffffffffu, nt, off);
    total += nt;
  }
  const int64_t g0 = total * blockIdx.x / gridDim.x, g1 = total * (blockIdx.x + 1) / gridDim.x;
  count = (int)(g1 - g0);
  b0 = 0;
  j0 = 0;
  if (count == 0) return;
  int64_t run = 0;
  for (int64_t base = 0; base < batch; base += 32) {
    const int64_t nt = base + lane < batch ? tiles_of(pos, base + lane, m, cap, tk) : 0;
    int64_t inc = nt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int64_t v = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += v;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, run + inc > g0);
    if (hit != 0) {
      const int f = __ffs(hit) - 1;
      const int64_t before = __shfl_sync(0xffffffffu, run + inc - nt, f);
      b0 = base + f;
      j0 = (int)(g0 - before);
      return;
    }
    run += __shfl_sync(0xffffffffu, inc, 31);
  }
}

template <int H>
__global__ void __launch_bounds__(kThreads, 1) decode_index_tc_kernel(
    const __grid_constant__ CUtensorMap tm_keys, const float* __restrict__ key_scale,
    PagedKeys pk, const uint8_t* __restrict__ qop, const int64_t* __restrict__ pos, int64_t batch,
    int64_t cap, int m, float* __restrict__ scores, uint32_t* __restrict__ ghist,
    uint32_t* __restrict__ idx_done,
    unsigned int* __restrict__ err) {
  using C = DecIdxCfg<H>;
  constexpr int S = C::STAGES;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sRaw = smem + C::OFF_RAW;
  uint8_t* sB = smem + C::OFF_B;
  float* sW = reinterpret_cast<float*>(smem + C::OFF_W);
  uint32_t* sHist = reinterpret_cast<uint32_t*>(smem + C::OFF_HIST);
  DecIdxBars<S>* bar = reinterpret_cast<DecIdxBars<S>*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j = threadIdx.x; j < 2 * kHistBins; j += kThreads) sHist[j] = 0u;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < S; ++s) {
        mbar_init(&bar->full[s], 1);
        mbar_init(&bar->empty[s], 1);
      }
      for (int q = 0; q < 2; ++q) {
        mbar_init(&bar->d_full[q], 1);
        mbar_init(&bar->d_empty[q], 4 * C::TPP);  // every epilogue warp with a tile in the pair
      }
      for (int u = 0; u < kBSlots; ++u) {
        mbar_init(&bar->b_full[u], 1);
        mbar_init(&bar->b_empty[u], 1);  // the MMAs of the sequence's last tile
      }
      for (int u = 0; u < kWSlots; ++u) {
        mbar_init(&bar->w_full[u], 1);
        mbar_init(&bar->w_empty[u], 8);  // every epilogue warp, once per sequence
      }
      mbar_init(&bar->drain, 1);
      fence_mbar_init();
      tma_prefetch_desc(&tm_keys);
    }
    int64_t b0;
    int j0, count;
    locate_range(pos, batch, m, cap, kKeys, b0, j0, count);
    if (lane == 0) {
      bar->b0 = b0;
      bar->j0 = j0;
      bar->count = count;
    }
  } else if (warp == 1) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  // everything above is set-up; the cache (the emitted key) is written by the
  // previous kernel
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) bar->abort = flag_value(err);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const int count = bar->count;
  const int64_t b0 = bar->b0;
  const int j0 = bar->j0;
  // the same decision in every thread: the barriers of the epilogue need all
  const bool live = count > 0 && bar->abort == 0;

  constexpr int TPP = C::TPP;
  const int npairs = (count + TPP - 1) / TPP;
  if (warp == 0 && live) {
    // ------------------------------- TMA producer --------------------------------
    TileWalk it;
    it.start(pos, b0, j0, m, cap, kKeys);
    int k = 0;
    for (; k < npairs; ++k) {
      const int s = k % S;
      if (k >= S && !mbar_wait(&bar->empty[s], (uint32_t)(((k / S) - 1) & 1), err)) break;
      const int here = min(TPP, count - k * TPP);
      if (pk.btab == nullptr) {
        if (lane == 0) mbar_arrive_expect_tx(&bar->full[s], here * kTileBytes);
        for (int r = 0; r < here; ++r, it.next(pos, batch, m, cap))
          if (lane == 0)
            tma_load_3d(sRaw + s * C::STAGE_BYTES + r * kTileBytes, &tm_keys, &bar->full[s], 0,
                        it.j * kKeys, (int)it.b);
      } else {  // paged: per-block boxes of each tile of the stage, one barrier arm
        int64_t rows[TPP][8];
        uint32_t bytes = 0;
        TileWalk w2 = it;
        for (int r = 0; r < here; ++r, w2.next(pos, batch, m, cap))
          bytes += paged_tile_rows(pk, w2.b, (int64_t)w2.j * kKeys, kKeys,
                                   min((pos[w2.b] + 1) / m, cap), cap, rows[r]);
        if (lane == 0) mbar_arrive_expect_tx(&bar->full[s], bytes);
        for (int r = 0; r < here; ++r, it.next(pos, batch, m, cap))
          if (lane == 0)
            paged_tile_load(&tm_keys, &bar->full[s], sRaw + s * C::STAGE_BYTES + r * kTileBytes,
                            pk, rows[r]);
      }
      __syncwarp();
    }
    // every issued stage has landed before the CTA exits
    for (int r = (k > S ? k - S : 0); r < k; ++r)
      mbar_wait(&bar->full[r % S], (uint32_t)((r / S) & 1), err, false);
  } else if (warp == 1 && live) {
    // ------------------------------- MMA issuer ----------------------------------
    constexpr uint32_t kIdesc = idesc_e4m3(kKeys, C::N);
    const uint32_t a0 = smem_u32(sRaw), bb0 = smem_u32(sB);
    TileWalk it;
    it.start(pos, b0, j0, m, cap, kKeys);
    int u = -1;  // sequence counter within the range
    bool ok = true;
    for (int k = 0; k < npairs && ok; ++k) {
      const int s = k % S, q = k & 1;
      if (!(ok = mbar_wait(&bar->full[s], (uint32_t)((k / S) & 1), err))) break;
      if (k >= 2 && !(ok = mbar_wait(&bar->d_empty[q], (uint32_t)(((k >> 1) - 1) & 1), err)))
        break;
      tc_fence_after();
      for (int r = 0; r < TPP && k * TPP + r < count; ++r, it.next(pos, batch, m, cap)) {
        const int i = k * TPP + r;
        if (i == 0 || it.j == 0) {
          ++u;
          if (!(ok = mbar_wait(&bar->b_full[u & 1], (uint32_t)((u >> 1) & 1), err))) break;
          tc_fence_after();
        }
        if (lane == 0) {
          const uint32_t bslot = bb0 + (u & 1) * C::B_BYTES;
          const uint32_t at = a0 + s * C::STAGE_BYTES + r * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < kCI / 32; ++kk)  // K = 32 bytes per instruction
            mma_f8(tmem + (q * TPP + r) * C::N, desc_sw128(at + kk * 32),
                   desc_sw128(bslot + kk * 32), kIdesc, kk > 0 ? 1u : 0u);
          if (i + 1 == count || it.j + 1 == it.nt) mma_commit(&bar->b_empty[u & 1]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) {
        mma_commit(&bar->d_full[q]);
        mma_commit(&bar->empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(&bar->drain);
    __syncwarp();
    mbar_wait(&bar->drain, 0, err, false);
  } else if (warp == 2 && live) {
    // ----------- query operands: one bulk copy each, per sequence of the range -----------
    TileWalk it;
    it.start(pos, b0, j0, m, cap, kKeys);
    int left = count;
    constexpr uint32_t kRec = (uint32_t)(C::B_BYTES + H * 4);
    for (int u = 0; left > 0; ++u) {
      const int64_t b = it.b;
      const int here = min(left, it.nt - it.j);
      const int slot = u & 1, ws = u % kWSlots;
      // the B slot once the MMAs of sequence u-2 are done; the weight slot once
      // the epilogue is past sequence u-16
      if (u >= kBSlots && !mbar_wait(&bar->b_empty[slot], (uint32_t)(((u >> 1) - 1) & 1), err))
        break;
      if (u >= kWSlots &&
          !mbar_wait(&bar->w_empty[ws], (uint32_t)(((u / kWSlots) - 1) & 1), err))
        break;
      if (lane == 0) {
        const uint8_t* rec = qop + b * kRec;
        mbar_arrive_expect_tx(&bar->b_full[slot], C::B_BYTES);
        bulk_load(sB + slot * C::B_BYTES, rec, C::B_BYTES, &bar->b_full[slot]);
        mbar_arrive_expect_tx(&bar->w_full[ws], H * 4);
        bulk_load(sW + ws * H, rec + C::B_BYTES, H * 4, &bar->w_full[ws]);
      }
      __syncwarp();
      left -= here;
      for (int r = 0; r < here; ++r) it.next(pos, batch, m, cap);
    }
  } else if (warp >= 4 && live) {
    // --- epilogue: hi + lo, ReLU, head weights, key scale (group g: tile g of each pair,
    //     or every other pair when a pair is one tile) ---
    const int quad = warp & 3, grp = (warp - 4) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    auto mine_of = [&](int i) { return TPP == 2 ? (i & 1) == grp : ((i / TPP) & 1) == grp; };
    TileWalk it;
    it.start(pos, b0, j0, m, cap, kKeys);
    int64_t V = 0;
    // key scale of this group's next tile, loaded a tile ahead
    auto scale_of = [&](const TileWalk& w) -> float {
      const int64_t sidx = (int64_t)w.j * kKeys + row;
      const int64_t Vw = min((pos[w.b] + 1) / m, cap);
      const int64_t kr = sidx < Vw ? paged_row(pk, w.b, sidx, cap) : -1;
      return kr >= 0 ? __ldcs(key_scale + kr) : 0.f;
    };
    TileWalk ahead = it;
    int first = 0;  // this group's first tile
    while (first < count && !mine_of(first)) {
      ahead.next(pos, batch, m, cap);
      ++first;
    }
    float ks_next = first < count ? scale_of(ahead) : 0.f;
    const int etid = threadIdx.x - 4 * 32;
    int u = -1;
    // false once a wait of this warp gave up (the flag is set): from then on
    // nothing is awaited or written, but every barrier below is still reached
    bool alive = true;
    int seq_tiles = 0;  // tiles of the current sequence in this CTA's range so far
    for (int i = 0; i < count; ++i, it.next(pos, batch, m, cap)) {
      if (i == 0 || it.j == 0) {
        ++u;
        V = min((pos[it.b] + 1) / m, cap);
        seq_tiles = 0;
      }
      ++seq_tiles;
      const bool seq_end = i + 1 == count || it.j + 1 == it.nt;
      if (mine_of(i)) {
        const float ks = ks_next;
        if (i + 2 < count) {  // this group's next tile is i + 2
          ahead.next(pos, batch, m, cap);
          ahead.next(pos, batch, m, cap);
          ks_next = scale_of(ahead);
        }
        const int k = i / TPP, q = k & 1;
        const uint32_t acc_col = (uint32_t)((q * TPP + i % TPP) * C::N);
        // the head weights of this sequence are in place, then the accumulator
        bool ok = alive &&
                  mbar_wait(&bar->w_full[u % kWSlots], (uint32_t)((u / kWSlots) & 1), err) &&
                  mbar_wait(&bar->d_full[q], (uint32_t)((k >> 1) & 1), err);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          const float* w = sW + (u % kWSlots) * H;
          tc_fence_after();
          float acc[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
          for (int c = 0; c < H / 32; ++c) {
            uint32_t dh[32], dl[32];
            tmem_ld32(lane_addr + acc_col + c * 32, dh);
            tmem_ld32(lane_addr + acc_col + H + c * 32, dl);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 w4 = *reinterpret_cast<const float4*>(w + c * 32 + e);
              float* a = &acc[(e >> 2) & 7];
              *a = fmaf(w4.x, fmaxf(__uint_as_float(dh[e]) + __uint_as_float(dl[e]), 0.f), *a);
              *a = fmaf(w4.y, fmaxf(__uint_as_float(dh[e + 1]) + __uint_as_float(dl[e + 1]), 0.f), *a);
              *a = fmaf(w4.z, fmaxf(__uint_as_float(dh[e + 2]) + __uint_as_float(dl[e + 2]), 0.f), *a);
              *a = fmaf(w4.w, fmaxf(__uint_as_float(dh[e + 3]) + __uint_as_float(dl[e + 3]), 0.f), *a);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar->d_empty[q]);
          const float sum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
          const int64_t sidx = (int64_t)it.j * kKeys + row;
          if (sidx < V) {
            const float v = sum * ks;
            scores[it.b * cap + sidx] = v;
            hist_add(sHist, u & 1, v);
          }
        }
        alive = ok;
      }
      if (seq_end) {
        // both groups release the sequence's weights once they pass its end,
        // then add its histogram (every score of it in this CTA is counted)
        __syncwarp();
        if (lane == 0 && alive) mbar_arrive(&bar->w_empty[u % kWSlots]);
        alive = !named_bar_or(3, kEpiThreads, !alive);
        if (alive && ghist != nullptr) flush_hist(sHist, u & 1, ghist, it.b, etid);
        if (idx_done != nullptr) {
          // every score and histogram count of the sequence from this CTA is
          // written and fenced before the CTA's tile count is published
          __threadfence();
          alive = !named_bar_or(3, kEpiThreads, !alive);
          if (etid == 0 && alive) atomicAdd(idx_done + it.b, (uint32_t)seq_tiles);
        }
      }
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

// ---------------------------------------------------------------------------
// 64 heads: the query operand on the M side.  Its 128 rows (64 heads x hi,
// lo) come in blocks of 16: rows 0-7 the hi halves and rows 8-15 the lo
// halves of 8 heads, so that one 16-lane x 256-bit TMEM load gives a thread
// the hi and the lo accumulator of the same head and keys.  One M = 128 x
// N = 256 keys x K = 128 tile is four MMAs, half the instructions per key of
// the keys-on-M form.  The epilogue (four warps per tile, two groups taking
// alternate tiles) adds hi and lo, applies ReLU and the head weights of the
// thread's two heads, sums over the 8 lanes that hold the same keys by a
// shuffle reduce-scatter and over the four warps in shared memory, then
// scales by the key scale.
// ---------------------------------------------------------------------------
constexpr int kSwH = 64;
constexpr int kSwKeys = 256;                        // keys per tile (MMA N)
constexpr int kSwTileBytes = kSwKeys * kCI;         // 32 KB, one ring stage
constexpr int kSwABytes = 2 * kSwH * 128;           // query operand, 16 KB
constexpr int kSwRedBytes = 2 * 2 * 4 * kSwKeys * 4;  // [group][buffer][warp][key] fp32
constexpr int kSwStages = (kSmemLimit - 2048 - kBSlots * kSwABytes - kWSlots * kSwH * 4 -
                           kSwRedBytes - kHistBytes) / kSwTileBytes;
constexpr int kSwOffA = kSwStages * kSwTileBytes;
constexpr int kSwOffW = kSwOffA + kBSlots * kSwABytes;
constexpr int kSwOffRed = kSwOffW + kWSlots * kSwH * 4;
constexpr int kSwOffHist = kSwOffRed + kSwRedBytes;
constexpr int kSwOffBar = kSwOffHist + kHistBytes;
constexpr int kSwSmem = kSwOffBar + (int)sizeof(DecIdxBars<kSwStages>) + 1024;
static_assert(kSwStages >= 4 && kSwSmem <= kSmemLimit, "shared memory budget");
static_assert(kSwABytes + kSwH * 4 == 64 * (2 * 128 + 4), "query operand record");

// Sum of v over the 8 lanes that share lane % 4, reduce-scattered: on
// return v[0] holds entry (lane / 4) % 8 of the 8 summed.
__device__ __forceinline__ void reduce_scatter8(float (&v)[8], int lane) {
#pragma unroll
  for (int w = 4, sh = 16; w >= 1; w >>= 1, sh >>= 1) {
    const bool up = (lane & sh) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = up ? v[i] : v[i + w];
      const float keep = up ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, sh);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) decode_index_sw_kernel(
    const __grid_constant__ CUtensorMap tm_keys, const float* __restrict__ key_scale,
    PagedKeys pk, const uint8_t* __restrict__ qop, const int64_t* __restrict__ pos, int64_t batch,
    int64_t cap, int m, float* __restrict__ scores, uint32_t* __restrict__ ghist,
    uint32_t* __restrict__ idx_done,
    unsigned int* __restrict__ err) {
  constexpr int S = kSwStages;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sRaw = smem;
  uint8_t* sA = smem + kSwOffA;
  float* sW = reinterpret_cast<float*>(smem + kSwOffW);
  float* sRed = reinterpret_cast<float*>(smem + kSwOffRed);
  uint32_t* sHist = reinterpret_cast<uint32_t*>(smem + kSwOffHist);
  DecIdxBars<S>* bar = reinterpret_cast<DecIdxBars<S>*>(smem + kSwOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j = threadIdx.x; j < 2 * kHistBins; j += kThreads) sHist[j] = 0u;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < S; ++s) {
        mbar_init(&bar->full[s], 1);
        mbar_init(&bar->empty[s], 1);
      }
      for (int q = 0; q < 2; ++q) {
        mbar_init(&bar->d_full[q], 1);
        mbar_init(&bar->d_empty[q], 4);  // the four warps of the tile's group
      }
      for (int u = 0; u < kBSlots; ++u) {
        mbar_init(&bar->b_full[u], 1);
        mbar_init(&bar->b_empty[u], 1);  // the MMAs of the sequence's last tile
      }
      for (int u = 0; u < kWSlots; ++u) {
        mbar_init(&bar->w_full[u], 1);
        mbar_init(&bar->w_empty[u], 8);  // every epilogue warp, once per sequence
      }
      mbar_init(&bar->drain, 1);
      fence_mbar_init();
      tma_prefetch_desc(&tm_keys);
    }
    int64_t b0;
    int j0, count;
    locate_range(pos, batch, m, cap, kSwKeys, b0, j0, count);
    if (lane == 0) {
      bar->b0 = b0;
      bar->j0 = j0;
      bar->count = count;
    }
  } else if (warp == 1) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  // everything above is set-up; the cache (the emitted key) is written by the
  // previous kernel
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) bar->abort = flag_value(err);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const int count = bar->count;
  const int64_t b0 = bar->b0;
  const int j0 = bar->j0;
  // the same decision in every thread: the barriers of the epilogue need all
  const bool live = count > 0 && bar->abort == 0;

  if (warp == 0 && live) {
    // ------------------------------- TMA producer --------------------------------
    TileWalk it;
    it.start(pos, b0, j0, m, cap, kSwKeys);
    int i = 0;
    for (; i < count; ++i, it.next(pos, batch, m, cap)) {
      const int s = i % S;
      if (i >= S && !mbar_wait(&bar->empty[s], (uint32_t)(((i / S) - 1) & 1), err)) break;
      if (pk.btab == nullptr) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&bar->full[s], kSwTileBytes);
          tma_load_3d(sRaw + s * kSwTileBytes, &tm_keys, &bar->full[s], 0, it.j * kSwKeys,
                      (int)it.b);
        }
      } else {  // paged: one box per block piece of the tile
        int64_t rows[8];
        const uint32_t bytes = paged_tile_rows(pk, it.b, (int64_t)it.j * kSwKeys, kSwKeys,
                                               min((pos[it.b] + 1) / m, cap), cap, rows);
        if (lane == 0) {
          mbar_arrive_expect_tx(&bar->full[s], bytes);
          paged_tile_load(&tm_keys, &bar->full[s], sRaw + s * kSwTileBytes, pk, rows);
        }
      }
      __syncwarp();
    }
    // every issued stage has landed before the CTA exits
    for (int r = (i > S ? i - S : 0); r < i; ++r)
      mbar_wait(&bar->full[r % S], (uint32_t)((r / S) & 1), err, false);
  } else if (warp == 1 && live) {
    // ------------------------------- MMA issuer ----------------------------------
    constexpr uint32_t kIdesc = idesc_e4m3(2 * kSwH, kSwKeys);
    const uint32_t raw0 = smem_u32(sRaw), a0 = smem_u32(sA);
    TileWalk it;
    it.start(pos, b0, j0, m, cap, kSwKeys);
    int u = -1;  // sequence counter within the range
    for (int i = 0; i < count; ++i, it.next(pos, batch, m, cap)) {
      const int s = i % S, q = i & 1;
      if (!mbar_wait(&bar->full[s], (uint32_t)((i / S) & 1), err)) break;
      if (i >= 2 && !mbar_wait(&bar->d_empty[q], (uint32_t)(((i >> 1) - 1) & 1), err)) break;
      if (i == 0 || it.j == 0) {
        ++u;
        if (!mbar_wait(&bar->b_full[u & 1], (uint32_t)((u >> 1) & 1), err)) break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t aslot = a0 + (u & 1) * kSwABytes;
        const uint32_t bt = raw0 + s * kSwTileBytes;
#pragma unroll
        for (int kk = 0; kk < kCI / 32; ++kk)  // K = 32 bytes per instruction
          mma_f8(tmem + q * kSwKeys, desc_sw128(aslot + kk * 32), desc_sw128(bt + kk * 32),
                 kIdesc, kk > 0 ? 1u : 0u);
        if (i + 1 == count || it.j + 1 == it.nt) mma_commit(&bar->b_empty[u & 1]);
        mma_commit(&bar->d_full[q]);
        mma_commit(&bar->empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(&bar->drain);
    __syncwarp();
    mbar_wait(&bar->drain, 0, err, false);
  } else if (warp == 2 && live) {
    // ----------- query operands: one bulk copy each, per sequence of the range -----------
    TileWalk it;
    it.start(pos, b0, j0, m, cap, kSwKeys);
    int left = count;
    constexpr uint32_t kRec = (uint32_t)(kSwABytes + kSwH * 4);
    for (int u = 0; left > 0; ++u) {
      const int64_t b = it.b;
      const int here = min(left, it.nt - it.j);
      const int slot = u & 1, ws = u % kWSlots;
      if (u >= kBSlots && !mbar_wait(&bar->b_empty[slot], (uint32_t)(((u >> 1) - 1) & 1), err))
        break;
      if (u >= kWSlots &&
          !mbar_wait(&bar->w_empty[ws], (uint32_t)(((u / kWSlots) - 1) & 1), err))
        break;
      if (lane == 0) {
        const uint8_t* rec = qop + b * kRec;
        mbar_arrive_expect_tx(&bar->b_full[slot], kSwABytes);
        bulk_load(sA + slot * kSwABytes, rec, kSwABytes, &bar->b_full[slot]);
        mbar_arrive_expect_tx(&bar->w_full[ws], kSwH * 4);
        bulk_load(sW + ws * kSwH, rec + kSwABytes, kSwH * 4, &bar->w_full[ws]);
      }
      __syncwarp();
      left -= here;
      for (int r = 0; r < here; ++r) it.next(pos, batch, m, cap);
    }
  } else if (warp >= 4 && live) {
    // ---- epilogue: group grp takes the tiles i with i % 2 == grp (accumulator grp) ----
    const int wq = warp & 3, grp = (warp - 4) >> 2;
    // this thread's heads: 16 wq + lane / 4 (TMEM lanes 32 wq + lane / 4 and
    // + 8) and 16 wq + 8 + lane / 4 (lanes 32 wq + 16 + lane / 4 and + 8)
    const int head_a = wq * 16 + (lane >> 2), head_b = head_a + 8;
    const uint32_t acc_a = tmem + ((uint32_t)(wq * 32) << 16) + (uint32_t)(grp * kSwKeys);
    const uint32_t acc_b = acc_a + (16u << 16);
    // key of each 32-key chunk that this lane holds after the reduce-scatter
    const int vk = (lane >> 2) & 7;
    const int key_in_chunk = 8 * (vk >> 1) + 2 * (lane & 3) + (vk & 1);
    float* red_g = sRed + grp * (2 * 4 * kSwKeys);
    const int p = wq * 32 + lane;  // this thread's key pair in the final sum
    const int etid = threadIdx.x - 4 * 32;
    TileWalk it;
    it.start(pos, b0, j0, m, cap, kSwKeys);
    int64_t V = 0;
    int u = -1, mine = 0;
    // false once a wait of this group gave up (the flag is set): from then on
    // nothing is awaited or written, but every barrier below is still reached
    bool alive = true;
    int seq_tiles = 0;  // tiles of the current sequence in this CTA's range so far
    for (int i = 0; i < count; ++i, it.next(pos, batch, m, cap)) {
      if (i == 0 || it.j == 0) {
        ++u;
        V = min((pos[it.b] + 1) / m, cap);
        seq_tiles = 0;
      }
      ++seq_tiles;
      const bool seq_end = i + 1 == count || it.j + 1 == it.nt;
      if ((i & 1) == grp) {
        // key scales of this thread's two keys, ahead of the accumulator
        const int64_t s0 = (int64_t)it.j * kSwKeys + 2 * p;
        const int64_t kr0 = s0 < V ? paged_row(pk, it.b, s0, cap) : -1;  // s0 even: one block
        const float ks0 = kr0 >= 0 ? __ldcs(key_scale + kr0) : 0.f;
        const float ks1 = kr0 >= 0 && s0 + 1 < V ? __ldcs(key_scale + kr0 + 1) : 0.f;
        const bool ok =
            alive && mbar_wait(&bar->w_full[u % kWSlots], (uint32_t)((u / kWSlots) & 1), err) &&
            mbar_wait(&bar->d_full[grp], (uint32_t)(mine & 1), err);
        float* red = red_g + (mine & 1) * (4 * kSwKeys) + wq * kSwKeys;
        if (ok) {
          const float* wr = sW + (u % kWSlots) * kSwH;
          const float wa = wr[head_a], wb = wr[head_b];  // w_h s_h
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {  // 64 keys per pass
            uint32_t ra[32], rb[32];
            tmem_ld16x256_x8(acc_a + c * 64, ra);
            tmem_ld16x256_x8(acc_b + c * 64, rb);
            tmem_ld_wait();
            if (c == 3) {  // the accumulator is free for the tile after next
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bar->d_empty[grp]);
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {  // 32-key chunk 2 c + half
              float v[8];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const int r = 4 * (4 * half + k);
                  const float ha = __uint_as_float(ra[r + e]) + __uint_as_float(ra[r + 2 + e]);
                  const float hb = __uint_as_float(rb[r + e]) + __uint_as_float(rb[r + 2 + e]);
                  v[2 * k + e] = fmaf(wa, fmaxf(ha, 0.f), wb * fmaxf(hb, 0.f));
                }
              }
              reduce_scatter8(v, lane);
              red[(2 * c + half) * 32 + key_in_chunk] = v[0];
            }
          }
        }
        // a failed wait set the error flag; the group stops together
        alive = !named_bar_or(1 + grp, 128, !ok);
        if (alive) {
          const float* rs = red_g + (mine & 1) * (4 * kSwKeys) + 2 * p;
          float2 sum = *reinterpret_cast<const float2*>(rs);
#pragma unroll
          for (int w = 1; w < 4; ++w) {
            const float2 x = *reinterpret_cast<const float2*>(rs + w * kSwKeys);
            sum.x += x.x;
            sum.y += x.y;
          }
          float* out = scores + it.b * cap + s0;
          if (s0 < V) {
            const float v0 = sum.x * ks0;
            __stcg(out, v0);
            hist_add(sHist, u & 1, v0);
          }
          if (s0 + 1 < V) {
            const float v1 = sum.y * ks1;
            __stcg(out + 1, v1);
            hist_add(sHist, u & 1, v1);
          }
        }
        ++mine;
      }
      if (seq_end) {
        // both groups release the sequence's weights once they pass its end,
        // then add its histogram (every score of it in this CTA is counted)
        __syncwarp();
        if (lane == 0 && alive) mbar_arrive(&bar->w_empty[u % kWSlots]);
        alive = !named_bar_or(3, kEpiThreads, !alive);
        if (alive && ghist != nullptr) flush_hist(sHist, u & 1, ghist, it.b, etid);
        if (idx_done != nullptr) {
          // every score and histogram count of the sequence from this CTA is
          // written and fenced before the CTA's tile count is published
          __threadfence();
          alive = !named_bar_or(3, kEpiThreads, !alive);
          if (etid == 0 && alive) atomicAdd(idx_done + it.b, (uint32_t)seq_tiles);
        }
      }
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

// The key tensor map: [batch][capacity][128] with boxes of `tk` keys, or
// (paged) the pool's [blocks * entries-per-block][128] rows with boxes of one
// block piece; the matching PagedKeys.
bool key_map(const csa_cache_desc& d, const CacheView& cv, int tk, CUtensorMap* tm,
             PagedKeys* pk) {
  if (cv.btab == nullptr) {
    *pk = PagedKeys{nullptr, 0, 0, 0, tk};
    return make_tmap_3d(tm, cv.ikey_fp8, 1, kCI, (uint64_t)d.capacity, (uint64_t)d.batch, kCI,
                        (uint64_t)d.capacity * kCI, kCI, (uint32_t)tk);
  }
  const int epb = 1 << cv.epb_shift;
  const int box = std::min(epb, tk);
  *pk = PagedKeys{cv.btab, cv.bt_stride, cv.nblocks, cv.epb_shift, box};
  const uint64_t rows = (uint64_t)cv.nblocks << cv.epb_shift;
  return make_tmap_3d(tm, cv.ikey_fp8, 1, kCI, rows, 1, kCI, rows * kCI, kCI, (uint32_t)box);
}

cudaError_t launch_sw(const csa_cache_desc& d, const CacheView& cv, const int64_t* pos,
                      const uint8_t* qop, float* scores, uint32_t* ghist, uint32_t* idx_done,
                      unsigned int* err, cudaStream_t s) {
  CUtensorMap tk;
  PagedKeys pk;
  if (!key_map(d, cv, kSwKeys, &tk, &pk)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(decode_index_sw_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSwSmem);
  if (e != cudaSuccess) return e;
  const int64_t max_tiles = d.batch * ((d.capacity + kSwKeys - 1) / kSwKeys);
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(sm_count(), max_tiles));
  return launch_pdl(decode_index_sw_kernel, dim3(grid), dim3(kThreads), (size_t)kSwSmem, s, tk,
                    (const float*)cv.ikey_scale, pk, qop, pos, (int64_t)d.batch,
                    (int64_t)d.capacity, d.m, scores, ghist, idx_done, err);
}

template <int H>
cudaError_t launch_h(const csa_cache_desc& d, const CacheView& cv, const int64_t* pos,
                     const uint8_t* qop, float* scores, uint32_t* ghist, uint32_t* idx_done,
                     unsigned int* err, cudaStream_t s) {
  using C = DecIdxCfg<H>;
  CUtensorMap tk;
  PagedKeys pk;
  if (!key_map(d, cv, kKeys, &tk, &pk)) return cudaErrorInvalidValue;
  auto kern = decode_index_tc_kernel<H>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t max_tiles = d.batch * ((d.capacity + kKeys - 1) / kKeys);
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(sm_count(), max_tiles));
  return launch_pdl(kern, dim3(grid), dim3(kThreads), (size_t)C::SMEM, s, tk,
                    (const float*)cv.ikey_scale, pk, qop, pos,
                    (int64_t)d.batch, (int64_t)d.capacity, d.m, scores, ghist, idx_done, err);
}

}  // namespace

bool decode_index_tc_supported(const csa_cache_desc& d) {
  return !d.is_hca && d.c_i == kCI && (d.nh_i == 64 || d.nh_i == 128);
}

int decode_index_tile_keys(const csa_cache_desc& d) { return d.nh_i == 64 ? kSwKeys : kKeys; }

cudaError_t launch_decode_index_tc(const csa_cache_desc& d, const CacheView& cv,
                                   const int64_t* pos, const uint8_t* qop, float* scores,
                                   uint32_t* ghist, uint32_t* idx_done, unsigned int* err,
                                   cudaStream_t s) {
  switch (d.nh_i) {
    case 64: return launch_sw(d, cv, pos, qop, scores, ghist, idx_done, err, s);
    case 128: return launch_h<128>(d, cv, pos, qop, scores, ghist, idx_done, err, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace csa
