// Decode attention on the tcgen05 tensor cores over the FP8/bf16 cache.
//
// For the decode token of sequence b at position t, E_t is (CSA) the selected
// entries sel[b, :] with 0 <= s < V = floor((t+1)/m), or (HCA) every visible
// entry, followed by the window rows max(0, t-W+1) .. t from the ring
// (sections 4.3 / 4.5 of "DeepSeek-V4: million-token context"; entries stored
// as 448 FP8 codes with one fp32 scale plus 64 bf16 RoPE dims, section 7.3 of
// the "DeepSeek paper-feature analysis"); one softmax over E_t and the sink.
//
// E_t is cut into 128-entry tiles and each sequence's tiles into `nsplit`
// contiguous ranges, one CTA per range (about one CTA per SM over the
// batch).  In a CTA:
//   * the eight softmax warps also gather: each thread owns one 16-dim
//     quarter of one 64-dim slab for 16 rows of the tile; once the
//     previous tile's P.V has released that slab it copies the rows' bytes
//     there by cp.async (the FP8 codes of a row are 448 contiguous bytes, the
//     RoPE dims and window rows 1 KB of bf16) and widens the FP8 quarters in
//     place (code * scale -> bf16, 128-byte swizzle);
//   * S^T = K Q^T (M = 128 entries, N = 64 heads), the eight softmax warps
//     keep a running max per head (moved, with O^T rescaled in TMEM, only
//     when a tile's max exceeds it by more than 2^8) and write P^T in bf16;
//   * O^T += V^T P^T (four M = 128 dim chunks) accumulates in TMEM across the
//     CTA's tiles; each chunk's completion frees two slabs for the next
//     tile's gather.
// The CTA's unnormalised O, max and sum go to the partial buffers and a
// combine kernel merges a sequence's ranges with the sink; with one range per
// sequence the CTA writes the normalised output itself.  Every wait is
// bounded: a fault upstream ends the kernel with the timeout flag set.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"
#include "tc_attn_util.cuh"

namespace csa {

namespace {

constexpr int kNH = 64, kC = 512, kTE = 128;
constexpr int kRope = 64, kBody = kC - kRope;  // FP8 dims, then bf16 RoPE dims
constexpr int kSlabs = kC / 64;                // 64-dim slabs; slab 7 holds the RoPE dims
constexpr int kSlabBytes = kTE * 128;          // 16 KB
constexpr int kQSlabBytes = kNH * 128;         // 8 KB
constexpr int kSoftWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kThreads = (kMmaWarp + 1) * 32;  // 288
constexpr int kGatherThreads = kMmaWarp * 32;  // 256: the softmax warps gather too
constexpr int kRowsPerThread = (kTE + kMmaWarp - 1) / kMmaWarp;  // 16
constexpr int kMaxSelDec = 1024;
constexpr float kRescaleLog2 = 8.f;
static_assert(kGatherThreads % 32 == 0, "a thread keeps one slab quarter for every row");

constexpr uint32_t kColS = 0, kColO = 64;  // S^T: 64 columns; O^T: 4 chunks x 64 columns

struct __align__(8) DecAttnBars {
  uint64_t slab_full[kSlabs], slab_empty[kSlabs];
  uint64_t q_full, s_full, p_full, p_empty, o_full, grp[2];
  uint32_t tmem_base;
  unsigned int abort;  // the timeout flag as read once for the whole CTA
};

constexpr int OFF_Q = 0;
constexpr int OFF_KV = OFF_Q + kSlabs * kQSlabBytes;    // 65536
constexpr int OFF_P = OFF_KV + kSlabs * kSlabBytes;     // 196608
constexpr int OFF_LIST = OFF_P + kTE * 128;             // 212992
constexpr int OFF_RED = OFF_LIST + kMaxSelDec * 4;      // [2 (max,sum)][2 hh][4 quad][32]
constexpr int OFF_SCAN = OFF_RED + 2 * 2 * 4 * 32 * 4;  // [12] warp counts
constexpr int OFF_BM = OFF_SCAN + 64;                   // selection bitmap, 1 bit per entry
// The selection stages the scores in the Q and KV slabs (192 KB): kSelScores
// floats, then the bitmap of the threshold bin's entries (kSelWords words).
constexpr int kSelStage = 49152;
constexpr int kSelWords = kSelStage / 32;
constexpr int kSelScores = kSelStage - kSelWords;
constexpr int OFF_SCALE = OFF_BM + kSelWords * 4;        // [128] FP8 scales of a tile's rows
constexpr int OFF_BAR = OFF_SCALE + kTE * 4;
constexpr int SMEM = OFF_BAR + (int)sizeof(DecAttnBars) + 1024;
static_assert(SMEM <= 232448, "shared memory budget");

// 16 FP8 codes -> 16 bf16 (code * scale), as two 16-byte chunks.
__device__ __forceinline__ void dequant16(const uint4 c8, float sc, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {c8.x, c8.y, c8.z, c8.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int hlf = 0; hlf < 2; ++hlf) {
      const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w[i] >> (16 * hlf)) & 0xffffu);
      const __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
      o[2 * i + hlf] = pack_bf16x2(f.x * sc, f.y * sc);
    }
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// ---------------------------------------------------------------------------
// The selection step inside the attention kernel (the top-k of section 4.2 of
// "DeepSeek-V4: million-token context"; larger score first, ties to the
// smaller index): the indexer left a histogram of the sequence's scores over
// the top 12 bits of their order keys, which gives the bin T holding the k-th
// largest score, the count G above it and the count C in it.  The scores land
// in shared memory by cp.async; one pass then marks, by warp ballots (one
// 32-entry word each), the scores above bin T in the selection bitmap and
// those in bin T in a candidate bitmap; the need = k - G largest candidates
// (two more radix digits of the key, then the smaller indices among equal
// keys) join the selection, and the chosen indices are emitted in ascending
// order from the bitmap.  Every thread of the CTA calls it; returns min(k, V).
// ---------------------------------------------------------------------------
constexpr int kSelBins = 4096;

struct SelState {
  uint32_t T, G, C;
};

// The bin T (among `nbins`, counts in h, bin nbins - 1 highest) where the
// count from the top reaches `need`, with the count above it (G) and in it.
__device__ __noinline__ void sel_find_bin(const uint32_t* h, int nbins, uint32_t need,
                                          int* wsum, SelState* st) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kPerMax = (kSelBins + kThreads - 1) / kThreads;
  const int per = (nbins + kThreads - 1) / kThreads;
  uint32_t c[kPerMax], loc = 0;
#pragma unroll
  for (int j = 0; j < kPerMax; ++j) {
    const int bin = nbins - 1 - (tid * per + j);
    c[j] = (j < per && bin >= 0) ? h[bin] : 0u;
    loc += c[j];
  }
  uint32_t inc = loc;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += x;
  }
  if (lane == 31) wsum[warp] = (int)inc;
  __syncthreads();
  uint32_t acc = inc - loc;
  for (int w = 0; w < warp; ++w) acc += (uint32_t)wsum[w];
#pragma unroll
  for (int j = 0; j < kPerMax; ++j) {
    const int bin = nbins - 1 - (tid * per + j);
    if (j < per && bin >= 0 && acc < need && acc + c[j] >= need) {
      st->T = (uint32_t)bin;
      st->G = acc;
      st->C = c[j];
    }
    acc += c[j];
  }
  __syncthreads();
}

// Block-wide exclusive prefix of v.
__device__ __forceinline__ uint32_t sel_excl(uint32_t v, int* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += x;
  }
  if (lane == 31) wsum[warp] = (int)inc;
  __syncthreads();
  uint32_t a = inc - v;
  for (int w = 0; w < warp; ++w) a += (uint32_t)wsum[w];
  __syncthreads();
  return a;
}

__device__ int fused_select(const float* __restrict__ row, const uint32_t* __restrict__ gh,
                            int V, int k, float* stage, uint32_t* hist, uint32_t* bm,
                            int32_t* list, int* wsum, SelState* st) {
  using namespace sm100;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (V <= k) {
#pragma unroll 1
    for (int i = tid; i < V; i += kThreads) list[i] = i;
    __syncthreads();
    return V;
  }
  // the scores (as 16-byte chunks from the row's 16-byte-aligned start: a
  // chunk holding any score of the row never crosses a page) and the
  // histogram, in one round trip
  const int r0 = (int)((reinterpret_cast<uintptr_t>(row) >> 2) & 3);
  const float* abase = row - r0;
  const int nchunk = (V + r0 + 3) >> 2;
  const uint32_t sk = smem_u32(stage), sh = smem_u32(hist);
#pragma unroll 1
  for (int c = tid; c < nchunk; c += kThreads) cp_async_16(sk + 16u * c, abase + 4 * c);
#pragma unroll 1
  for (int c = tid; c < kSelBins / 4; c += kThreads) cp_async_16(sh + 16u * c, gh + 4 * c);
  cp_async_wait_all();
  if (tid == 0) *st = SelState{0u, 0u, 0u};  // (a histogram short of k: a capped result)
  __syncthreads();
  sel_find_bin(hist, kSelBins, (uint32_t)k, wsum, st);
  const uint32_t T = st->T;
  uint32_t need = (uint32_t)k - st->G;
  const bool all_of_T = st->C == need;
  const float* sc = stage + r0;  // score i at sc[i]
  uint32_t* cbm = reinterpret_cast<uint32_t*>(stage + kSelScores);
  const int nwords = (V + 31) >> 5;
  // one pass: "above bin T" (or "in or above" when bin T is taken whole) and
  // "in bin T".  A warp takes 128 scores a step, four per lane; each lane's
  // four bits are OR-reduced over the eight lanes of a 32-score word.
  const int nblk = (nwords + 3) >> 2;
#pragma unroll 1
  for (int q = warp; q < nblk; q += kThreads / 32) {
    const int i0 = q * 128 + 4 * lane;
    uint32_t ab = 0u, cd = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = i0 + e;
      const uint32_t bin = i < V ? order_key(sc[i]) >> 20 : 0u;
      const bool in = i < V && bin == T;
      ab |= (i < V && (bin > T || (all_of_T && in)) ? 1u : 0u) << e;
      cd |= (in && !all_of_T ? 1u : 0u) << e;
    }
    ab <<= 4 * (lane & 7);
    cd <<= 4 * (lane & 7);
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      ab |= __shfl_xor_sync(0xffffffffu, ab, off);
      cd |= __shfl_xor_sync(0xffffffffu, cd, off);
    }
    const int w = q * 4 + (lane >> 3);
    if ((lane & 7) == 0 && w < nwords) {
      bm[w] = ab;
      cbm[w] = cd;
    }
  }
  __syncthreads();
  // thread tid owns words [w0, w1) from here on
  const int per = (nwords + kThreads - 1) / kThreads;
  const int w0 = min(nwords, tid * per), w1 = min(nwords, w0 + per);
  if (!all_of_T) {
    // the need largest candidates by the value (key bits 19..0, then
    // 65535 - index): radix digits of 11, 9, 8 and 8 bits until a digit's
    // bin is taken whole (the values are unique, so the last one is)
    auto val = [&](int i) -> uint64_t {
      return ((uint64_t)(order_key(sc[i]) & 0xfffffu) << 16) | (uint64_t)(0xffffu - (uint32_t)i);
    };
    uint64_t pfx = 0, msk = 0;
    bool settled = false;
    constexpr int kShift[4] = {25, 16, 8, 0};
    constexpr int kWidth[4] = {11, 9, 8, 8};
#pragma unroll 1
    for (int lvl = 0; lvl < 4 && !settled; ++lvl) {
      const int shf = kShift[lvl], nb = 1 << kWidth[lvl];
#pragma unroll 1
      for (int j = tid; j < nb; j += kThreads) hist[j] = 0u;
      __syncthreads();
#pragma unroll 1
      for (int w = w0; w < w1; ++w) {
        uint32_t x = cbm[w];
        while (x != 0u) {
          const int i = w * 32 + __ffs(x) - 1;
          x &= x - 1u;
          const uint64_t v = val(i);
          if ((v & msk) == pfx) atomicAdd(&hist[(uint32_t)(v >> shf) & (uint32_t)(nb - 1)], 1u);
        }
      }
      __syncthreads();
      sel_find_bin(hist, nb, need, wsum, st);
      need -= st->G;
      pfx |= (uint64_t)st->T << shf;
      msk |= (uint64_t)(nb - 1) << shf;
      settled = st->C == need;
    }
    // chosen candidates: above the prefix on the ranked bits, or equal to it
#pragma unroll 1
    for (int w = w0; w < w1; ++w) {
      uint32_t x = cbm[w], take = 0u;
      while (x != 0u) {
        const int bit = __ffs(x) - 1;
        x &= x - 1u;
        if ((val(w * 32 + bit) & msk) >= pfx) take |= 1u << bit;
      }
      bm[w] |= take;
    }
  }
  // emit: the marked indices in ascending order
  uint32_t cnt = 0;
#pragma unroll 1
  for (int w = w0; w < w1; ++w) cnt += (uint32_t)__popc(bm[w]);
  uint32_t o = sel_excl(cnt, wsum);
#pragma unroll 1
  for (int w = w0; w < w1; ++w) {
    uint32_t x = bm[w];
    while (x != 0u) {
      const int bit = __ffs(x) - 1;
      x &= x - 1u;
      if (o < (uint32_t)k) list[o] = w * 32 + bit;
      ++o;
    }
  }
  fence_proxy_async();  // the staged scores are overwritten by TMA next
  __syncthreads();
  return k;
}

// Split s > 0 of a selecting launch, before its first tile that needs the
// selection: waits (thread 0) for split 0 to publish it, then the gather
// threads copy slots [lo, hi) of it into shared memory.  False if the wait
// gave up (in every gather thread).
__device__ __noinline__ bool fetch_list(const uint32_t* ready, const int32_t* src, int32_t* list,
                                        int lo, int hi, unsigned int* err) {
  using namespace sm100;
  const int tid = threadIdx.x;
  const bool got = tid != 0 || wait_count(ready, 1u, err);
  if (named_bar_or(2, kGatherThreads, !got)) return false;
  for (int sl = lo + tid; sl < hi; sl += kGatherThreads) list[sl] = __ldcg(src + sl);
  named_bar_or(2, kGatherThreads, false);
  return true;
}

// kSelect: the launch selects (scores != NULL); the other instance (HCA, or
// a selection given in sel) holds none of the selection code.
template <bool kSelect>
__global__ void __launch_bounds__(kThreads, 1) decode_attn_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CacheView cv,
    const int64_t* __restrict__ pos, const int32_t* __restrict__ sel, int k, int window, int m,
    int64_t cap, const float* __restrict__ sink, float scale, int nsplit,
    float* __restrict__ part_o, float* __restrict__ part_ms, __nv_bfloat16* __restrict__ out,
    const float* __restrict__ scores, const uint32_t* __restrict__ ghist,
    int32_t* __restrict__ sel_out, const uint32_t* __restrict__ idx_done, int idx_tile,
    int32_t* __restrict__ xlist, uint32_t* __restrict__ list_ready,
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
  float* sScale = reinterpret_cast<float*>(smem + OFF_SCALE);
  DecAttnBars* bar = reinterpret_cast<DecAttnBars*>(smem + OFF_BAR);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x;
  const int64_t b = blockIdx.y;
  const bool direct = nsplit == 1;
  const int64_t pbase = (b * nsplit + split) * kNH;

  if (tid == 0) {
#pragma unroll 1
    for (int s = 0; s < kSlabs; ++s) {
      mbar_init(&bar->slab_full[s], kGatherThreads / 8);  // 4 lanes per slab in each warp
      mbar_init(&bar->slab_empty[s], 1);
    }
    mbar_init(&bar->q_full, 1);
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->p_full, kSoftWarps);
    mbar_init(&bar->p_empty, 1);
    mbar_init(&bar->o_full, 1);
    mbar_init(&bar->grp[0], 4);
    mbar_init(&bar->grp[1], 4);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  // the window ring of the sequence (the rows of the range's last tile)
  // starts moving into L2 under the wait: a prefetch changes no data
  if (split == nsplit - 1 && tid == 0 && window <= 4096)
    bulk_prefetch_l2(cv.window + b * window * kC, (uint32_t)window * kC * 2);
  // set-up above; the selection and the cache are written by earlier kernels.
  // Selecting here from the indexer's scores, the sequence's own tile count
  // is awaited rather than the end of the indexer's grid, so a sequence
  // starts as soon as its keys are scored (the cache itself was written
  // before the indexer started)
  if (kSelect && idx_done != nullptr) {
    // (only the selecting CTA of a sequence reads what the indexer wrote)
    if (tid == 0 && split == 0) {
      const int64_t tp = pos[b];
      const int64_t Vp = tp < 0 ? 0 : min((tp + 1) / m, cap);
      const uint32_t want = (uint32_t)((Vp + idx_tile - 1) / idx_tile);
      const bool ok = want == 0 || wait_count(idx_done + b, want, err);
      bar->abort = ok ? flag_value(err) : 1u;
    }
    if (tid == 0 && split != 0) bar->abort = flag_value(err);
    __syncthreads();  // nothing indexer-written is read before the count is complete
  } else {
    pdl_wait();
    if (tid == 0) bar->abort = flag_value(err);
  }
  pdl_trigger();
  const int64_t t = pos[b];
  const int64_t V = t < 0 ? 0 : min((t + 1) / m, cap);
  const int64_t w0 = max((int64_t)0, t - window + 1);
  const int nwin = t < 0 ? 0 : (int)(t - w0 + 1);
  // ring slot of window row w0 (row w0 + i sits at slot w0m + i, wrapped
  // once: i < window), so no 64-bit remainder per row
  const int w0m = (int)(w0 % window);
  const __nv_bfloat16* const ring = cv.window + b * window * kC;

  // -------- the entry list: valid selections in order (CSA) or 0..V-1 (HCA) ----
  // (scores != NULL: the CSA selection itself runs here, from the indexer's
  // scores and histogram)
  const bool csa = sel != nullptr || kSelect;
  int nsel;
  // (split > 0 of a selecting launch: the selection comes from split 0 of the
  // same sequence through xlist; the range's window-only tiles go first)
  bool xfetch = false;
  if (kSelect && split == 0) {
    SelState* st = reinterpret_cast<SelState*>(red);
    nsel = fused_select(scores + b * cap, ghist + b * kSelBins, (int)V, k,
                        reinterpret_cast<float*>(sQ), reinterpret_cast<uint32_t*>(sP),
                        reinterpret_cast<uint32_t*>(smem + OFF_BM), list, wcount, st);
    if (nsplit > 1 && V > k && xlist != nullptr) {
#pragma unroll 1
      for (int j = tid; j < nsel; j += kThreads) xlist[b * k + j] = list[j];
      __threadfence();
      __syncthreads();
      if (tid == 0)
        asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(list_ready + b), "r"(1u)
                     : "memory");
    }
    if (sel_out != nullptr)
#pragma unroll 1
      for (int j = tid; j < k; j += kThreads) sel_out[b * k + j] = j < nsel ? list[j] : -1;
  } else if (kSelect) {
    nsel = (int)min(V, (int64_t)k);
    if (V <= k) {
#pragma unroll 1
      for (int i = tid; i < nsel; i += kThreads) list[i] = i;
    } else {
      xfetch = true;
    }
  } else if (sel != nullptr) {
    const int32_t* row = sel + b * k;
    const int per = (k + kThreads - 1) / kThreads;
    const int lo = min(k, tid * per), hi = min(k, lo + per);
    int cnt = 0;
#pragma unroll 1
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
#pragma unroll 1
    for (int j = lo; j < hi; ++j)
      if (row[j] >= 0 && row[j] < V) list[p++] = row[j];
  } else {
    nsel = (int)V;
  }
  const int N = nsel + nwin;
  const int T = (N + kTE - 1) / kTE;
  const int tile0 = (int)((int64_t)T * split / nsplit);
  const int tile1 = (int)((int64_t)T * (split + 1) / nsplit);
  const int ntile = tile1 - tile0;
  // tiles of the range in processing order: with xfetch, the tiles holding
  // only window rows (slots >= nsel) first, while split 0 selects
  const int wtile = max(tile0, (nsel + kTE - 1) / kTE);
  const int nw = xfetch ? max(0, tile1 - wtile) : 0;
  auto tile_at = [&](int jt) { return jt < nw ? wtile + jt : tile0 + (jt - nw); };
  tc_fence_before();
  __syncthreads();  // the list, the barriers and the TMEM address
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const bool live = ntile > 0 && bar->abort == 0;
  if (!live && !direct && tid < kNH) {  // an empty range adds nothing to the combine
    part_ms[(pbase + tid) * 2 + 0] = kNegInf;
    part_ms[(pbase + tid) * 2 + 1] = 0.f;
  }

  // -------- gather of tile jt of the range by one thread -------------------------
  // Thread tid owns 16-dim quarter q_me of slab s_me for rows warp + 8 i.
  // The bytes travel by cp.async straight into the slab (no registers held
  // across the copy): a bf16 quarter (RoPE dims, window rows) lands in its two
  // final 16-byte chunks; an FP8 quarter (16 codes) lands in the second of
  // them and is widened in place once it has arrived (code * scale -> bf16
  // into both chunks; only this thread touches them).
  const int s_me = (tid & 31) >> 2, q_me = tid & 3;
  auto gather_tile = [&](int jt) -> bool {
    const int tile = tile_at(jt);
    const bool body = s_me < kBody / 64;
    // the slab is free once the previous tile's P.V chunk that reads it is done
    const bool free_ok =
        jt == 0 || mbar_wait_small(&bar->slab_empty[s_me], (uint32_t)((jt - 1) & 1), err);
    const uint32_t dst = smem_u32(sKV) + (uint32_t)(s_me * kSlabBytes);
    if (free_ok) {
#pragma unroll 2
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int r = warp + kMmaWarp * i;
        const int slot = tile * kTE + r;
        const uint32_t d0 = dst + (uint32_t)(r * 128 + (((2 * q_me) ^ (r & 7)) * 16));
        const uint32_t d1 = d0 ^ 16u;  // chunks 2 q and 2 q + 1 differ in bit 4 only
        const int64_t es =
            slot < nsel ? entry_row(cv, b, csa ? (int64_t)list[slot] : (int64_t)slot, cap) : -1;
        if (es >= 0) {
          if (body) {
            cp_async_16(d1, cv.entry_fp8 + es * kBody + s_me * 64 + q_me * 16);
            if (lane == 0)  // the row's scale, for every thread of the row
              asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                               smem_u32(sScale + r)),
                           "l"(cv.entry_scale + es)
                           : "memory");
          } else {
            const __nv_bfloat16* p = cv.entry_rope + es * kRope + q_me * 16;
            cp_async_16(d0, p);
            cp_async_16(d1, p + 8);
          }
        } else if (slot >= nsel && slot < N) {
          int u = w0m + (slot - nsel);
          u -= u >= window ? window : 0;
          const __nv_bfloat16* p = ring + (int64_t)u * kC + s_me * 64 + q_me * 16;
          cp_async_16(d0, p);
          cp_async_16(d1, p + 8);
        } else {  // past the end, or an entry without a block: zeros
          st_shared_v4(d0, make_uint4(0, 0, 0, 0));
          st_shared_v4(d1, make_uint4(0, 0, 0, 0));
          if (lane == 0) sScale[r] = 0.f;
        }
      }
    }
    cp_async_wait_all();
    // every gather thread's copies (the scales included) have landed; a
    // failed wait anywhere stops them all here
    if (named_bar_or(1, kGatherThreads, !free_ok)) return false;
    if (body) {
#pragma unroll 2
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int r = warp + kMmaWarp * i;
        if (tile * kTE + r >= nsel) continue;
        const uint32_t d0 = dst + (uint32_t)(r * 128 + (((2 * q_me) ^ (r & 7)) * 16));
        const uint32_t d1 = d0 ^ 16u;
        uint4 a, c;
        dequant16(ld_shared_v4(d1), sScale[r], a, c);
        st_shared_v4(d0, a);
        st_shared_v4(d1, c);
      }
    }
    fence_proxy_async();  // generic-proxy writes before the tensor core reads them
    mbar_arrive(&bar->slab_full[s_me]);
    return true;
  };

  if (warp == kMmaWarp) {
    // -------------------------------- MMA ----------------------------------------
    if (live) {
      constexpr uint32_t kIdQK = idesc_bf16(kTE, kNH, 0, 0);
      constexpr uint32_t kIdPV = idesc_bf16(128, kNH, 1, 1);
      const uint32_t kv0 = smem_u32(sKV), q0 = smem_u32(sQ), p0 = smem_u32(sP);
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar->q_full, kSlabs * kQSlabBytes);
        for (int s = 0; s < kSlabs; ++s)
          tma_load_3d(sQ + s * kQSlabBytes, &tm_q, &bar->q_full, s * 64, 0, (int)b);
      }
      __syncwarp();
      bool ok = mbar_wait_small(&bar->q_full, 0, err);
      int issued = 0;  // tiles whose P.V was issued
      for (int jt = 0; jt < ntile && ok; ++jt) {
        for (int s = 0; s < kSlabs && ok; ++s)
          ok = mbar_wait_small(&bar->slab_full[s], (uint32_t)(jt & 1), err);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
#pragma unroll 1
          for (int s = 0; s < kSlabs; ++s)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(tmem + kColS, desc_sw128(kv0 + s * kSlabBytes + kk * 32),
                       desc_sw128(q0 + s * kQSlabBytes + kk * 32), kIdQK, (s | kk) != 0 ? 1u : 0u);
          mma_commit(&bar->s_full);
        }
        __syncwarp();
        if (!(ok = mbar_wait_small(&bar->p_full, (uint32_t)(jt & 1), err))) break;
        tc_fence_after();
        if (lane == 0) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int kk = 0; kk < kTE / 16; ++kk)
              mma_bf16(tmem + kColO + c * kNH,
                       desc_sw128_mn(kv0 + 2 * c * kSlabBytes + kk * 2048, kSlabBytes, 1024),
                       desc_sw128_mn(p0 + kk * 2048, 1024, 1024), kIdPV,
                       (jt == 0 && kk == 0) ? 0u : 1u);
            mma_commit(&bar->slab_empty[2 * c]);
            mma_commit(&bar->slab_empty[2 * c + 1]);
          }
          mma_commit(&bar->p_empty);
        }
        __syncwarp();
        ++issued;
      }
      if (lane == 0) mma_commit(&bar->o_full);
      __syncwarp();
      mbar_wait_small(&bar->o_full, 0, err, false);  // every MMA done before TMEM is released
      if (!ok && issued == 0) mbar_wait_small(&bar->q_full, 0, err, false);  // the Q load has landed
    }
  } else if (live) {
    // -------- gather, softmax and epilogue (warps 0-7) ------------------------------
    // the rows of the range's later tiles start moving into L2 now (one bulk
    // prefetch per piece), so that their gathers, which wait for the slabs,
    // read L2 rather than HBM
#pragma unroll 1
    for (int slot = (tile0 + 1) * kTE + tid; slot < min(N, tile1 * kTE); slot += kGatherThreads) {
      if (slot < nsel) {
        if (xfetch) continue;  // (the selection is not known yet)
        const int64_t es = entry_row(cv, b, csa ? (int64_t)list[slot] : (int64_t)slot, cap);
        if (es >= 0) {
          bulk_prefetch_l2(cv.entry_fp8 + es * kBody, kBody);
          bulk_prefetch_l2(cv.entry_rope + es * kRope, kRope * 2);
          bulk_prefetch_l2(cv.entry_scale + (es & ~(int64_t)3), 16);
        }
      } else {
        int u = w0m + (slot - nsel);
        u -= u >= window ? window : 0;
        bulk_prefetch_l2(ring + (int64_t)u * kC, kC * 2);
      }
    }
    const int quad = warp & 3, hh = (warp >> 2) & 1;
    const int row = quad * 32 + lane;  // entry row within a tile / dim within a chunk
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t s_addr = lane_base + kColS + hh * 32;
    const float qscale = scale * kLog2e;
    uint32_t gphase = 0;
    float m_run = kNegInf;  // lane i: running max (log2 units) of head hh*32+i
    float lsum = 0.f;       // lane i: its head's sum of P over this warp's rows
    bool ok = true;
    for (int jt = 0; jt < ntile && ok; ++jt) {
      if (xfetch && jt == nw &&
          !(ok = fetch_list(list_ready + b, xlist + b * k, list, tile0 * kTE,
                            min(tile1 * kTE, nsel), err)))
        break;
      if (!(ok = gather_tile(jt))) break;
      if (!(ok = mbar_wait_small(&bar->s_full, (uint32_t)(jt & 1), err))) break;
      tc_fence_after();
      const bool valid = tile_at(jt) * kTE + row < N;
      float v[32];
      {
        uint32_t r[32];
        tmem_ld32(s_addr, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = valid ? __uint_as_float(r[i]) * qscale : kNegInf;
      }
      float* rmax = red + (hh * 4) * 32;
      rmax[quad * 32 + lane] = transpose_reduce<true>(v);
      if (!(ok = group_sync(&bar->grp[hh], gphase, err))) break;
      const float mtile = fmaxf(fmaxf(rmax[lane], rmax[32 + lane]),
                                fmaxf(rmax[64 + lane], rmax[96 + lane]));
      float f_lane = 1.f;
      bool resc = false;
      if (jt == 0) {
        m_run = mtile;
      } else if (mtile > m_run + kRescaleLog2) {
        resc = true;
        f_lane = ex2(m_run - mtile);
        m_run = mtile;
      }
      // rmax is rewritten next tile only after every warp of the group has read it
      if (!(ok = group_sync(&bar->grp[hh], gphase, err))) break;
      // P^T (and, for a rescale, O^T) is free once the previous P.V is done
      if (jt >= 1 && !(ok = mbar_wait_small(&bar->p_empty, (uint32_t)((jt - 1) & 1), err))) break;
      tc_fence_after();
      if (__any_sync(0xffffffffu, resc)) {
        float f[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          f[i] = __shfl_sync(0xffffffffu, f_lane, i);
        }
        lsum *= f_lane;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColO + c * kNH + hh * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f[i]);
          tmem_st32(lane_base + kColO + c * kNH + hh * 32, o);
        }
        tmem_st_wait();
      }
      uint32_t r[32];  // the logits again (cheaper than holding them across the reductions)
      tmem_ld32(s_addr, r);
      tmem_ld_wait();
      uint32_t pk[16];
      float ps[32];  // this tile's P of the thread's entry row, per head
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float ma = __shfl_sync(0xffffffffu, m_run, i);
        float mb = __shfl_sync(0xffffffffu, m_run, i + 1);
        ma = ma == kNegInf ? 0.f : ma;
        mb = mb == kNegInf ? 0.f : mb;
        const float la = valid ? __uint_as_float(r[i]) * qscale : kNegInf;
        const float lb = valid ? __uint_as_float(r[i + 1]) * qscale : kNegInf;
        const float pa = ex2(la - ma), pb = ex2(lb - mb);
        ps[i] = pa;
        ps[i + 1] = pb;
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
      lsum += transpose_reduce<false>(ps);  // (after P is handed over)
    }
    // ---- epilogue: this range's O^T, max and sum (or, alone, the output) ----------
    if (ok) ok = mbar_wait_small(&bar->o_full, 0, err);
    if (ok) {
      tc_fence_after();
      float* rsum = red + (2 * 4 + hh * 4) * 32;
      rsum[quad * 32 + lane] = lsum;
      ok = group_sync(&bar->grp[hh], gphase, err);
    }
    if (ok) {
      const int h = hh * 32 + lane;
      const float* rsum = red + (2 * 4 + hh * 4) * 32;
      const float tot = rsum[lane] + rsum[32 + lane] + rsum[64 + lane] + rsum[96 + lane];
      float inv = 1.f;
      if (direct) {
        const float mref = m_run == kNegInf ? 0.f : m_run;
        const float z = sink != nullptr ? sink[h] * kLog2e : kNegInf;
        inv = 1.f / (tot + (z == kNegInf ? 0.f : ex2(z - mref)));
      } else if (quad == 0) {
        part_ms[(pbase + h) * 2 + 0] = m_run;
        part_ms[(pbase + h) * 2 + 1] = tot;
      }
#pragma unroll 1
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
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

constexpr int kMaxCombine = 8;  // ranges whose partials are loaded together

// Merges the ranges of each sequence: o = sum_i 2^(m_i - M) O_i /
// (sum_i 2^(m_i - M) l_i + 2^(sink - M)).  One CTA per (head, sequence).
__global__ void __launch_bounds__(128) decode_combine_kernel(
    const float* __restrict__ part_o, const float* __restrict__ part_ms,
    const float* __restrict__ sink, int nsplit, __nv_bfloat16* __restrict__ out) {
  sm100::pdl_wait();  // the partials come from the previous kernel
  sm100::pdl_trigger();
  const int64_t b = blockIdx.y;
  const int h = blockIdx.x;
  const float z = sink != nullptr ? sink[h] * kLog2e : kNegInf;
  const int d0 = threadIdx.x * 4;
  // ranges in chunks of kMaxCombine, each chunk's max, sum and slice of O
  // in flight at once; the running max moves between chunks
  float M = z;
  float den = z == kNegInf ? 0.f : 1.f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int c0 = 0; c0 < nsplit; c0 += kMaxCombine) {
    float mi[kMaxCombine], li[kMaxCombine];
    float4 oi[kMaxCombine];
#pragma unroll
    for (int i = 0; i < kMaxCombine; ++i) {
      mi[i] = kNegInf;
      li[i] = 0.f;
      oi[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + i < nsplit) {
        const int64_t base = (b * nsplit + c0 + i) * kNH + h;
        mi[i] = part_ms[base * 2];
        li[i] = part_ms[base * 2 + 1];
        oi[i] = __ldcs(reinterpret_cast<const float4*>(part_o + base * kC + d0));
      }
    }
    float mc = kNegInf;
#pragma unroll
    for (int i = 0; i < kMaxCombine; ++i) mc = fmaxf(mc, mi[i]);
    if (mc > M) {  // rescale what is summed so far to the new max
      const float f = M == kNegInf ? 0.f : ex2(M - mc);
      den *= f;
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] *= f;
      M = mc;
    }
#pragma unroll
    for (int i = 0; i < kMaxCombine; ++i) {
      if (mi[i] == kNegInf) continue;
      const float wgt = ex2(mi[i] - M);
      den = fmaf(wgt, li[i], den);
      acc[0] = fmaf(wgt, oi[i].x, acc[0]);
      acc[1] = fmaf(wgt, oi[i].y, acc[1]);
      acc[2] = fmaf(wgt, oi[i].z, acc[2]);
      acc[3] = fmaf(wgt, oi[i].w, acc[3]);
    }
  }
  const float inv = 1.f / den;
  __nv_bfloat16* o = out + (b * kNH + h) * kC + d0;
  *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv),
                                            pack_bf16x2(acc[2] * inv, acc[3] * inv));
}

}  // namespace

bool decode_attn_tc_supported(const csa_cache_desc& d) {
  return d.nh == kNH && d.c == kC && d.rope_dims == kRope && (d.is_hca || d.k <= kMaxSelDec);
}

int decode_attn_splits(const csa_cache_desc& d) {
  const int64_t slots = (d.is_hca ? d.capacity : (int64_t)std::min<int64_t>(d.k, d.capacity)) +
                        d.window;
  const int64_t tmax = (slots + kTE - 1) / kTE;
  const int64_t per_sm = std::max<int64_t>(1, sm_count() / std::max<int64_t>(1, d.batch));
  return (int)std::max<int64_t>(1, std::min<int64_t>(tmax, per_sm));
}

bool decode_attn_selects(const csa_cache_desc& d) {
  return !d.is_hca && d.capacity + 8 <= kSelScores && d.k <= kMaxSelDec;
}

cudaError_t launch_decode_attn_tc(const csa_cache_desc& d, const CacheView& cv,
                                  const int64_t* pos, const void* q, const int32_t* sel,
                                  const float* sink, float scale, int nsplit, void* out,
                                  float* part_o, float* part_ms, const float* scores,
                                  const uint32_t* ghist, int32_t* sel_out,
                                  const uint32_t* idx_done, int idx_tile, int32_t* xlist,
                                  uint32_t* list_ready, unsigned int* err, cudaStream_t s) {
  CUtensorMap tq;
  if (!make_tmap_bf16_3d(&tq, q, kC, kNH, d.batch, kC * 2ull, (uint64_t)kNH * kC * 2, 64, kNH))
    return cudaErrorInvalidValue;
  auto kern = scores != nullptr ? decode_attn_tc_kernel<true> : decode_attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3((unsigned)nsplit, (unsigned)d.batch), dim3(kThreads),
                 (size_t)SMEM, s, tq, cv, pos, d.is_hca ? nullptr : sel, (int)d.k, (int)d.window,
                 (int)d.m, (int64_t)d.capacity, sink, scale, nsplit, part_o, part_ms,
                 (__nv_bfloat16*)out, scores, ghist, sel_out, idx_done, idx_tile, xlist,
                 list_ready, err);
  if (e != cudaSuccess || nsplit == 1) return e;
  return launch_pdl(decode_combine_kernel, dim3(kNH, (unsigned)d.batch), dim3(kC / 4), 0, s,
                    (const float*)part_o, (const float*)part_ms, sink, nsplit,
                    (__nv_bfloat16*)out);
}

}  // namespace csa
