// Decode top-k: the k entries with the largest indexer score among the V
// visible entries of each sequence (the selection step of sections 4.2 / 4.3
// of "DeepSeek-V4: million-token context"; ties to the smaller index, the
// chosen indices listed ascending; all V entries when V <= k).
//
// The indexer kernel leaves, next to the scores, a histogram of each
// sequence's scores over the top 12 bits of their order keys (unsigned
// integers whose order is the float order).  That fixes, before any score is
// read again, the bin T where the count from the top reaches k: every score
// in a higher bin is chosen, none in a lower one, and only the few scores in
// bin T need ranking.  So the selection is one pass over the scores, spread
// over many CTAs, plus a small exact step:
//   * CTA (j, b) takes slice j (4096 scores) of sequence b: it marks the
//     chosen scores of the slice in a bitmap (one bit per entry) and copies
//     the slice's bin-T scores, in index order, to the slice's candidate area;
//   * the last CTA to finish a sequence (an atomic count of finished slices;
//     no CTA waits for another) gathers the candidates in index order, finds
//     among them the `need` = k - (count above bin T) largest by the same
//     order (radix select, ties to the earlier position = the smaller index),
//     marks them in the bitmap and writes the chosen indices in ascending
//     order from the bitmap.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"
#include "topk.cuh"

namespace csa {

namespace {

constexpr int kThreads = 256;
constexpr int kPer = 16;                   // scores per thread
constexpr int kSlice = kThreads * kPer;    // 4096 scores per CTA
constexpr int kBins = kDecHistBins;        // 4096
constexpr int kBinsPerThread = kBins / kThreads;  // 16
constexpr int kSmemCand = 2048;            // threshold-bin candidates staged in shared memory
constexpr int kMaxSmemWords = 45056;       // bitmap words stageable in shared memory (1,441,792 entries)
static_assert(kBins % kThreads == 0 && kSlice % 32 == 0, "shapes");

struct KeysInGlobal {
  const uint32_t* k;
  __device__ __forceinline__ uint32_t key(int64_t i) const { return __ldcg(k + i); }
};

struct __align__(16) SelShared {
  SelectShared<kThreads> sel;
  uint32_t wsum[kThreads / 32];
  uint32_t T, G, CT;
  uint32_t last;
  uint32_t slice_off[kDecMaxSlices + 1];
};

// Block-wide exclusive prefix of v (every thread gets its own and the total).
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wsum, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += x;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  uint32_t before = 0;
  total = 0;
  for (int w = 0; w < kThreads / 32; ++w) {
    if (w < warp) before += wsum[w];
    total += wsum[w];
  }
  __syncthreads();
  return before + inc - v;
}

__global__ void __launch_bounds__(kThreads, 4) decode_topk_hist_kernel(
    const int64_t* __restrict__ pos, int64_t cap, int m, int k, const float* __restrict__ scores,
    DecodeSelectWs ws, int32_t* __restrict__ sel, int smem_words) {
  __shared__ SelShared sh;
  // [kSmemCand] keys, [kSmemCand] indices, [smem_words] bitmap words
  extern __shared__ __align__(16) uint32_t dyn_smem[];
  uint32_t* dyn_key = dyn_smem;
  int32_t* dyn_idx = reinterpret_cast<int32_t*>(dyn_smem + kSmemCand);
  uint32_t* dyn_bm = dyn_smem + 2 * kSmemCand;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = blockIdx.x;
  const int64_t b = blockIdx.y;

  const int64_t t = pos[b];  // an input of the step: read before the wait
  sm100::pdl_wait();         // the scores and the histogram come from the indexer
  sm100::pdl_trigger();
  const int64_t V = t < 0 ? 0 : min((t + 1) / m, cap);
  int32_t* out = sel + b * k;
  if (V <= k) {  // every visible entry
    if (j == 0)
      for (int i = tid; i < k; i += kThreads) out[i] = i < V ? i : -1;
    return;
  }
  const int64_t lo = (int64_t)j * kSlice;
  if (lo >= V) return;  // past the sequence's last slice (not counted below)
  const int nsl = (int)((V + kSlice - 1) / kSlice);

  // this thread's 16 scores start loading now, under the histogram scan
  const int64_t s0 = lo + (int64_t)tid * kPer;
  const float* row = scores + b * cap;
  uint32_t keys[kPer];  // (rows are `cap` floats apart: no vector loads)
#pragma unroll
  for (int i = 0; i < kPer; ++i) keys[i] = s0 + i < V ? order_key(__ldcg(row + s0 + i)) : 0u;

  // 1. the bin T where the count from the top reaches k (thread tid owns
  //    bins 4095 - 16 tid - i, i = 0 .. 15, i.e. descending)
  if (tid == 0) {  // (a histogram that cannot reach k leaves a defined, capped result)
    sh.T = 0u;
    sh.G = 0u;
    sh.CT = 0u;
  }
  {
    const uint32_t* gh = ws.ghist + b * kBins;
    uint32_t c[kBinsPerThread], loc = 0;
#pragma unroll
    for (int i = 0; i < kBinsPerThread; ++i) {
      c[i] = __ldcg(gh + kBins - 1 - (tid * kBinsPerThread + i));
      loc += c[i];
    }
    uint32_t total;
    uint32_t acc = block_excl_scan(loc, sh.wsum, total);
#pragma unroll
    for (int i = 0; i < kBinsPerThread; ++i) {
      if (acc < (uint32_t)k && acc + c[i] >= (uint32_t)k) {
        sh.T = (uint32_t)(kBins - 1 - (tid * kBinsPerThread + i));
        sh.G = acc;
        sh.CT = c[i];
      }
      acc += c[i];
    }
    __syncthreads();
  }
  const uint32_t T = sh.T, G = sh.G, CT = sh.CT;
  const uint32_t need = (uint32_t)k - G;
  const bool all_of_T = CT == need;  // bin T is taken whole: no candidates

  // 2. classify this thread's 16 scores (loaded above): chosen outright, or a
  //    bin-T candidate
  uint32_t strict = 0, cand = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    if (s0 + i < V) {
      const uint32_t bin = keys[i] >> kDecHistShift;
      if (bin > T || (all_of_T && bin == T)) strict |= 1u << i;
      else if (bin == T) cand |= 1u << i;
    }
  }
  // two threads make one bitmap word (lo half: the even thread)
  const uint32_t other = __shfl_xor_sync(0xffffffffu, strict, 1);
  if ((lane & 1) == 0) __stcg(ws.bitmap + b * ws.words + (s0 >> 5), strict | (other << 16));
  uint32_t ncand = 0;
  const uint32_t off = block_excl_scan((uint32_t)__popc(cand), sh.wsum, ncand);
  {
    uint32_t* ck = ws.cand_key + b * cap + lo;
    int32_t* ci = ws.cand_idx + b * cap + lo;
    uint32_t p = off;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (cand & (1u << i)) {
        __stcg(ck + p, keys[i]);
        __stcg(ci + p, (int32_t)(s0 + i));
        ++p;
      }
  }
  if (tid == 0) __stcg(ws.cand_cnt + b * kDecMaxSlices + j, ncand);

  // 3. the last CTA of the sequence finishes it
  __threadfence();
  __syncthreads();
  if (tid == 0) sh.last = atomicAdd(ws.done + b, 1u) == (uint32_t)(nsl - 1) ? 1u : 0u;
  __syncthreads();
  if (sh.last == 0u) return;
  __threadfence();

  // the sequence's bitmap into shared memory when it fits (loads issued now,
  // under the candidate bookkeeping)
  const int64_t nwords = (V + 31) / 32;
  const bool bm_smem = nwords <= smem_words;
  uint32_t* bmg = ws.bitmap + b * ws.words;
  uint32_t* bm = bm_smem ? dyn_bm : bmg;
  if (bm_smem) {  // every load in flight at once (rows of words are 512-byte aligned)
    const int nchunk = (int)((nwords + 3) / 4);
    for (int c = tid; c < nchunk; c += kThreads)
      sm100::cp_async_16(sm100::smem_u32(dyn_bm) + 16u * c, bmg + 4 * c);
  }

  if (!all_of_T) {
    // the candidates of every slice, in index order, into one array: shared
    // memory when they fit (the usual case: bin T holds a few hundred to a
    // couple of thousand scores), else the global gather area
    if (warp == 0) {  // slice offsets: a shuffle scan, lane l owns slices l, l + 32, ..
      uint32_t run = 0;
      for (int q0 = 0; q0 < nsl; q0 += 32) {
        const int q = q0 + lane;
        const uint32_t c = q < nsl ? __ldcg(ws.cand_cnt + b * kDecMaxSlices + q) : 0u;
        uint32_t inc = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t x = __shfl_up_sync(0xffffffffu, inc, off);
          if (lane >= off) inc += x;
        }
        if (q < nsl) sh.slice_off[q] = run + inc - c;
        run += __shfl_sync(0xffffffffu, inc, 31);
      }
      if (lane == 0) sh.slice_off[nsl] = run;
    }
    __syncthreads();
    const uint32_t C = sh.slice_off[nsl];
    const bool in_smem = C <= (uint32_t)kSmemCand;
    uint32_t* cck = in_smem ? dyn_key : ws.cc_key + b * cap;
    int32_t* cci = in_smem ? dyn_idx : ws.cc_idx + b * cap;
    for (int q = warp; q < nsl; q += kThreads / 32) {
      const uint32_t base = sh.slice_off[q], n = sh.slice_off[q + 1] - base;
      const uint32_t* ck = ws.cand_key + b * cap + (int64_t)q * kSlice;
      const int32_t* ci = ws.cand_idx + b * cap + (int64_t)q * kSlice;
      for (uint32_t i = lane; i < n; i += 32) {
        if (in_smem) {  // 4-byte copies, all in flight
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sm100::smem_u32(cck + base + i)),
                       "l"(ck + i)
                       : "memory");
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sm100::smem_u32(cci + base + i)),
                       "l"(ci + i)
                       : "memory");
        } else {
          __stcg(cck + base + i, __ldcg(ck + i));
          __stcg(cci + base + i, __ldcg(ci + i));
        }
      }
    }
    sm100::cp_async_wait_all();  // (the bitmap's copies too)
    __threadfence_block();
    __syncthreads();
    // the need largest of them (ties: the earlier position, i.e. the smaller
    // index), marked in the bitmap
    uint32_t Tk = 0u, take_eq = 0u;
    const bool all = need >= C;
    if (!all) {
      if (in_smem)
        radix_kth<kThreads>(KeysInSmem{cck}, C, (int)need, sh.sel, Tk, take_eq);
      else
        radix_kth<kThreads>(KeysInGlobal{cck}, C, (int)need, sh.sel, Tk, take_eq);
    }
    // (plain loads through the chosen pointer: a select between a shared and
    // an L2 load would issue both, and wait for the L2 one, every time)
    auto key_at = [&](int64_t i) { return cck[i]; };
    const int64_t seg = ((C + kThreads / 32 - 1) / (kThreads / 32) + 31) / 32 * 32;
    const int64_t plo = (int64_t)warp * seg, phi = min((int64_t)C, plo + seg);
    uint32_t eq = 0;
    for (int64_t base = plo; base < phi; base += 32) {
      const int64_t i = base + lane;
      eq += __popc(__ballot_sync(0xffffffffu, i < phi && !all && key_at(i) == Tk));
    }
    if (lane == 0) sh.sel.warp_b[warp] = eq;
    __syncthreads();
    uint32_t eq_before = 0;
    for (int w = 0; w < warp; ++w) eq_before += sh.sel.warp_b[w];
    const uint32_t lt = (1u << lane) - 1u;
    for (int64_t base = plo; base < phi; base += 32) {
      const int64_t i = base + lane;
      const uint32_t key = i < phi ? key_at(i) : 0u;
      const bool is_eq = i < phi && !all && key == Tk;
      const uint32_t em = __ballot_sync(0xffffffffu, is_eq);
      const bool take = i < phi && (all || key > Tk || (is_eq && eq_before + __popc(em & lt) < take_eq));
      if (take) {
        const int32_t s = cci[i];
        atomicOr(bm + (s >> 5), 1u << (s & 31));
      }
      eq_before += __popc(em);
    }
    if (!bm_smem) __threadfence();
  }
  sm100::cp_async_wait_all();
  __syncthreads();

  // 4. the chosen indices in ascending order, from the bitmap: warp w takes
  //    a contiguous run of words, 128 words a step with lane l on words
  //    4l .. 4l+3 (one 16-byte access per lane); counts first, then, from
  //    the warps' offsets, the indices
  constexpr int kWarps = kThreads / 32;
  const int64_t seg = ((nwords + kWarps - 1) / kWarps + 127) / 128 * 128;
  const int64_t ws0 = min(nwords, (int64_t)warp * seg), ws1 = min(nwords, ws0 + seg);
  auto quad = [&](int64_t w) -> uint4 {  // words w .. w+3 (w a multiple of 4), zero past ws1
    if (w + 4 <= ws1) return *reinterpret_cast<const uint4*>(bm + w);
    uint4 q = make_uint4(0u, 0u, 0u, 0u);
    if (w < ws1) q.x = bm[w];
    if (w + 1 < ws1) q.y = bm[w + 1];
    if (w + 2 < ws1) q.z = bm[w + 2];
    return q;
  };
  uint32_t cnt = 0;
#pragma unroll 2
  for (int64_t w = ws0 + 4 * lane; w < ws1; w += 128) {
    const uint4 q = quad(w);
    cnt += __popc(q.x) + __popc(q.y) + __popc(q.z) + __popc(q.w);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
  if (lane == 0) sh.wsum[warp] = cnt;
  __syncthreads();
  uint32_t o = 0, total = 0;
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) o += sh.wsum[w];
    total += sh.wsum[w];
  }
#pragma unroll 1
  for (int64_t base = ws0; base < ws1; base += 128) {
    const int64_t w = base + 4 * lane;
    const uint4 q = quad(w);
    const uint32_t wd[4] = {q.x, q.y, q.z, q.w};
    const uint32_t c = __popc(q.x) + __popc(q.y) + __popc(q.z) + __popc(q.w);
    uint32_t inc = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += y;
    }
    uint32_t p = o + inc - c;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint32_t x = wd[e];
      while (x != 0u) {
        const int bit = __ffs(x) - 1;
        x &= x - 1u;
        if (p < (uint32_t)k) out[p] = (int32_t)((w + e) * 32 + bit);
        ++p;
      }
    }
    o += __shfl_sync(0xffffffffu, inc, 31);
  }
  for (uint32_t i = total + tid; i < (uint32_t)k; i += kThreads) out[i] = -1;  // (total == k)
}

}  // namespace

bool decode_select_supported(const csa_cache_desc& d) {
  return !d.is_hca && (d.capacity + kSlice - 1) / kSlice <= kDecMaxSlices;
}

DecodeSelectWs decode_select_ws(const csa_cache_desc& d, uint8_t* base, size_t* bytes) {
  DecodeSelectWs w = {};
  const size_t B = (size_t)d.batch, cap = (size_t)d.capacity;
  w.words = (int64_t)((cap + kSlice - 1) / kSlice * (kSlice / 32));
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t o = off;
    off = (off + n + 255) & ~(size_t)255;
    return o;
  };
  const size_t o_gh = take(B * kBins * 4), o_done = take(B * 4), o_idone = take(B * 4),
               o_lready = take(B * 4),
               o_bm = take(B * w.words * 4),
               o_ck = take(B * cap * 4), o_ci = take(B * cap * 4),
               o_cnt = take(B * kDecMaxSlices * 4), o_cck = take(B * cap * 4),
               o_cci = take(B * cap * 4);
  *bytes = off;
  if (base != nullptr) {
    w.ghist = reinterpret_cast<uint32_t*>(base + o_gh);
    w.done = reinterpret_cast<uint32_t*>(base + o_done);
    w.idx_done = reinterpret_cast<uint32_t*>(base + o_idone);
    w.list_ready = reinterpret_cast<uint32_t*>(base + o_lready);
    w.bitmap = reinterpret_cast<uint32_t*>(base + o_bm);
    w.cand_key = reinterpret_cast<uint32_t*>(base + o_ck);
    w.cand_idx = reinterpret_cast<int32_t*>(base + o_ci);
    w.cand_cnt = reinterpret_cast<uint32_t*>(base + o_cnt);
    w.cc_key = reinterpret_cast<uint32_t*>(base + o_cck);
    w.cc_idx = reinterpret_cast<int32_t*>(base + o_cci);
  }
  return w;
}

cudaError_t launch_decode_select(const csa_cache_desc& d, const int64_t* pos, const float* scores,
                                 const DecodeSelectWs& ws, int32_t* sel, cudaStream_t s) {
  const unsigned nsl = (unsigned)((d.capacity + kSlice - 1) / kSlice);
  if (nsl > (unsigned)kDecMaxSlices) return cudaErrorInvalidValue;
  // the bitmap of a whole sequence in shared memory when it fits the limit
  const int64_t words = ((d.capacity + 31) / 32 + 3) / 4 * 4;
  const int smem_words = (int)std::min<int64_t>(words, kMaxSmemWords);
  const size_t kDyn = (size_t)kSmemCand * 8 + (size_t)smem_words * 4;
  const cudaError_t e = cudaFuncSetAttribute(decode_topk_hist_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDyn);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_topk_hist_kernel, dim3(nsl, (unsigned)d.batch), dim3(kThreads), kDyn, s,
                    pos, (int64_t)d.capacity, d.m, d.k, scores, ws, sel, smem_words);
}

}  // namespace csa
