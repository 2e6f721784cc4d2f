// Block-wide exact top-k select (radix select, no sort), shared by the
// prefill top-k kernel and the decode selection.
//
// Order: larger score first; among equal scores the earlier position wins.
// The chosen positions are emitted in ascending position order, which is the
// order the selection is compacted in, so no sort is needed.
//
// Three front ends:
//   block_select_topk          radix select over all V keys (4 histogram
//                              passes + 2 compaction passes);
//   block_select_topk_sampled  estimates a threshold from a strided sample,
//                              keeps the (few) keys at or above it in order,
//                              and runs the exact radix select on those only
//                              -- two passes over V instead of six;
//   block_select_topk_ranked   the same, but the sample and the kept keys are
//                              ranked by direct comparison counts, which costs
//                              a few block barriers instead of dozens.
// The sampled front ends fall back to the full select when the estimate
// keeps fewer than k or too many keys.
#pragma once

#include "common.cuh"

namespace csa {

template <int NT>
struct SelectShared {
  static constexpr int kWarps = NT / 32;
  uint32_t hist[kWarps][256];
  uint32_t total[256];
  uint32_t warp_a[kWarps];
  uint32_t warp_b[kWarps];
  uint32_t digit, remaining;
};

// Key sources: key(i) is an unsigned key with the score order; 0 = never chosen.
struct KeysInSmem {
  const uint32_t* k;
  __device__ __forceinline__ uint32_t key(int64_t i) const { return k[i]; }
};
struct ScoresIn {
  const float* s;
  __device__ __forceinline__ uint32_t key(int64_t i) const { return order_key(s[i]); }
};
struct CandidatesInGlobal {  // (score, index) pairs; index < 0 is padding
  const float* s;
  const int32_t* id;
  __device__ __forceinline__ uint32_t key(int64_t i) const {
    return id[i] < 0 ? 0u : order_key(s[i]);
  }
};
template <class Src>
struct Gathered {  // keys of positions pos[0..)
  Src src;
  const int32_t* pos;
  __device__ __forceinline__ uint32_t key(int64_t i) const { return src.key(pos[i]); }
};

// Radix search for the key T of the k-th largest element among [0, V)
// (1 <= k <= V) and the number of elements equal to T inside the top k.
template <int NT, class Src>
__device__ void radix_kth(const Src& src, int64_t V, int k, SelectShared<NT>& sh, uint32_t& T,
                          uint32_t& take_eq) {
  constexpr int W = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, mask = 0;
  if (tid == 0) sh.remaining = (uint32_t)k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < W * 256; i += NT) (&sh.hist[0][0])[i] = 0;
    __syncthreads();
    for (int64_t i = tid; i < V; i += NT) {
      const uint32_t u = src.key(i);
      const bool in = (u & mask) == prefix;
      const uint32_t dig = (u >> shift) & 255u;
      // aggregate equal digits inside the warp before touching shared memory
      const uint32_t act = __ballot_sync(__activemask(), in);
      if (in) {
        const uint32_t peers = __match_any_sync(act, dig);
        if ((peers & ((1u << lane) - 1u)) == 0) atomicAdd(&sh.hist[warp][dig], __popc(peers));
      }
    }
    __syncthreads();
    for (int d = tid; d < 256; d += NT) {
      uint32_t s = 0;
#pragma unroll
      for (int w = 0; w < W; ++w) s += sh.hist[w][d];
      sh.total[d] = s;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns bins 255-8l-7 .. 255-8l (lane 0 the top bins)
      const uint32_t rem = sh.remaining;  // read before any lane rewrites it
      uint32_t cnt[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { cnt[j] = sh.total[255 - 8 * lane - j]; sum += cnt[j]; }
      uint32_t incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      const uint32_t above = incl - sum;  // elements in higher bins
      __syncwarp();
      if (above < rem && rem <= incl) {
        uint32_t acc = above;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (acc < rem && rem <= acc + cnt[j]) {
            sh.digit = 255u - 8u * lane - j;
            sh.remaining = rem - acc;
          }
          acc += cnt[j];
        }
      }
    }
    __syncthreads();
    prefix |= sh.digit << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  T = prefix;
  take_eq = sh.remaining;
  __syncthreads();
}

// Writes, in ascending position order, out[j] = map ? map[pos] : pos for the
// positions whose key is > T, plus the first take_eq positions whose key == T.
template <int NT, class Src>
__device__ void emit_selected(const Src& src, int64_t V, uint32_t T, uint32_t take_eq, int k,
                              int32_t* __restrict__ out, const int32_t* __restrict__ map,
                              SelectShared<NT>& sh) {
  constexpr int W = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t seg = ((V + W - 1) / W + 31) / 32 * 32;  // contiguous per warp
  const int64_t lo = (int64_t)warp * seg, hi = min(V, lo + seg);
  uint32_t gt = 0, eq = 0;
  for (int64_t base = lo; base < hi; base += 32) {
    const int64_t i = base + lane;
    const uint32_t u = i < hi ? src.key(i) : 0u;
    gt += __popc(__ballot_sync(0xffffffffu, i < hi && u > T));
    eq += __popc(__ballot_sync(0xffffffffu, i < hi && u == T));
  }
  if (lane == 0) { sh.warp_a[warp] = gt; sh.warp_b[warp] = eq; }
  __syncthreads();
  uint32_t eq_before = 0, sel_before = 0;
  for (int w = 0; w < warp; ++w) {
    const uint32_t e = sh.warp_b[w];
    const uint32_t take = eq_before >= take_eq ? 0u : min(e, take_eq - eq_before);
    sel_before += sh.warp_a[w] + take;
    eq_before += e;
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t run_eq = eq_before, run_sel = sel_before;
  for (int64_t base = lo; base < hi; base += 32) {
    const int64_t i = base + lane;
    const uint32_t u = i < hi ? src.key(i) : 0u;
    const bool is_gt = i < hi && u > T;
    const bool is_eq = i < hi && u == T;
    const uint32_t eq_mask = __ballot_sync(0xffffffffu, is_eq);
    const bool take = is_gt || (is_eq && run_eq + __popc(eq_mask & lt_mask) < take_eq);
    const uint32_t sel_mask = __ballot_sync(0xffffffffu, take);
    if (take) {
      const uint32_t p = run_sel + __popc(sel_mask & lt_mask);
      if (p < (uint32_t)k) out[p] = map ? map[i] : (int32_t)i;
    }
    run_eq += __popc(eq_mask);
    run_sel += __popc(sel_mask);
  }
  __syncthreads();
}

// Selects the k largest keys among positions [0, V) (V >= k) and writes, in
// ascending position order, out[j] = map ? map[pos] : pos.  All NT threads
// of the block must call it.
template <int NT, class Src>
__device__ void block_select_topk(const Src& src, int64_t V, int k, int32_t* __restrict__ out,
                                  const int32_t* __restrict__ map, SelectShared<NT>& sh) {
  uint32_t T, take_eq;
  radix_kth<NT>(src, V, k, sh, T, take_eq);
  emit_selected<NT>(src, V, T, take_eq, k, out, map, sh);
}

// Same result as block_select_topk (positions, no map).  `cand` is scratch
// for up to `cap` positions and `sample` for `nsample` keys, both owned by
// the block (shared or global memory).
template <int NT, class Src>
__device__ void block_select_topk_sampled(const Src& src, int64_t V, int k,
                                          int32_t* __restrict__ out, SelectShared<NT>& sh,
                                          int32_t* __restrict__ cand, int cap,
                                          uint32_t* __restrict__ sample, int nsample) {
  constexpr int W = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (V <= (int64_t)cap || nsample < 64) {
    block_select_topk<NT>(src, V, k, out, nullptr, sh);
    return;
  }
  // 1. threshold from a strided sample: about 1.5x the wanted share, + 16
  const int S = nsample;
  for (int i = tid; i < S; i += NT) sample[i] = src.key((V * (int64_t)i) / S);
  __syncthreads();
  const int r = min(S, (int)((1.5 * S * (double)k) / (double)V) + 16);
  uint32_t T0, unused;
  radix_kth<NT>(KeysInSmem{sample}, S, r, sh, T0, unused);
  // 2. count the keys >= T0 (per warp over a contiguous segment)
  const int64_t seg = ((V + W - 1) / W + 31) / 32 * 32;
  const int64_t lo = (int64_t)warp * seg, hi = min(V, lo + seg);
  uint32_t c = 0;
  for (int64_t base = lo; base < hi; base += 32) {
    const int64_t i = base + lane;
    c += __popc(__ballot_sync(0xffffffffu, i < hi && src.key(i) >= T0));
  }
  if (lane == 0) sh.warp_a[warp] = c;
  __syncthreads();
  uint32_t before = 0, total = 0;
  for (int w = 0; w < W; ++w) {
    const uint32_t x = sh.warp_a[w];
    if (w < warp) before += x;
    total += x;
  }
  __syncthreads();
  if (total < (uint32_t)k || total > (uint32_t)cap) {  // the estimate missed: exact path
    block_select_topk<NT>(src, V, k, out, nullptr, sh);
    return;
  }
  // 3. keep those positions in order, then the exact select among them
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t run = before;
  for (int64_t base = lo; base < hi; base += 32) {
    const int64_t i = base + lane;
    const bool keep = i < hi && src.key(i) >= T0;
    const uint32_t msk = __ballot_sync(0xffffffffu, keep);
    if (keep) cand[run + __popc(msk & lt_mask)] = (int32_t)i;
    run += __popc(msk);
  }
  __syncthreads();
  // candidates are in ascending position order: emitting the chosen slots in
  // order and mapping each slot to its position keeps the output ascending
  block_select_topk<NT>(Gathered<Src>{src, cand}, total, k, out, cand, sh);
}

// Rank of element i among n keys (larger first, ties to the smaller index).
__device__ __forceinline__ uint32_t rank_in(const uint32_t* __restrict__ keys, int n, int i) {
  const uint32_t ki = keys[i];
  uint32_t r = 0;
  for (int j = 0; j < n; ++j) {
    const uint32_t kj = keys[j];
    r += (kj > ki || (kj == ki && j < i)) ? 1u : 0u;
  }
  return r;
}

// Same result as block_select_topk (positions, no map), for k <= V.  A strided
// sample of S keys is ranked exactly to pick a threshold somewhat below the
// k-th largest; one pass keeps the keys at or above it (in position order);
// those are ranked exactly when there are at most `rank_max`, radix-selected
// otherwise.  Scratch: skey / spos hold `cap` entries (shared memory).
template <int NT, class Src>
__device__ void block_select_topk_ranked(const Src& src, int64_t V, int k,
                                         int32_t* __restrict__ out, SelectShared<NT>& sh,
                                         uint32_t* __restrict__ skey, int32_t* __restrict__ spos,
                                         int cap, int rank_max) {
  constexpr int W = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t C;
  if (V <= (int64_t)rank_max) {  // small: every key is a candidate
    for (int i = tid; i < V; i += NT) {
      skey[i] = src.key(i);
      spos[i] = i;
    }
    C = (uint32_t)V;
    __syncthreads();
  } else {
    // 1. threshold: the r-th largest of a strided sample
    const int S = (int)min(V, (int64_t)(V > 65536 ? 2048 : 1024));
    const int r = (int)min((int64_t)S, (3 * (int64_t)S * k) / (2 * V) + 12);
    for (int i = tid; i < S; i += NT) skey[i] = src.key((V * (int64_t)i) / S);
    if (tid == 0) sh.digit = 0;
    __syncthreads();
    for (int i = tid; i < S; i += NT)
      if (rank_in(skey, S, i) == (uint32_t)(r - 1)) sh.digit = skey[i];
    __syncthreads();
    const uint32_t T0 = sh.digit;
    // 2. count and keep the keys >= T0, per warp over a contiguous segment
    const int64_t seg = ((V + W - 1) / W + 31) / 32 * 32;
    const int64_t lo = (int64_t)warp * seg, hi = min(V, lo + seg);
    uint32_t c = 0;
    for (int64_t base = lo; base < hi; base += 32) {
      const int64_t i = base + lane;
      c += __popc(__ballot_sync(0xffffffffu, i < hi && src.key(i) >= T0));
    }
    if (lane == 0) sh.warp_a[warp] = c;
    __syncthreads();
    uint32_t before = 0;
    C = 0;
    for (int w = 0; w < W; ++w) {
      if (w < warp) before += sh.warp_a[w];
      C += sh.warp_a[w];
    }
    __syncthreads();
    if (C < (uint32_t)k || C > (uint32_t)cap) {  // the estimate missed: exact path
      block_select_topk<NT>(src, V, k, out, nullptr, sh);
      return;
    }
    uint32_t run = before;
    for (int64_t base = lo; base < hi; base += 32) {
      const int64_t i = base + lane;
      const uint32_t key = i < hi ? src.key(i) : 0u;
      const bool keep = i < hi && key >= T0;
      const uint32_t msk = __ballot_sync(0xffffffffu, keep);
      if (keep) {
        const uint32_t p = run + __popc(msk & lt);
        skey[p] = key;
        spos[p] = (int32_t)i;
      }
      run += __popc(msk);
    }
    __syncthreads();
    if (C > (uint32_t)rank_max) {
      block_select_topk<NT>(KeysInSmem{skey}, C, k, out, spos, sh);
      return;
    }
  }
  // 3. exact ranks among the candidates; contiguous candidates per thread
  //    keep the output in ascending position order
  const int per = (int)((C + NT - 1) / NT);
  const int lo = min((int)C, tid * per), hi = min((int)C, lo + per);
  uint32_t mine = 0;
  for (int i = lo; i < hi; ++i) mine += rank_in(skey, C, i) < (uint32_t)k ? 1u : 0u;
  uint32_t inc = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += v;
  }
  if (lane == 31) sh.warp_b[warp] = inc;
  __syncthreads();
  uint32_t o = inc - mine;
  for (int w = 0; w < warp; ++w) o += sh.warp_b[w];
  for (int i = lo; i < hi; ++i)
    if (rank_in(skey, C, i) < (uint32_t)k && o < (uint32_t)k) out[o++] = spos[i];
  __syncthreads();
}

}  // namespace csa
