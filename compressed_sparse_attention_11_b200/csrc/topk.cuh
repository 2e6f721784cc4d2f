// Block-wide exact top-k select (radix select, no sort), shared by the
// prefill top-k kernel and the decode candidate merge.
//
// Order: larger score first; among equal scores the earlier position wins.
// The chosen positions are emitted in ascending position order, which is the
// order the selection is compacted in, so no sort is needed.
#pragma once

#include "common.cuh"

namespace csa {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;

struct SelectShared {
  uint32_t hist[kSelWarps][256];
  uint32_t total[256];
  uint32_t warp_a[kSelWarps];
  uint32_t warp_b[kSelWarps];
  uint32_t digit, remaining;
};

// Key sources: key(i) is an unsigned key with the score order; 0 = never chosen.
struct KeysInSmem {
  const uint32_t* k;
  __device__ __forceinline__ uint32_t key(int64_t i) const { return k[i]; }
};
struct ScoresInGlobal {
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

// Selects the k largest keys among positions [0, V) (V > k) and writes, in
// ascending position order, out[j] = map ? map[pos] : pos.  All threads of a
// kSelThreads block must call it.
template <class Src>
__device__ void block_select_topk(const Src& src, int64_t V, int k, int32_t* __restrict__ out,
                                  const int32_t* __restrict__ map, SelectShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, mask = 0;
  if (tid == 0) sh.remaining = (uint32_t)k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < kSelWarps * 256; i += kSelThreads) (&sh.hist[0][0])[i] = 0;
    __syncthreads();
    for (int64_t i = tid; i < V; i += kSelThreads) {
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
    if (tid < 256) {
      uint32_t s = 0;
#pragma unroll
      for (int w = 0; w < kSelWarps; ++w) s += sh.hist[w][tid];
      sh.total[tid] = s;
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
  const uint32_t T = prefix;             // key of the k-th largest element
  const uint32_t take_eq = sh.remaining; // how many elements equal to T are chosen

  // contiguous segment per warp, a multiple of 32 long
  const int64_t seg = ((V + kSelWarps - 1) / kSelWarps + 31) / 32 * 32;
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

}  // namespace csa
