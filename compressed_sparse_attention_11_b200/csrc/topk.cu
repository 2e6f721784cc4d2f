// Prefill top-k: one block per query row selects the k best of its V(t)
// visible index scores (section 4.2 step 4 of "DeepSeek-V4: million-token
// context"; ties to the smaller entry index; indices ascending, -1 padded).
#include "launch.h"
#include "topk.cuh"

namespace csa {

constexpr int kSelThreads = 512;
constexpr int64_t kSelSmemKeys = 32768;  // rows up to this long are staged in shared memory
constexpr int kSelCap = 4096;            // candidates kept above the sampled threshold
constexpr int kSelSample = 2048;         // sample size of the threshold estimate

__global__ void __launch_bounds__(kSelThreads) topk_rows_kernel(
    const float* __restrict__ scores, int64_t ld, int64_t n, int m, int64_t E, int k,
    int64_t smem_keys, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelectShared<kSelThreads>& sh = *reinterpret_cast<SelectShared<kSelThreads>*>(smem_raw);
  int32_t* cand = reinterpret_cast<int32_t*>(smem_raw + sizeof(SelectShared<kSelThreads>));
  uint32_t* sample = reinterpret_cast<uint32_t*>(cand + kSelCap);
  uint32_t* keys = sample + kSelSample;
  const int64_t t = blockIdx.x, b = blockIdx.y;
  const int64_t V = min((t + 1) / m, E);
  int32_t* out = idx + (b * n + t) * k;
  if (V <= k) {
    for (int j = threadIdx.x; j < k; j += kSelThreads) out[j] = j < V ? j : -1;
    return;
  }
  const float* row = scores + (b * n + t) * ld;
  if (V <= smem_keys) {
    for (int64_t i = threadIdx.x; i < V; i += kSelThreads) keys[i] = order_key(row[i]);
    __syncthreads();
    block_select_topk_sampled<kSelThreads>(KeysInSmem{keys}, V, k, out, sh, cand, kSelCap,
                                           sample, kSelSample);
  } else {
    block_select_topk_sampled<kSelThreads>(ScoresIn{row}, V, k, out, sh, cand, kSelCap, sample,
                                           kSelSample);
  }
}

// ---------------------------------------------------------------------------
// One CTA per row, the row staged in shared memory as order keys (unsigned
// integers with the float order).  One radix pass histograms the keys into
// 2048 bins spanning [min, max] of the row; the bin T where the count from
// the top reaches k decides: keys above T are chosen, and the keys of bin T
// (few, when the bins are fine enough) are ranked among themselves by (key
// descending, index ascending) to give the exact cut (key, index) of the
// k-th choice.  A crowded bin T narrows the window to that bin with 2048x
// finer bins and repeats.  The chosen indices are written in ascending order
// by warps over contiguous segments.  About eight block barriers per row.
// ---------------------------------------------------------------------------
constexpr int kRowThreads = 512;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kRowBins = 2048;
constexpr int kRowBinBits = 11;
constexpr int kRowBinsPerThread = kRowBins / kRowThreads;  // 4
constexpr int kRowCand = 256;                              // bin-T keys ranked directly (3 CTAs per SM at 16K keys)
constexpr int64_t kRowMaxKeys = 32768;                     // keys staged per row
// 32-key groups of one warp's compaction segment (two masks each in the histogram)
constexpr int kRowMaxGroups = (int)((kRowMaxKeys / kRowWarps + 31) / 32);
static_assert(2 * kRowMaxGroups * kRowWarps <= kRowBins, "masks fit in the histogram");

struct __align__(16) RowTopkShared {
  uint32_t hist[kRowBins];
  uint32_t cand_key[kRowCand];
  int32_t cand_pos[kRowCand];
  uint32_t wred[2][kRowWarps];
  uint32_t wcnt[kRowWarps];
  uint32_t T, G, C, cand_n, cut_key;
  int32_t cut_pos;
};

__device__ __forceinline__ uint32_t bit_length(uint32_t x) { return x == 0 ? 0u : 32u - __clz(x); }

// ST: float, or __nv_bfloat16 for scores stored in bf16 (each widened to fp32
// exactly, so the order and the ties are those of the bf16 values).
template <typename ST>
__global__ void __launch_bounds__(kRowThreads) topk_rows_staged_kernel(
    const ST* __restrict__ scores, int64_t ld, int64_t n, int m, int64_t E, int k,
    int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  RowTopkShared& sh = *reinterpret_cast<RowTopkShared*>(smem_raw);
  uint32_t* key = reinterpret_cast<uint32_t*>(smem_raw + sizeof(RowTopkShared));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t = blockIdx.x, b = blockIdx.y;
  const int V = (int)min((t + 1) / m, E);
  int32_t* out = idx + (b * n + t) * k;
  if (V <= k) {
    for (int j = tid; j < k; j += kRowThreads) out[j] = j < V ? j : -1;
    return;
  }
  // 1. the row as order keys, with its key range
  const ST* row = scores + (b * n + t) * ld;
  uint32_t mn = 0xffffffffu, mx = 0u;
  if (sizeof(ST) == 4 && (ld & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0) {
    // 16-byte rows: the whole row lands in shared memory in one round trip
    // (cp.async, zero past V), then becomes order keys in place
    const int nch = (V + 3) >> 2;
    for (int c = tid; c < nch; c += kRowThreads) {
      const int rem = V - 4 * c;
      const uint32_t bytes = rem >= 4 ? 16u : (uint32_t)rem * 4u;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                       (uint32_t)__cvta_generic_to_shared(key + 4 * c)),
                   "l"(row + 4 * c), "r"(bytes)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
    __syncthreads();
    for (int i = tid; i < V; i += kRowThreads) {
      const uint32_t ky = order_key(__uint_as_float(key[i]));
      key[i] = ky;
      mn = min(mn, ky);
      mx = max(mx, ky);
    }
  } else {
    constexpr int kBatch = 8;
    for (int i0 = tid; i0 < V; i0 += kRowThreads * kBatch) {
      float v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * kRowThreads;
        v[u] = i < V ? to_f32(__ldcs(row + i)) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * kRowThreads;
        if (i < V) {
          const uint32_t ky = order_key(v[u]);
          key[i] = ky;
          mn = min(mn, ky);
          mx = max(mx, ky);
        }
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  if (lane == 0) {
    sh.wred[0][warp] = mn;
    sh.wred[1][warp] = mx;
  }
  if (tid == 0) sh.cand_n = 0u;
  __syncthreads();
  // the 16 warps' extremes, reduced by shuffles in every warp
  uint32_t kmin = lane < kRowWarps ? sh.wred[0][lane] : 0xffffffffu;
  uint32_t kmax = lane < kRowWarps ? sh.wred[1][lane] : 0u;
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
  }
  kmin = __shfl_sync(0xffffffffu, kmin, 0);
  kmax = __shfl_sync(0xffffffffu, kmax, 0);
  // warp w's contiguous segment of the row (the candidate and writing passes)
  const int seg = ((V + kRowWarps - 1) / kRowWarps + 31) & ~31;
  const int s0 = min(V, warp * seg), s1 = min(V, s0 + seg);
  // 2. radix refinement of the window [base, base + 2048 << shift)
  uint32_t base = kmin, need = (uint32_t)k;
  int shift = (int)bit_length(kmax - kmin) - kRowBinBits;
  shift = shift < 0 ? 0 : shift;
  uint32_t klo, khi, need_w = 0u, cut_key = 0u;
  int32_t cut_pos = 0;
  bool exact = false;
  for (;;) {
    for (int i = tid; i < kRowBins; i += kRowThreads) sh.hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < V; i += kRowThreads) {
      const uint32_t ky = key[i];
      if (ky >= base) {
        const uint32_t bin = (ky - base) >> shift;
        if (bin < (uint32_t)kRowBins) atomicAdd(&sh.hist[bin], 1u);
      }
    }
    __syncthreads();
    {  // the bin where the count from the top reaches `need` (thread tid owns
       // bins 2047 - 4 tid .. 2044 - 4 tid, descending)
      uint32_t mine[kRowBinsPerThread], loc = 0;
#pragma unroll
      for (int j = 0; j < kRowBinsPerThread; ++j) {
        mine[j] = sh.hist[kRowBins - 1 - (tid * kRowBinsPerThread + j)];
        loc += mine[j];
      }
      uint32_t inc = loc;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += x;
      }
      if (lane == 31) sh.wred[0][warp] = inc;
      __syncthreads();
      uint32_t acc = inc - loc;
      {  // plus the totals of the warps before this one (a 16-lane scan)
        uint32_t wt = lane < kRowWarps ? sh.wred[0][lane] : 0u;
#pragma unroll
        for (int off = 1; off < kRowWarps; off <<= 1) {
          const uint32_t x = __shfl_up_sync(0xffffffffu, wt, off);
          if (lane >= off) wt += x;
        }
        const uint32_t before = __shfl_sync(0xffffffffu, wt, warp > 0 ? warp - 1 : 0);
        acc += warp > 0 ? before : 0u;
      }
#pragma unroll
      for (int j = 0; j < kRowBinsPerThread; ++j) {
        if (acc < need && acc + mine[j] >= need) {
          sh.T = (uint32_t)(kRowBins - 1 - (tid * kRowBinsPerThread + j));
          sh.G = acc;
          sh.C = mine[j];
        }
        acc += mine[j];
      }
      __syncthreads();
    }
    const uint32_t T = sh.T, G = sh.G, C = sh.C;
    klo = base + (T << shift);
    khi = klo + ((1u << shift) - 1u);
    need -= G;
    if (shift == 0 || C == need) {
      need_w = need;
      break;
    }
    if (C <= (uint32_t)kRowCand) {  // rank the bin-T keys among themselves
      // One pass over the warps' segments gathers the bin-T keys and keeps,
      // per 32-key group, the masks of keys above bin T (chosen outright) and
      // in it (chosen by rank) and each warp's count of the former; the
      // writing pass below needs no counting pass of its own.
      uint32_t* gm = sh.hist + warp * (2 * kRowMaxGroups);  // the histogram is no longer read
      uint32_t above = 0;
      for (int i0 = s0, gi = 0; i0 < s1; i0 += 32, ++gi) {
        const int i = i0 + lane;
        const uint32_t ky = i < s1 ? key[i] : 0u;
        const bool in_t = i < s1 && ky >= klo && ky <= khi;
        const uint32_t am = __ballot_sync(0xffffffffu, i < s1 && ky > khi);
        const uint32_t tm = __ballot_sync(0xffffffffu, in_t);
        if (lane == 0) {
          gm[2 * gi] = am;
          gm[2 * gi + 1] = tm;
        }
        above += __popc(am);
        if (in_t) {
          const uint32_t slot = atomicAdd(&sh.cand_n, 1u);
          sh.cand_key[slot] = ky;
          sh.cand_pos[slot] = i;
        }
      }
      if (lane == 0) sh.wcnt[warp] = above << 16;
      __syncthreads();
      for (int e = tid; e < (int)C; e += kRowThreads) {
        const uint32_t ke = sh.cand_key[e];
        const int32_t pe = sh.cand_pos[e];
        uint32_t rank = 0;
        for (int f = 0; f < (int)C; ++f) {
          const uint32_t kf = sh.cand_key[f];
          rank += (kf > ke || (kf == ke && sh.cand_pos[f] < pe)) ? 1u : 0u;
        }
        if (rank < need) atomicAdd(&sh.wcnt[pe / seg], 1u << 16);  // chosen by rank
        if (rank == need - 1) {
          sh.cut_key = ke;
          sh.cut_pos = pe;
        }
      }
      __syncthreads();
      exact = true;
      cut_key = sh.cut_key;
      cut_pos = sh.cut_pos;
      break;
    }
    base = klo;
    shift = shift > kRowBinBits ? shift - kRowBinBits : 0;
    __syncthreads();  // T / G / C are rewritten by the next pass
  }
  // 3. chosen: above the window, or in it and among the first need_w by index
  auto strict_of = [&](uint32_t ky, int i) {
    return exact ? (ky > cut_key || (ky == cut_key && i <= cut_pos)) : ky > khi;
  };
  auto window_of = [&](uint32_t ky) { return !exact && ky >= klo && ky <= khi; };
  // per 32-key group of the warp's segment: the masks of chosen and window
  // keys, kept in the (now unused) histogram for the writing pass (the exact
  // case recorded them, and the counts, while gathering the bin-T keys)
  uint32_t* gmask = sh.hist + warp * (2 * kRowMaxGroups);
  uint32_t strict = 0, win = 0;
  for (int i0 = s0, gi = 0; i0 < s1 && !exact; i0 += 32, ++gi) {
    const int i = i0 + lane;
    const uint32_t ky = i < s1 ? key[i] : 0u;
    const uint32_t sm = __ballot_sync(0xffffffffu, i < s1 && strict_of(ky, i));
    const uint32_t wm = __ballot_sync(0xffffffffu, i < s1 && window_of(ky));
    if (lane == 0) {
      gmask[2 * gi] = sm;
      gmask[2 * gi + 1] = wm;
    }
    strict += __popc(sm);
    win += __popc(wm);
  }
  if (!exact) {
    if (lane == 0) sh.wcnt[warp] = (strict << 16) | win;  // both < 2^16
    __syncthreads();
  }
  uint32_t win_before, out_before;
  {  // lane w < 16: warp w's chosen count; exclusive 16-lane scans
    const uint32_t cw = lane < kRowWarps ? sh.wcnt[lane] : 0u;
    const uint32_t st = cw >> 16, wi = cw & 0xffffu;
    uint32_t wscan = wi;
#pragma unroll
    for (int off = 1; off < kRowWarps; off <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, wscan, off);
      if (lane >= off) wscan += x;
    }
    const uint32_t wpre = wscan - wi;  // window keys in the warps before
    const uint32_t take = need_w > wpre ? min(wi, need_w - wpre) : 0u;
    const uint32_t v = lane < kRowWarps ? st + take : 0u;
    uint32_t oscan = v;
#pragma unroll
    for (int off = 1; off < kRowWarps; off <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, oscan, off);
      if (lane >= off) oscan += x;
    }
    win_before = __shfl_sync(0xffffffffu, wpre, warp);
    out_before = __shfl_sync(0xffffffffu, oscan - v, warp);
  }
  const uint32_t lt = (1u << lane) - 1u;
  for (int i0 = s0, gi = 0; i0 < s1; i0 += 32, ++gi) {
    const int i = i0 + lane;
    const uint32_t sm = gmask[2 * gi], wm = gmask[2 * gi + 1];
    const bool is_w = (wm >> lane) & 1u;
    // exact: wm marks bin-T keys, chosen by the cut; else window keys, chosen
    // in index order up to need_w
    const bool pick = ((sm >> lane) & 1u) ||
                      (is_w && (exact ? strict_of(key[i], i)
                                      : win_before + __popc(wm & lt) < need_w));
    const uint32_t pm = wm == 0u ? sm : __ballot_sync(0xffffffffu, pick);
    const uint32_t o = out_before + __popc(pm & lt);
    if (pick && o < (uint32_t)k) out[o] = i;
    out_before += __popc(pm);
    win_before += __popc(wm);
  }
}

cudaError_t launch_topk_rows_bf16(const __nv_bfloat16* scores, int64_t ld, int64_t batch,
                                  int64_t n, int m, int64_t E, int k, int32_t* idx,
                                  cudaStream_t s) {
  if (E > kRowMaxKeys) return cudaErrorInvalidValue;
  const size_t smem = sizeof(RowTopkShared) + (size_t)E * sizeof(uint32_t);
  auto kern = topk_rows_staged_kernel<__nv_bfloat16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3((unsigned)n, (unsigned)batch), kRowThreads, smem, s>>>(scores, ld, n, m, E, k, idx);
  return cudaGetLastError();
}

cudaError_t launch_topk_rows(const float* scores, int64_t ld, int64_t batch, int64_t n, int m,
                             int64_t E, int k, int32_t* idx, cudaStream_t s) {
  if (E <= kRowMaxKeys) {
    const size_t smem = sizeof(RowTopkShared) + (size_t)E * sizeof(uint32_t);
    auto kern = topk_rows_staged_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3((unsigned)n, (unsigned)batch), kRowThreads, smem, s>>>(scores, ld, n, m, E, k,
                                                                     idx);
    return cudaGetLastError();
  }
  const int64_t smem_keys = E <= kSelSmemKeys ? E : 0;
  const size_t smem = sizeof(SelectShared<kSelThreads>) + (size_t)kSelCap * 4 +
                      (size_t)kSelSample * 4 + (size_t)smem_keys * sizeof(uint32_t);
  cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  dim3 grid((unsigned)n, (unsigned)batch);
  topk_rows_kernel<<<grid, kSelThreads, smem, s>>>(scores, ld, n, m, E, k, smem_keys, idx);
  return cudaGetLastError();
}

}  // namespace csa
