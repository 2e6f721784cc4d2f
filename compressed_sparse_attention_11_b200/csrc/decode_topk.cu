// Decode top-k: the k entries with the largest indexer score among the V
// visible entries of each sequence (the selection step of sections 4.2 / 4.3
// of "DeepSeek-V4: million-token context"; ties to the smaller index, the
// chosen indices listed ascending; all V entries when V <= k).
//
// One thread-block cluster per sequence (up to 16 CTAs); CTA r of the cluster
// copies the contiguous slice r of the sequence's scores (L2-resident after
// the indexer) into shared memory as order keys -- unsigned integers whose
// order is the float order -- so every later pass reads shared memory only.
// An exact radix refinement then finds the k-th largest key: each pass
// histograms the keys of the current window into 4096 bins, the bins are
// summed across the cluster through distributed shared memory (each CTA
// reduces 4096/CS bins and writes the totals into every peer), and every CTA
// finds the same bin T where the count from the top reaches what is still
// needed.  Keys above bin T are chosen.  When bin T holds few keys (the usual
// case after one pass) they are copied into the first CTA of the cluster,
// which ranks them by (key descending, index ascending) and publishes the
// exact cut (key, index) of the k-th choice; otherwise the window narrows to
// bin T with a 4096x finer bin, until the bin holds one key value or is taken
// whole (three passes at most for 32-bit keys).  A last pass writes the
// chosen positions in index order.  Every decision is taken from
// cluster-wide sums, so all CTAs of a cluster run the same passes and
// cluster barriers.
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace csa {

namespace {

namespace cg = cooperative_groups;

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 4096;
constexpr int kBinBits = 12;
constexpr int kBinsPerThread = kBins / kThreads;  // 8
constexpr int kMaxSlice = 45056;                  // keys per CTA (176 KB)
constexpr int kMaxCluster = 16;                   // above 8: a non-portable cluster size
constexpr int kSliceTarget = 16384;               // keys per CTA the cluster size aims for
constexpr int kSmallWin = 512;                    // bin-T keys ranked directly

struct __align__(16) TopkShared {
  uint32_t hist[kBins];   // this CTA's counts
  uint32_t ghist[kBins];  // the cluster's counts
  uint32_t wcnt[kWarps];  // per warp: strict << 16 | window (final pass)
  uint32_t wred[2][kWarps];
  uint32_t pub[4];        // read by peers: min, max key; then strict, window counts
  uint32_t T, G, C;
  uint32_t cand_key[kSmallWin];  // first CTA: the cluster's bin-T keys and positions
  int32_t cand_pos[kSmallWin];
  uint32_t cand_n;
  uint32_t cut_key;  // written by the first CTA into every CTA
  int32_t cut_pos;
};

__device__ __forceinline__ uint32_t bitlen(uint32_t x) { return x == 0 ? 0u : 32u - __clz(x); }

__global__ void __launch_bounds__(kThreads) decode_topk_kernel(
    const int64_t* __restrict__ pos, int64_t cap, int m, int k, const float* __restrict__ scores,
    int32_t* __restrict__ sel, int slice) {
  cg::cluster_group cl = cg::this_cluster();
  const int CS = (int)cl.num_blocks(), r = (int)cl.block_rank();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(smem_raw);
  uint32_t* key = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkShared));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t b = blockIdx.y;

  sm100::pdl_wait();  // the scores come from the previous kernel
  sm100::pdl_trigger();
  const int64_t t = pos[b];
  const int64_t V = t < 0 ? 0 : min((t + 1) / m, cap);
  int32_t* out = sel + b * k;
  if (V <= k) {  // the same decision in every CTA of the cluster
    if (r == 0)
      for (int j = tid; j < k; j += kThreads) out[j] = j < V ? j : -1;
    return;
  }
  const int64_t lo = (int64_t)r * slice;
  const int n = (int)max((int64_t)0, min((int64_t)slice, V - lo));
  if (tid == 0) sh.cand_n = 0u;  // peers add to it only after the first cluster barrier

  // 1. slice -> shared memory as order keys; the slice's key range
  uint32_t mn = 0xffffffffu, mx = 0u;
  {
    const float* row = scores + b * cap + lo;
    constexpr int kBatch = 16;  // loads in flight per thread
    for (int i0 = tid; i0 < n; i0 += kThreads * kBatch) {
      float v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * kThreads;
        v[u] = i < n ? __ldcg(row + i) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * kThreads;
        if (i < n) {
          const uint32_t ky = order_key(v[u]);
          key[i] = ky;
          mn = min(mn, ky);
          mx = max(mx, ky);
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
    __syncthreads();
    if (tid == 0) {
      for (int w = 0; w < kWarps; ++w) {
        mn = min(mn, sh.wred[0][w]);
        mx = max(mx, sh.wred[1][w]);
      }
      sh.pub[0] = mn;
      sh.pub[1] = mx;
    }
  }
  cl.sync();
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int q = 0; q < CS; ++q) {
    const uint32_t* p = cl.map_shared_rank(sh.pub, q);
    kmin = min(kmin, p[0]);
    kmax = max(kmax, p[1]);
  }

  // 2. radix refinement of the window [base, base + 4096 << shift)
  uint32_t base = kmin, need = (uint32_t)k;
  int shift = (int)bitlen(kmax - kmin) - kBinBits;
  shift = shift < 0 ? 0 : shift;
  uint32_t klo, khi, need_w;
  bool exact = false;  // the cut (cut_key, cut_pos) decides instead of the window
  uint32_t cut_key = 0u;
  int32_t cut_pos = 0;
  for (;;) {
    for (int i = tid; i < kBins; i += kThreads) sh.hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kThreads) {
      const uint32_t ky = key[i];
      if (ky >= base) {
        const uint32_t bin = (ky - base) >> shift;
        if (bin < (uint32_t)kBins) atomicAdd(&sh.hist[bin], 1u);
      }
    }
    __syncthreads();
    cl.sync();
    {  // this CTA's share of the bins, summed over the cluster, into every peer
      const int per = kBins / CS;
      for (int bin = r * per + tid; bin < (r + 1) * per; bin += kThreads) {
        uint32_t s = 0;
        for (int q = 0; q < CS; ++q) s += cl.map_shared_rank(sh.hist, q)[bin];
        for (int q = 0; q < CS; ++q) cl.map_shared_rank(sh.ghist, q)[bin] = s;
      }
    }
    cl.sync();
    {  // the bin where the count from the top reaches `need` (thread tid owns
       // bins 4095 - 8 tid .. 4088 - 8 tid, descending)
      uint32_t mine[kBinsPerThread], loc = 0;
#pragma unroll
      for (int j = 0; j < kBinsPerThread; ++j) {
        mine[j] = sh.ghist[kBins - 1 - (tid * kBinsPerThread + j)];
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
      for (int w = 0; w < warp; ++w) acc += sh.wred[0][w];
#pragma unroll
      for (int j = 0; j < kBinsPerThread; ++j) {
        if (acc < need && acc + mine[j] >= need) {
          sh.T = (uint32_t)(kBins - 1 - (tid * kBinsPerThread + j));
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
    if (C <= (uint32_t)kSmallWin) {
      // the bin-T keys of the whole cluster into the first CTA, ranked there
      uint32_t* cnt = cl.map_shared_rank(&sh.cand_n, 0);
      uint32_t* ck = cl.map_shared_rank(sh.cand_key, 0);
      int32_t* cp = cl.map_shared_rank(sh.cand_pos, 0);
      for (int i = tid; i < n; i += kThreads) {
        const uint32_t ky = key[i];
        if (ky >= klo && ky <= khi) {
          const uint32_t slot = atomicAdd(cnt, 1u);
          if (slot < (uint32_t)kSmallWin) {
            ck[slot] = ky;
            cp[slot] = (int32_t)(lo + i);
          }
        }
      }
      cl.sync();
      if (r == 0) {
        const int nc = (int)min(sh.cand_n, (uint32_t)kSmallWin);
        for (int e = tid; e < nc; e += kThreads) {
          const uint32_t ke = sh.cand_key[e];
          const int32_t pe = sh.cand_pos[e];
          uint32_t rank = 0;
          for (int f = 0; f < nc; ++f) {
            const uint32_t kf = sh.cand_key[f];
            rank += (kf > ke || (kf == ke && sh.cand_pos[f] < pe)) ? 1u : 0u;
          }
          if (rank == need - 1) {  // the last choice: publish the cut everywhere
            for (int q = 0; q < CS; ++q) {
              *cl.map_shared_rank(&sh.cut_key, q) = ke;
              *cl.map_shared_rank(&sh.cut_pos, q) = pe;
            }
          }
        }
      }
      cl.sync();
      exact = true;
      cut_key = sh.cut_key;
      cut_pos = sh.cut_pos;
      need_w = 0u;
      break;
    }
    base = klo;
    shift = shift > kBinBits ? shift - kBinBits : 0;
    __syncthreads();  // sh.T / G / C are rewritten by the next pass
  }

  // 3. chosen: key > khi, or klo <= key <= khi among the first need_w of those
  //    (in index order across the cluster).  Warp w scans a contiguous segment.
  const int seg = ((n + kWarps - 1) / kWarps + 31) & ~31;
  const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
  // strict: chosen outright; in window: chosen by index order up to need_w
  auto strict_of = [&](uint32_t ky, int i) {
    return exact ? (ky > cut_key || (ky == cut_key && (int32_t)(lo + i) <= cut_pos)) : ky > khi;
  };
  auto window_of = [&](uint32_t ky) { return !exact && ky >= klo && ky <= khi; };
  uint32_t strict = 0, win = 0;
  for (int i0 = s0; i0 < s1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t ky = i < s1 ? key[i] : 0u;
    strict += __popc(__ballot_sync(0xffffffffu, i < s1 && strict_of(ky, i)));
    win += __popc(__ballot_sync(0xffffffffu, i < s1 && window_of(ky)));
  }
  if (lane == 0) sh.wcnt[warp] = (strict << 16) | win;  // both < 2^16
  __syncthreads();
  if (tid == 0) {
    uint32_t st = 0, wi = 0;
    for (int w = 0; w < kWarps; ++w) {
      st += sh.wcnt[w] >> 16;
      wi += sh.wcnt[w] & 0xffffu;
    }
    sh.pub[2] = st;
    sh.pub[3] = wi;
  }
  cl.sync();
  uint32_t win_before = 0, out_before = 0;  // over the earlier CTAs of the cluster
  for (int q = 0; q < r; ++q) {
    const uint32_t* p = cl.map_shared_rank(sh.pub, q);
    const uint32_t wq = p[3];
    const uint32_t take = need_w > win_before ? min(wq, need_w - win_before) : 0u;
    out_before += p[2] + take;
    win_before += wq;
  }
  cl.sync();  // no CTA leaves while a peer may still read its shared memory
  for (int w = 0; w < warp; ++w) {
    const uint32_t st = sh.wcnt[w] >> 16, wi = sh.wcnt[w] & 0xffffu;
    const uint32_t take = need_w > win_before ? min(wi, need_w - win_before) : 0u;
    out_before += st + take;
    win_before += wi;
  }
  const uint32_t lt = (1u << lane) - 1u;
  for (int i0 = s0; i0 < s1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t ky = i < s1 ? key[i] : 0u;
    const bool is_w = i < s1 && window_of(ky);
    const uint32_t wm = __ballot_sync(0xffffffffu, is_w);
    const bool pick = (i < s1 && strict_of(ky, i)) || (is_w && win_before + __popc(wm & lt) < need_w);
    const uint32_t pm = __ballot_sync(0xffffffffu, pick);
    const uint32_t o = out_before + __popc(pm & lt);
    if (pick && o < (uint32_t)k) out[o] = (int32_t)(lo + i);
    out_before += __popc(pm);
    win_before += __popc(wm);
  }
}

// Cluster size and slice length for a capacity: slices of about
// kSliceTarget keys, at most kMaxCluster CTAs.
void topk_shape(int64_t cap, int& cs, int& slice) {
  cs = 1;
  while (cs < kMaxCluster && (int64_t)cs * kSliceTarget < cap) cs *= 2;
  const int64_t s = (cap + cs - 1) / cs;
  slice = (int)((s + 31) & ~(int64_t)31);
}

}  // namespace

bool decode_topk_supported(const csa_cache_desc& d) {
  int cs, slice;
  topk_shape(d.capacity, cs, slice);
  return !d.is_hca && slice <= kMaxSlice;
}

cudaError_t launch_decode_topk(const csa_cache_desc& d, const int64_t* pos, const float* scores,
                               int32_t* sel, cudaStream_t s) {
  int cs, slice;
  topk_shape(d.capacity, cs, slice);
  if (slice > kMaxSlice) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  auto configure = [&]() -> cudaError_t {
    const size_t smem = sizeof(TopkShared) + (size_t)slice * 4;
    cudaError_t e = cudaFuncSetAttribute(decode_topk_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)cs, (unsigned)d.batch);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaSuccess;
  };
  cudaError_t e = configure();
  if (e != cudaSuccess) return e;
  if (cs > 8) {  // a non-portable cluster: use it only where the device can place one
    int clusters = 0;
    if (cudaFuncSetAttribute(decode_topk_kernel,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&clusters, decode_topk_kernel, &cfg) != cudaSuccess ||
        clusters < 1) {
      cudaGetLastError();  // clear a refusal; fall back to eight CTAs
      cs = 8;
      const int64_t sl = (d.capacity + cs - 1) / cs;
      slice = (int)((sl + 31) & ~(int64_t)31);
      if (slice > kMaxSlice) return cudaErrorInvalidValue;
      if ((e = configure()) != cudaSuccess) return e;
    }
  }
  return cudaLaunchKernelEx(&cfg, decode_topk_kernel, pos, (int64_t)d.capacity, d.m, d.k,
                            scores, sel, slice);
}

}  // namespace csa
