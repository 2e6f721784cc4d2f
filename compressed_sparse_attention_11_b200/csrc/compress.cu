// Token-level KV compressor (CSA overlapped, HCA single-stream).
//
// Defined by the B9 CSA/HCA compressor equations of the "Core formulas
// chapter" and sections 4.1 / 5.1 of "DeepSeek-V4: million-token context":
// entry i, dim d is a per-dimension softmax over the logits Z + B of its rows
// (CSA: m own-block rows of Za/Ca and m previous-block rows of Zb/Cb; the
// first entry has no previous block), applied as Hadamard weights to C.
//
// HBM-streaming kernels: every input row is read exactly once, lanes along
// the dims so that each load instruction of a warp reads contiguous bytes of
// one row.  Entries of at most eight rows (CSA m <= 4) take one thread per
// (entry, 4-dim chunk): all of its rows are loaded at once (8 bytes of a
// bf16 row per lane), then each dim takes a two-pass softmax over them in
// registers, branch-free unless a maximum is infinite; 64 registers keep
// four blocks of 256 threads per SM, and with them enough loads in flight
// to stream.  Larger row sets are split over R warps of one block, one
// thread per (entry, 8-dim chunk, row group); a thread's rows are read in
// rounds of four with all loads of a round issued before its arithmetic,
// and the R partial states are merged through shared memory.  A row whose
// logit equals an infinite maximum gets weight 1 exactly, so a single +inf
// logit selects its row.
#include "common.cuh"
#include "launch.h"
#include "rope.cuh"

namespace csa {

namespace {

// Eight elements of one row, raw, and the rows per thread per round.
template <typename T>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
  static constexpr int kSlots = 4;
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    u = __ldcs(reinterpret_cast<const uint4*>(p));
  }
  __device__ __forceinline__ float get(int q) const {
    const uint32_t w = q < 2 ? u.x : q < 4 ? u.y : q < 6 ? u.z : u.w;
    return __uint_as_float((q & 1) ? (w & 0xffff0000u) : (w << 16));
  }
};
template <>
struct Raw8<float> {
  static constexpr int kSlots = 4;
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldcs(reinterpret_cast<const float4*>(p));
    b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ float get(int q) const {
    switch (q) {
      case 0: return a.x;
      case 1: return a.y;
      case 2: return a.z;
      case 3: return a.w;
      case 4: return b.x;
      case 5: return b.y;
      case 6: return b.z;
      default: return b.w;
    }
  }
};

// Softmax state of one dim over a set of rows: max logit M, sum of
// exp(l - M) S, weighted sum A.  A row whose logit equals the max gets weight
// 1 exactly, so a single +inf logit selects its row.
struct Osm {
  float M, S, A;
};

__device__ __forceinline__ Osm osm_combine(Osm x, Osm y) {
  const float mn = fmaxf(x.M, y.M);
  if (mn == kNegInf) return x;
  const float fx = x.M >= mn ? 1.f : ex2((x.M - mn) * kLog2e);
  const float fy = y.M >= mn ? 1.f : ex2((y.M - mn) * kLog2e);
  return Osm{mn, x.S * fx + y.S * fy, x.A * fx + y.A * fy};
}

// Row j (0 <= j < rows) of entry i: own block rows first, then (CSA) the
// previous block's rows.  Returns false for the previous block of entry 0.
template <typename T>
__device__ __forceinline__ bool row_ptrs(const T* ca, const T* cb, const T* za, const T* zb,
                                         const float* ba, const float* bb, int64_t seq,
                                         int64_t i, int j, int m, int c, int d0, const T*& cp,
                                         const T*& zp, const float*& bp) {
  if (j < m) {
    const int64_t row = seq + i * m + j;
    cp = ca + row * c + d0;
    zp = za + row * c + d0;
    bp = ba + (int64_t)j * c + d0;
    return true;
  }
  if (i == 0) return false;
  const int64_t row = seq + (i - 1) * m + (j - m);
  cp = cb + row * c + d0;
  zp = zb + row * c + d0;
  bp = bb + (int64_t)(j - m) * c + d0;
  return true;
}

// One round: rows j = r0 + stride * t, t < kSlots, of one entry and one
// 8-dim chunk; all loads first, then the two-pass softmax into st[8].
template <typename T>
__device__ __forceinline__ void round_rows(const T* ca, const T* cb, const T* za, const T* zb,
                                           const float* ba, const float* bb, int64_t seq,
                                           int64_t i, int m, int rows, int c, int d0, int r0,
                                           int stride, Osm st[8]) {
  constexpr int kSlots = Raw8<T>::kSlots;
  Raw8<T> cr[kSlots], zr[kSlots];
  const float* bp[kSlots];
  bool act[kSlots];
#pragma unroll
  for (int t = 0; t < kSlots; ++t) {
    const int j = r0 + stride * t;
    const T* cp = nullptr;
    const T* zp = nullptr;
    bp[t] = nullptr;
    act[t] = j < rows && row_ptrs(ca, cb, za, zb, ba, bb, seq, i, j, m, c, d0, cp, zp, bp[t]);
    if (act[t]) {
      cr[t].load(cp);
      zr[t].load(zp);
    }
  }
  float bv[kSlots][8];
#pragma unroll
  for (int t = 0; t < kSlots; ++t) {
    if (act[t]) {
      load8(bp[t], bv[t]);
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) bv[t][q] = kNegInf;
    }
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    float mx = kNegInf;
#pragma unroll
    for (int t = 0; t < kSlots; ++t)
      if (act[t]) mx = fmaxf(mx, zr[t].get(q) + bv[t][q]);
    float s = 0.f, a = 0.f;
    if (mx != kNegInf) {
#pragma unroll
      for (int t = 0; t < kSlots; ++t) {
        if (!act[t]) continue;
        const float l = zr[t].get(q) + bv[t][q];
        const float w = l >= mx ? 1.f : ex2((l - mx) * kLog2e);
        s += w;
        a = fmaf(w, cr[t].get(q), a);
      }
    }
    st[q] = Osm{mx, s, a};
  }
}

// RMSNorm + partial RoPE of the compressed entries (sections 4.5 / 7.4 of
// "DeepSeek-V4: million-token context"), applied as they are written; entry
// i is rotated for position m * i.  NULL gamma: plain compression.
struct EntryNormRope {
  const float* gamma;
  float eps;
  int rope_dims;
  float base;
};

// Four elements of one row, raw.
template <typename T>
struct Raw4;
template <>
struct Raw4<__nv_bfloat16> {
  uint2 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    u = __ldcs(reinterpret_cast<const uint2*>(p));
  }
  __device__ __forceinline__ float get(int q) const {
    const uint32_t w = q < 2 ? u.x : u.y;
    return __uint_as_float((q & 1) ? (w & 0xffff0000u) : (w << 16));
  }
};
template <>
struct Raw4<float> {
  float4 a;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldcs(reinterpret_cast<const float4*>(p));
  }
  __device__ __forceinline__ float get(int q) const {
    return q == 0 ? a.x : q == 1 ? a.y : q == 2 ? a.z : a.w;
  }
};

// Four consecutive dims d0 .. d0 + 3 (d0 a multiple of 4) of an entry whose
// reciprocal RMS is `inv`: scaled by inv * gamma[d], and turned pairwise for
// position `pos` where they lie in the trailing rope_dims dims.
__device__ __forceinline__ void norm_rope4(float v[4], int d0, int c, float inv,
                                           const float* __restrict__ gamma, int64_t pos,
                                           int rope_dims, float base) {
#pragma unroll
  for (int q = 0; q < 4; ++q) v[q] = v[q] * inv * __ldg(gamma + d0 + q);
  if (d0 >= c - rope_dims) {
    const int j0 = (d0 - (c - rope_dims)) >> 1;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      float cs, sn;
      rope_cos_sin(pos, j0 + p, rope_dims, base, cs, sn);
      rope_turn(v[2 * p], v[2 * p + 1], cs, sn);
    }
  }
}

// Softmax over the live rows of four dims: o[q] = sum_j w_j C_j[q] / sum_j w_j
// with w_j = exp(l_j - max l), l_j = Z_j[q] + bias_j[q].  The logits are kept
// in base-2 units.  When every maximum is finite the weights are ex2(l - max)
// throughout; otherwise the guarded form gives the row at the maximum weight
// 1 exactly (a +inf logit selects its row, all -inf logits weigh alike),
// where l - max would be inf - inf.
template <int kMaxRows, typename T, typename Bias>
__device__ __forceinline__ void fold_rows4(const Raw4<T> (&cr)[kMaxRows],
                                           const Raw4<T> (&zr)[kMaxRows],
                                           const bool (&live)[kMaxRows], const Bias& bias,
                                           float o[4]) {
  float lg[kMaxRows][4], mx[4], sum[4], acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    mx[q] = kNegInf;
    sum[q] = 0.f;
    acc[q] = 0.f;
  }
#pragma unroll
  for (int j = 0; j < kMaxRows; ++j) {
    if (!live[j]) continue;
    const float4 bj = bias(j);
    const float b4[4] = {bj.x, bj.y, bj.z, bj.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      lg[j][q] = (zr[j].get(q) + b4[q]) * kLog2e;
      mx[q] = fmaxf(mx[q], lg[j][q]);
    }
  }
  const float kInf = -kNegInf;
  const bool finite = fabsf(mx[0]) < kInf && fabsf(mx[1]) < kInf &&
                      fabsf(mx[2]) < kInf && fabsf(mx[3]) < kInf;
  if (finite) {
#pragma unroll
    for (int j = 0; j < kMaxRows; ++j) {
      if (!live[j]) continue;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float w = ex2(lg[j][q] - mx[q]);
        sum[q] += w;
        acc[q] = fmaf(w, cr[j].get(q), acc[q]);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < kMaxRows; ++j) {
      if (!live[j]) continue;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float w = lg[j][q] >= mx[q] ? 1.f : ex2(lg[j][q] - mx[q]);
        sum[q] += w;
        acc[q] = fmaf(w, cr[j].get(q), acc[q]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) o[q] = acc[q] / sum[q];
}

// Entries with at most eight rows, one thread per (entry, 4-dim chunk): all
// rows of the thread are loaded at once (8 bytes of a bf16 row per lane, so a
// warp reads 256 contiguous bytes of it), then each dim takes a two-pass
// softmax over its rows in registers (branch-free unless a maximum is
// infinite).
template <typename T, bool kNorm>
__global__ void __launch_bounds__(256, sizeof(T) == 2 ? 4 : 2) compress_rows_kernel(
    const T* __restrict__ ca, const T* __restrict__ cb, const T* __restrict__ za,
    const T* __restrict__ zb, const float* __restrict__ ba, const float* __restrict__ bb,
    int64_t n, int c, int m, int rows, int64_t E, int64_t items, EntryNormRope nr,
    T* __restrict__ out) {
  constexpr int kMaxRows = 8;
  const int64_t g0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (!kNorm && g0 >= items) return;
  const bool act = g0 < items;  // (with the norm every thread reaches the block barrier)
  const int64_t g = act ? g0 : items - 1;
  const int chunks = c >> 2;
  const int d0 = (int)(g % chunks) * 4;
  const int64_t rest = g / chunks;
  const int64_t i = rest % E, b = rest / E;
  Raw4<T> cr[kMaxRows], zr[kMaxRows];
  bool live[kMaxRows];
#pragma unroll
  for (int j = 0; j < kMaxRows; ++j) {
    const T* cp = nullptr;
    const T* zp = nullptr;
    const float* bp = nullptr;
    live[j] = j < rows && row_ptrs(ca, cb, za, zb, ba, bb, b * n, i, j, m, c, d0, cp, zp, bp);
    if (live[j]) {
      cr[j].load(cp);
      zr[j].load(zp);
    }
  }
  // the positional bias of row j (a few KB shared by all entries: L1 hits),
  // read once per pass rather than held in registers
  const auto bias = [&](int j) {
    return __ldg(reinterpret_cast<const float4*>((j < m ? ba + (int64_t)j * c
                                                        : bb + (int64_t)(j - m) * c) + d0));
  };
  float o[4];
  fold_rows4(cr, zr, live, bias, o);
  if constexpr (kNorm) {
    __shared__ float wsum[8];
    float ss = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) ss = fmaf(o[q], o[q], ss);
    const int seg = chunks < 32 ? chunks : 32;
    for (int off = seg >> 1; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (chunks > 32) {  // the entry spans chunks / 32 warps of the block
      const int warp = threadIdx.x >> 5;
      if ((threadIdx.x & 31) == 0) wsum[warp] = ss;
      __syncthreads();
      const int w0 = warp & ~(chunks / 32 - 1);
      ss = 0.f;
      for (int w = 0; w < chunks / 32; ++w) ss += wsum[w0 + w];
    }
    const float inv = 1.f / sqrtf(ss / (float)c + nr.eps);
    norm_rope4(o, d0, c, inv, nr.gamma, (int64_t)m * i, nr.rope_dims, nr.base);
  }
  if (act) {
    T* dst = out + (b * E + i) * c + d0;
    if constexpr (sizeof(T) == 2) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
    } else {
      *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
    }
  }
}

// Entries with more rows: block (CX chunks) x (R row groups); thread (x, r)
// reads rows r, r + R, r + 2R, ... of its chunk in rounds of four; the R
// states are merged in shared memory.  CX = blockDim.x is 32, or the whole
// entry's c / 8 chunks (at most 64) when the entry is normed (kNorm): the
// block then holds the entry and sums its squares itself.
template <typename T, bool kNorm>
__global__ void __launch_bounds__(256) compress_split_kernel(
    const T* __restrict__ ca, const T* __restrict__ cb, const T* __restrict__ za,
    const T* __restrict__ zb, const float* __restrict__ ba, const float* __restrict__ bb,
    int64_t n, int c, int m, int rows, int64_t E, int chunk_blocks, EntryNormRope nr,
    T* __restrict__ out) {
  extern __shared__ float sh[];  // [3][R][8][CX]
  const int x = threadIdx.x, r = threadIdx.y, R = blockDim.y, CX = blockDim.x;
  const int cblk = (int)(blockIdx.x % chunk_blocks);
  const int64_t ent = blockIdx.x / chunk_blocks;
  const int64_t i = ent % E, b = ent / E;
  const int chunks = c >> 3;
  const int chunk = cblk * CX + x;
  const bool valid = chunk < chunks;
  const int d0 = valid ? chunk * 8 : 0;

  Osm st[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) st[q] = Osm{kNegInf, 0.f, 0.f};
  if (valid) {
    for (int r0 = r; r0 < rows; r0 += R * Raw8<T>::kSlots) {
      Osm part[8];
      round_rows(ca, cb, za, zb, ba, bb, b * n, i, m, rows, c, d0, r0, R, part);
#pragma unroll
      for (int q = 0; q < 8; ++q) st[q] = osm_combine(st[q], part[q]);
    }
  }
  const int plane = R * 8 * CX;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int at = (r * 8 + q) * CX + x;
    sh[at] = st[q].M;
    sh[plane + at] = st[q].S;
    sh[2 * plane + at] = st[q].A;
  }
  __syncthreads();
  // thread (x, r) merges dims r, r + R, ... of its chunk over the R groups
  float* res = sh;  // reused after the merge: [8][CX]
  float v[8];  // v[u]: dim r + u R
  int nq = 0;
  for (int q = r; q < 8; q += R, ++nq) {
    Osm acc{kNegInf, 0.f, 0.f};
    for (int u = 0; u < R; ++u) {
      const int at = (u * 8 + q) * CX + x;
      acc = osm_combine(acc, Osm{sh[at], sh[plane + at], sh[2 * plane + at]});
    }
    v[nq] = acc.A / acc.S;
  }
  __syncthreads();
  for (int u = 0; u < nq; ++u) res[(r + u * R) * CX + x] = v[u];
  __syncthreads();
  if (r == 0) {
    float o[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) o[q] = res[q * CX + x];
    if constexpr (kNorm) {
      // the block holds the whole entry: sum of squares over its CX chunks
      float ss = 0.f;
      if (valid)
#pragma unroll
        for (int q = 0; q < 8; ++q) ss = fmaf(o[q], o[q], ss);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      float* wsum = sh + 8 * CX;  // past res
      if ((x & 31) == 0) wsum[x >> 5] = ss;
      asm volatile("bar.sync 1, %0;" ::"r"(CX) : "memory");  // the r == 0 threads only
      ss = 0.f;
      for (int w = 0; w < (CX + 31) / 32; ++w) ss += wsum[w];
      const float inv = 1.f / sqrtf(ss / (float)c + nr.eps);
      if (valid) norm_rope8(o, d0, c, inv, nr.gamma, (int64_t)m * i, nr.rope_dims, nr.base);
    }
    if (valid) store8(out + (b * E + i) * c + d0, o);
  }
}

template <typename T>
cudaError_t launch_compress_t(const void* ca, const void* cb, const void* za, const void* zb,
                              const float* ba, const float* bb, int64_t batch, int64_t n, int c,
                              int m, int overlap, const csa_norm_rope* nr, void* out,
                              cudaStream_t s) {
  const int64_t E = n / m;
  const int rows = overlap ? 2 * m : m;
  if (batch * E == 0) return cudaSuccess;
  const int chunks = c / 8;
  if (rows <= 8) {
    const int chunks4 = c / 4;
    const bool fused4 = nr != nullptr && chunks4 <= 256 && 256 % chunks4 == 0;
    const int64_t items = batch * E * chunks4;
    const unsigned grid = (unsigned)((items + 255) / 256);
    if (fused4) {
      const EntryNormRope enr{nr->gamma, nr->eps, nr->rope_dims, nr->rope_base};
      compress_rows_kernel<T, true><<<grid, 256, 0, s>>>(
          (const T*)ca, (const T*)cb, (const T*)za, (const T*)zb, ba, bb, n, c, m, rows, E,
          items, enr, (T*)out);
      return cudaGetLastError();
    }
    compress_rows_kernel<T, false><<<grid, 256, 0, s>>>(
        (const T*)ca, (const T*)cb, (const T*)za, (const T*)zb, ba, bb, n, c, m, rows, E, items,
        EntryNormRope{nullptr, 0.f, 0, 0.f}, (T*)out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || nr == nullptr) return e;
    // the entry's chunks do not tile a block: norm and rotation as a second
    // pass over the (small) compressed output, in place
    return launch_norm_rope_rows(out, batch, E, 1, c, m, nr,
                                 sizeof(T) == 2 ? CSA_BF16 : CSA_F32, out, s);
  }
  // R = groups of rows: one round per thread where possible; with the norm
  // the block takes the whole entry (c / 8 <= 64 chunks, a multiple of 32)
  constexpr int kSlots = Raw8<T>::kSlots;
  const bool split_fused = nr != nullptr && chunks <= 64 && chunks % 32 == 0;
  const int CX = split_fused ? chunks : 32;
  const int max_r = 256 / CX;
  int R = 1;
  while (R < max_r && R * kSlots < rows) R <<= 1;
  const int chunk_blocks = (chunks + CX - 1) / CX;
  const size_t smem = (size_t)3 * R * 8 * CX * sizeof(float) + 64;
  const unsigned grid = (unsigned)(batch * E * chunk_blocks);
  cudaError_t e;
  if (split_fused) {
    auto kern = compress_split_kernel<T, true>;
    if (smem > 48 * 1024 &&
        (e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
            cudaSuccess)
      return e;
    kern<<<grid, dim3(CX, R), smem, s>>>((const T*)ca, (const T*)cb, (const T*)za,
                                         (const T*)zb, ba, bb, n, c, m, rows, E, chunk_blocks,
                                         EntryNormRope{nr->gamma, nr->eps, nr->rope_dims,
                                                       nr->rope_base},
                                         (T*)out);
    return cudaGetLastError();
  }
  auto kern = compress_split_kernel<T, false>;
  if (smem > 48 * 1024 &&
      (e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
          cudaSuccess)
    return e;
  kern<<<grid, dim3(CX, R), smem, s>>>((const T*)ca, (const T*)cb, (const T*)za, (const T*)zb,
                                       ba, bb, n, c, m, rows, E, chunk_blocks,
                                       EntryNormRope{nullptr, 0.f, 0, 0.f}, (T*)out);
  e = cudaGetLastError();
  if (e != cudaSuccess || nr == nullptr) return e;
  // an entry of this kernel spans several blocks: the norm and rotation run as
  // a second pass over the (n/m rows of) compressed output, in place
  return launch_norm_rope_rows(out, batch, E, 1, c, m, nr, sizeof(T) == 2 ? CSA_BF16 : CSA_F32,
                               out, s);
}

}  // namespace

cudaError_t launch_compress(const void* ca, const void* cb, const void* za, const void* zb,
                            const float* ba, const float* bb, int64_t batch, int64_t n, int c,
                            int m, int overlap, csa_dtype dt, const csa_norm_rope* nr, void* out,
                            cudaStream_t s) {
  if (dt == CSA_F32)
    return launch_compress_t<float>(ca, cb, za, zb, ba, bb, batch, n, c, m, overlap, nr, out, s);
  return launch_compress_t<__nv_bfloat16>(ca, cb, za, zb, ba, bb, batch, n, c, m, overlap, nr,
                                          out, s);
}

}  // namespace csa
