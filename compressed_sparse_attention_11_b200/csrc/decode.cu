// Decode over a persistent compressed cache (one token per sequence).
//
// Cache model ("DeepSeek paper-feature analysis", section "Inference KV
// Cache"): a state cache holding the sliding-window rows and the raw rows
// still waiting for compression, and a classical cache of compressed entries.
// Entries are stored with the RoPE dims in bf16 and the rest in FP8 E4M3
// with one fp32 scale per entry (section 7.3 "KV mixed-precision storage");
// index keys are FP8 with their own scale.  The compressor state is the raw
// tail plus, for CSA, the previous block's overlap rows (reader's notes,
// section 2), kept in two block-parity slots.
//
// One step, in order (each kernel on the caller's stream):
//   1. append_emit   : write the token's rows; if (t+1) % m == 0 compress
//                      entry t/m from the state, quantise, store (and its key)
//   2. index_chunk   : CSA - score a chunk of visible index keys, keep the
//                      chunk's top-k candidates
//   3. topk_merge    : CSA - top-k over all chunks' candidates
//   4. attn_split    : attention over a slice of the entry set (selected or
//                      all visible entries, then the window), partial softmax
//   5. attn_combine  : merge the slices and the sink, write bf16 output
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"
#include "topk.cuh"

#include <algorithm>

namespace csa {

constexpr int kSelThreads = 512;          // CUDA-core chunk top-k / merge blocks
constexpr int kDecSelThreads = 1024;      // one selection block per sequence


static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

void cache_layout(const csa_cache_desc& d, csa_cache_layout_t* L, const csa_paging* pg) {
  const size_t B = (size_t)d.batch, cap = (size_t)d.capacity;
  const size_t body = (size_t)(d.c - d.rope_dims);
  // entry rows: batch x capacity, or the paged pool's blocks x entries per block
  const size_t rows = pg != nullptr ? (size_t)pg->num_blocks * (size_t)(pg->block_tokens / d.m)
                                    : B * cap;
  size_t off = 0;
  L->entry_fp8 = off;   off = align256(off + rows * body);
  L->entry_scale = off; off = align256(off + rows * 4);
  L->entry_rope = off;  off = align256(off + rows * (size_t)d.rope_dims * 2);
  L->ikey_fp8 = off;    if (!d.is_hca) off = align256(off + rows * (size_t)d.c_i);
  L->ikey_scale = off;  if (!d.is_hca) off = align256(off + rows * 4);
  L->window = off;      off = align256(off + B * (size_t)d.window * d.c * 2);
  L->state = off;
  off = align256(off + B * 2 * (d.is_hca ? 1 : 4) * (size_t)d.m * d.c * 2);
  L->istate = off;
  if (!d.is_hca) off = align256(off + B * 2 * 4 * (size_t)d.m * d.c_i * 2);
  L->total_bytes = off;
}

CacheView cache_view(const csa_cache_desc& d, void* cache, const csa_paging* pg) {
  csa_cache_layout_t L;
  cache_layout(d, &L, pg);
  uint8_t* base = static_cast<uint8_t*>(cache);
  CacheView v;
  v.entry_fp8 = base + L.entry_fp8;
  v.entry_scale = reinterpret_cast<float*>(base + L.entry_scale);
  v.entry_rope = reinterpret_cast<__nv_bfloat16*>(base + L.entry_rope);
  v.ikey_fp8 = base + L.ikey_fp8;
  v.ikey_scale = reinterpret_cast<float*>(base + L.ikey_scale);
  v.window = reinterpret_cast<__nv_bfloat16*>(base + L.window);
  v.state = reinterpret_cast<__nv_bfloat16*>(base + L.state);
  v.istate = reinterpret_cast<__nv_bfloat16*>(base + L.istate);
  v.btab = pg != nullptr ? pg->block_table : nullptr;
  v.bt_stride = pg != nullptr ? pg->max_blocks : 0;
  v.nblocks = pg != nullptr ? pg->num_blocks : 0;
  int sh = 0;
  if (pg != nullptr)
    while ((1 << sh) < pg->block_tokens / d.m) ++sh;
  v.epb_shift = sh;
  return v;
}

// ---------------------------------------------------------------------------
// Entry quantisation: scale = amax/448 over the FP8 dims (1 if amax == 0);
// code = E4M3(x / scale), round to nearest even, saturating; trailing
// rope_dims dims as bf16.  `x` is in shared memory; called by all threads.
// ---------------------------------------------------------------------------
__device__ __noinline__ void quantize_store(const float* x, int c, int rope, uint8_t* codes,
                                            float* scale_out, __nv_bfloat16* rope_out,
                                            float* red) {
  const int body = c - rope;
  float amax = 0.f;
  for (int d = threadIdx.x; d < body; d += blockDim.x) amax = fmaxf(amax, fabsf(x[d]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) amax = fmaxf(amax, red[w]);
  const float scale = amax > 0.f ? amax / 448.f : 1.f;
  for (int d = threadIdx.x; d < body; d += blockDim.x) codes[d] = e4m3_code(x[d] / scale);
  for (int d = threadIdx.x; d < rope; d += blockDim.x)
    rope_out[d] = __float2bfloat16_rn(x[body + d]);
  if (threadIdx.x == 0) *scale_out = scale;
  __syncthreads();
}

template <typename T>
__global__ void __launch_bounds__(256) store_entries_kernel(
    csa_cache_desc d, CacheView cv, int64_t first, int64_t count, const T* __restrict__ kv,
    const T* __restrict__ ikey) {
  extern __shared__ float sx[];  // [c + c_i] + reduction scratch
  const int64_t j = blockIdx.x, b = blockIdx.y;
  const int64_t slot = first + j;
  float* red = sx + d.c + (d.is_hca ? 0 : d.c_i);
  for (int e = threadIdx.x; e < d.c; e += blockDim.x)
    sx[e] = to_f32(kv[(b * count + j) * d.c + e]);
  if (!d.is_hca)
    for (int e = threadIdx.x; e < d.c_i; e += blockDim.x)
      sx[d.c + e] = to_f32(ikey[(b * count + j) * d.c_i + e]);
  __syncthreads();
  const int64_t es = entry_row(cv, b, slot, d.capacity);
  if (es < 0) return;  // no block for this entry (uniform over the block)
  quantize_store(sx, d.c, d.rope_dims, cv.entry_fp8 + es * (d.c - d.rope_dims),
                 cv.entry_scale + es, cv.entry_rope + es * d.rope_dims, red);
  if (!d.is_hca)
    quantize_store(sx + d.c, d.c_i, 0, cv.ikey_fp8 + es * d.c_i, cv.ikey_scale + es, nullptr,
                   red);
}

cudaError_t launch_store_entries(const csa_cache_desc& d, const CacheView& cv, int64_t first,
                                 int64_t count, const void* kv, const void* ikey, csa_dtype dt,
                                 cudaStream_t s) {
  const size_t smem = sizeof(float) * (d.c + (d.is_hca ? 0 : d.c_i) + 32);
  dim3 grid((unsigned)count, (unsigned)d.batch);
  if (dt == CSA_F32)
    store_entries_kernel<float><<<grid, 256, smem, s>>>(d, cv, first, count, (const float*)kv,
                                                        (const float*)ikey);
  else
    store_entries_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(
        d, cv, first, count, (const __nv_bfloat16*)kv, (const __nv_bfloat16*)ikey);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Raw rows -> window ring and compressor state.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void copy_row(__nv_bfloat16* dst, const __nv_bfloat16* src, int dim) {
  for (int e = threadIdx.x * 8; e < dim; e += blockDim.x * 8)
    *reinterpret_cast<uint4*>(dst + e) = *reinterpret_cast<const uint4*>(src + e);
}

// Writes position u's rows (source row `r` of [batch][count][dim] arrays).
__device__ void put_rows(const csa_cache_desc& d, const CacheView& cv, const csa_rows& rows,
                         int64_t b, int64_t count, int64_t r, int64_t u, bool ring, bool state) {
  typedef __nv_bfloat16 bf;
  const int64_t c = d.c, ci = d.c_i, m = d.m;
  if (ring)
    copy_row(cv.window + (b * d.window + u % d.window) * c,
             (const bf*)rows.kv_win + (b * count + r) * c, (int)c);
  if (!state) return;
  const int64_t row = u % m;
  if (d.is_hca) {
    bf* st = cv.state + b * 2 * m * c;
    copy_row(st + (0 * m + row) * c, (const bf*)rows.ca + (b * count + r) * c, (int)c);
    copy_row(st + (1 * m + row) * c, (const bf*)rows.za + (b * count + r) * c, (int)c);
    return;
  }
  const int64_t par = (u / m) & 1;
  const void* src[4] = {rows.ca, rows.cb, rows.za, rows.zb};
  const void* isrc[4] = {rows.ica, rows.icb, rows.iza, rows.izb};
  for (int st = 0; st < 4; ++st) {
    copy_row(cv.state + (((b * 2 + par) * 4 + st) * m + row) * c,
             (const bf*)src[st] + (b * count + r) * c, (int)c);
    copy_row(cv.istate + (((b * 2 + par) * 4 + st) * m + row) * ci,
             (const bf*)isrc[st] + (b * count + r) * ci, (int)ci);
  }
}

__global__ void __launch_bounds__(256) write_rows_kernel(csa_cache_desc d, CacheView cv,
                                                         int64_t first, int64_t count,
                                                         csa_rows rows) {
  const int64_t r = blockIdx.x, b = blockIdx.y;
  const int64_t u = first + r, last = first + count - 1;
  // only the last writer of each ring / state slot writes (blocks run in any order)
  const bool ring = u > last - d.window;
  const bool state = u > last - (d.is_hca ? 1 : 2) * (int64_t)d.m;
  put_rows(d, cv, rows, b, count, r, u, ring, state);
}

cudaError_t launch_write_rows(const csa_cache_desc& d, const CacheView& cv, int64_t first_pos,
                              int64_t count, const csa_rows& rows, cudaStream_t s) {
  dim3 grid((unsigned)count, (unsigned)d.batch);
  write_rows_kernel<<<grid, 256, 0, s>>>(d, cv, first_pos, count, rows);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Step 1: append the token's rows and emit a finished entry.
// ---------------------------------------------------------------------------
// One block's rows of dim d folded into the online softmax state (M, S, A).
__device__ __noinline__ void emit_fold(const __nv_bfloat16* cp, const __nv_bfloat16* zp,
                                       const float* bias, int m, int dim, int d, float* state) {
  float M = state[0], S = state[1], A = state[2];
#pragma unroll 1
  for (int j0 = 0; j0 < m; j0 += 4) {
    float cval[4], zval[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      cval[q] = 0.f;
      zval[q] = kNegInf;
      if (j0 + q < m) {
        const int64_t o = (int64_t)(j0 + q) * dim + d;
        cval[q] = __bfloat162float(cp[o]);
        zval[q] = __bfloat162float(zp[o]) + bias[o];
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (j0 + q < m) osm_update(M, S, A, zval[q], cval[q]);
  }
  state[0] = M;
  state[1] = S;
  state[2] = A;
}

// Per-dim softmax over the state rows of entry i (dims d of a `dim`-wide
// stream set).  CSA: own block (parity i%2, streams ca/za) and, for i > 0, the
// previous block (parity (i-1)%2, streams cb/zb).  HCA: streams C/Z.  The
// rows are loaded four at a time before they are folded in, so a CSA block
// of rows costs one memory latency, not one per row.  (Out of line and rolled,
// like quantize_store: the emission runs once per entry, so its code is
// fetched about once per launch and its size is what it costs.)
__device__ __noinline__ float emit_dim(const __nv_bfloat16* st, int64_t b, int64_t i, int m,
                                       int dim, int d, const float* ba, const float* bb,
                                       bool hca) {
  float state[3] = {kNegInf, 0.f, 0.f};
  if (hca) {
    const __nv_bfloat16* base = st + b * 2 * (int64_t)m * dim;
    emit_fold(base, base + (int64_t)m * dim, ba, m, dim, d, state);
  } else {
    auto blk = [&](int64_t par, int s) { return st + ((b * 2 + par) * 4 + s) * (int64_t)m * dim; };
    emit_fold(blk(i & 1, 0), blk(i & 1, 2), ba, m, dim, d, state);
    if (i > 0) emit_fold(blk((i - 1) & 1, 1), blk((i - 1) & 1, 3), bb, m, dim, d, state);
  }
  return state[2] / state[1];
}

// The token's rows -- the window row and the compressor-state rows -- copied
// into the cache with every load issued before any store.
__device__ void append_rows(const csa_cache_desc& d, const CacheView& cv, const csa_rows& rows,
                            int64_t b, int64_t u) {
  typedef __nv_bfloat16 bf;
  constexpr int kMaxRows = 9;
  const int64_t c = d.c, ci = d.c_i, m = d.m, row = u % m;
  const bf* src[kMaxRows];
  bf* dst[kMaxRows];
  int nch[kMaxRows];  // 16-byte chunks per row
  int nr = 0;
  auto add = [&](const void* sp, bf* dp, int64_t dim) {
    src[nr] = (const bf*)sp + b * dim;
    dst[nr] = dp;
    nch[nr++] = (int)(dim / 8);
  };
  add(rows.kv_win, cv.window + (b * d.window + u % d.window) * c, c);
  if (d.is_hca) {
    bf* st = cv.state + b * 2 * m * c;
    add(rows.ca, st + row * c, c);
    add(rows.za, st + (m + row) * c, c);
  } else {
    const int64_t par = (u / m) & 1;
    const void* sv[4] = {rows.ca, rows.cb, rows.za, rows.zb};
    const void* iv[4] = {rows.ica, rows.icb, rows.iza, rows.izb};
    for (int s = 0; s < 4; ++s) {
      add(sv[s], cv.state + (((b * 2 + par) * 4 + s) * m + row) * c, c);
      add(iv[s], cv.istate + (((b * 2 + par) * 4 + s) * m + row) * ci, ci);
    }
  }
  int total = 0;
  for (int r = 0; r < nr; ++r) total += nch[r];
  constexpr int kPer = 4;  // chunks per thread per round
  for (int base = 0; base < total; base += (int)blockDim.x * kPer) {
    uint4 v[kPer];
    bf* dp[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      int ch = base + q * (int)blockDim.x + (int)threadIdx.x;
      dp[q] = nullptr;
      if (ch >= total) continue;
      int r = 0;
      while (ch >= nch[r]) ch -= nch[r++];
      v[q] = *reinterpret_cast<const uint4*>(src[r] + ch * 8);
      dp[q] = dst[r] + ch * 8;
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (dp[q] != nullptr) *reinterpret_cast<uint4*>(dp[q]) = v[q];
  }
}

// The tensor-core indexer's query operand of one sequence (H heads of
// dim 128): per head a power of two s_h >= max|q_h|/448 and the E4M3 pair
// hi = E4M3(q/s_h), lo = E4M3(q/s_h - hi), written as the MMA's B operand
// image (2H rows of 128 bytes with the 128-byte swizzle: hi rows 0..H-1, lo
// rows H..2H-1), followed by the H weights w_h * s_h.  s_h (hi + lo) equals
// the bf16 query except for elements below 2^-2 s_h in magnitude, whose
// residual falls under E4M3's subnormal step (absolute error <= 2^-10 s_h).
// A half-warp per head, eight dims per thread.
__device__ void build_query_operand(const __nv_bfloat16* __restrict__ q,
                                    const float* __restrict__ w, int H, uint8_t* rec) {
  const int hw = threadIdx.x >> 4, hl = threadIdx.x & 15, nhw = blockDim.x >> 4;
  float* wout = reinterpret_cast<float*>(rec + 2 * H * 128);
  for (int h0 = 0; h0 < H; h0 += nhw) {  // the same trip count in every thread
    const int h = h0 + hw;
    const bool act = h < H;
    const uint4 raw = act ? *reinterpret_cast<const uint4*>(q + (int64_t)h * 128 + hl * 8)
                          : make_uint4(0, 0, 0, 0);
    const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
    float v[8];
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] = __uint_as_float(wd[e] << 16);
      v[2 * e + 1] = __uint_as_float(wd[e] & 0xffff0000u);
      amax = fmaxf(amax, fmaxf(fabsf(v[2 * e]), fabsf(v[2 * e + 1])));
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1)
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    float sc = 1.f;
    if (amax > 0.f) {  // smallest power of two >= amax / 448
      const uint32_t ub = __float_as_uint(amax / 448.f);
      sc = (ub & 0x007fffffu) == 0 ? __uint_as_float(ub)
                                   : __uint_as_float((ub & 0x7f800000u) + 0x00800000u);
    }
    const float inv = 1.f / sc;  // exact: sc is a normal power of two
    uint32_t hi2[2] = {0u, 0u}, lo2[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = make_float2(v[2 * e] * inv, v[2 * e + 1] * inv);  // exact scaling
      const __nv_fp8x2_storage_t hc = __nv_cvt_float2_to_fp8x2(x, __NV_SATFINITE, __NV_E4M3);
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(hc, __NV_E4M3);
      const float2 hv = __half22float2(*reinterpret_cast<const __half2*>(&hr));
      const __nv_fp8x2_storage_t lc =
          __nv_cvt_float2_to_fp8x2(make_float2(x.x - hv.x, x.y - hv.y), __NV_SATFINITE, __NV_E4M3);
      hi2[e >> 1] |= (uint32_t)hc << (16 * (e & 1));
      lo2[e >> 1] |= (uint32_t)lc << (16 * (e & 1));
    }
    if (act) {
      const int dd = hl * 8, ch = dd >> 4;
      const int rh = decode_qop_row(h, 0, H), rl = decode_qop_row(h, 1, H);
      *reinterpret_cast<uint2*>(rec + rh * 128 + ((ch ^ (rh & 7)) * 16) + (dd & 15)) =
          make_uint2(hi2[0], hi2[1]);
      *reinterpret_cast<uint2*>(rec + rl * 128 + ((ch ^ (rl & 7)) * 16) + (dd & 15)) =
          make_uint2(lo2[0], lo2[1]);
      if (hl == 0) wout[h] = w[h] * sc;
    }
  }
}

__global__ void __launch_bounds__(1024) append_emit_kernel(csa_cache_desc d, CacheView cv,
                                                          const int64_t* __restrict__ pos,
                                                          csa_rows rows, csa_decode_params p,
                                                          const __nv_bfloat16* __restrict__ q_i,
                                                          const float* __restrict__ w_i,
                                                          uint8_t* __restrict__ qop,
                                                          uint32_t* __restrict__ ghist,
                                                          uint32_t* __restrict__ sel_done,
                                                          uint32_t* __restrict__ idx_done,
                                                          uint32_t* __restrict__ list_ready) {
  extern __shared__ float sx[];  // [c + c_i] + 32
  const int64_t b = blockIdx.x;
  // the previous step's kernels read the window slot this token overwrites
  sm100::pdl_wait();
  sm100::pdl_trigger();
  if (blockIdx.y == 1) {  // the indexer's query operand, for every sequence
    build_query_operand(q_i + b * d.nh_i * 128, w_i + b * d.nh_i, d.nh_i,
                        qop + b * decode_qop_bytes(d.nh_i));
    // the score histogram the indexer adds to, and the selection's count of
    // finished slices, start at zero
    if (ghist != nullptr) {
      uint4* gh = reinterpret_cast<uint4*>(ghist + b * kDecHistBins);
      for (int e = threadIdx.x; e < kDecHistBins / 4; e += blockDim.x) gh[e] = make_uint4(0, 0, 0, 0);
      if (threadIdx.x == 0) {
        sel_done[b] = 0u;
        idx_done[b] = 0u;
        list_ready[b] = 0u;
      }
    }
    return;
  }
  const int64_t t = pos[b];
  if (t < 0) return;  // no token for this sequence
  append_rows(d, cv, rows, b, t);
  if ((t + 1) % d.m != 0) return;  // uniform over the block
  __syncthreads();                 // the rows just written are read back below
  const int64_t i = t / d.m;
  if (i >= d.capacity) return;
  // one dim of the entry, or of the index key after it, per thread and round
  const int ndim = d.c + (d.is_hca ? 0 : d.c_i);
#pragma unroll 1
  for (int e = threadIdx.x; e < ndim; e += blockDim.x) {
    const bool key = e >= d.c;
    sx[e] = emit_dim(key ? cv.istate : cv.state, b, i, d.m, key ? d.c_i : d.c, key ? e - d.c : e,
                     key ? p.iba : p.ba, key ? p.ibb : p.bb, d.is_hca);
  }
  __syncthreads();
  float* red = sx + d.c + (d.is_hca ? 0 : d.c_i);
  const int64_t es = entry_row(cv, b, i, d.capacity);
  if (es < 0) return;  // no block for the emitted entry (uniform over the block)
  quantize_store(sx, d.c, d.rope_dims, cv.entry_fp8 + es * (d.c - d.rope_dims),
                 cv.entry_scale + es, cv.entry_rope + es * d.rope_dims, red);
  if (!d.is_hca)
    quantize_store(sx + d.c, d.c_i, 0, cv.ikey_fp8 + es * d.c_i, cv.ikey_scale + es, nullptr,
                   red);
}

// ---------------------------------------------------------------------------
// Step 2 (CSA): indexer over one chunk of visible keys + chunk-local top-k.
// ---------------------------------------------------------------------------
constexpr int kDecChunk = 2048;  // index keys per block

__global__ void __launch_bounds__(kSelThreads) index_chunk_kernel(
    csa_cache_desc d, CacheView cv, const int64_t* __restrict__ pos,
    const __nv_bfloat16* __restrict__ q_i, const float* __restrict__ w_i, int nchunks,
    float* __restrict__ cand_score, int32_t* __restrict__ cand_idx) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelectShared<kSelThreads>& sh = *reinterpret_cast<SelectShared<kSelThreads>*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(SelectShared<kSelThreads>));
  float* sc = reinterpret_cast<float*>(keys + kDecChunk);                          // [kDecChunk]
  int32_t* pick = reinterpret_cast<int32_t*>(sc + kDecChunk);                      // [k]
  float* qs = reinterpret_cast<float*>(pick + ((d.k + 3) & ~3));  // [c_i][nh_i]
  float* ws = qs + (size_t)d.c_i * d.nh_i;                        // [nh_i]
  const int chunk = blockIdx.x;
  const int64_t b = blockIdx.y;
  const int64_t t = max(pos[b], (int64_t)-1);
  const int64_t V = min((t + 1) / d.m, d.capacity);
  const int64_t c0 = (int64_t)chunk * kDecChunk;
  const int64_t Vc = max((int64_t)0, min((int64_t)kDecChunk, V - c0));
  float* osc = cand_score + ((int64_t)b * nchunks + chunk) * d.k;
  int32_t* oid = cand_idx + ((int64_t)b * nchunks + chunk) * d.k;
  if (Vc == 0) {
    for (int j = threadIdx.x; j < d.k; j += blockDim.x) { oid[j] = -1; osc[j] = 0.f; }
    return;
  }
  const int H = d.nh_i, ci = d.c_i;
  for (int e = threadIdx.x; e < H * ci; e += blockDim.x) {
    const int h = e / ci, dd = e % ci;
    qs[dd * H + h] = __bfloat162float(q_i[(b * H + h) * ci + dd]);
  }
  for (int h = threadIdx.x; h < H; h += blockDim.x) ws[h] = w_i[b * H + h];
  __syncthreads();
  for (int64_t e = threadIdx.x; e < Vc; e += blockDim.x) {
    const int64_t s = c0 + e;
    const int64_t er = entry_row(cv, b, s, d.capacity);
    if (er < 0) {  // no block: the entry scores 0
      sc[e] = 0.f;
      keys[e] = order_key(0.f);
      continue;
    }
    const uint8_t* kr = cv.ikey_fp8 + er * ci;
    const float ks = cv.ikey_scale[er];
    float score = 0.f;
    for (int hg = 0; hg < H; hg += 32) {
      float acc[32];
#pragma unroll
      for (int h = 0; h < 32; ++h) acc[h] = 0.f;
      for (int dd = 0; dd < ci; dd += 16) {
        const uint4 raw = *reinterpret_cast<const uint4*>(kr + dd);
        const uint8_t* by = reinterpret_cast<const uint8_t*>(&raw);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float kv = e4m3_value(by[u]);
          const float* qrow = qs + (dd + u) * H + hg;
#pragma unroll
          for (int h = 0; h < 32; ++h)
            if (hg + h < H) acc[h] = fmaf(qrow[h], kv, acc[h]);
        }
      }
#pragma unroll
      for (int h = 0; h < 32; ++h)
        if (hg + h < H) score = fmaf(ws[hg + h], fmaxf(acc[h] * ks, 0.f), score);
    }
    sc[e] = score;
    keys[e] = order_key(score);
  }
  __syncthreads();
  if (Vc <= d.k) {
    for (int j = threadIdx.x; j < d.k; j += blockDim.x) {
      oid[j] = j < Vc ? (int32_t)(c0 + j) : -1;
      osc[j] = j < Vc ? sc[j] : 0.f;
    }
    return;
  }
  block_select_topk<kSelThreads>(KeysInSmem{keys}, Vc, d.k, pick, nullptr, sh);
  for (int j = threadIdx.x; j < d.k; j += blockDim.x) {
    const int32_t pp = pick[j];
    oid[j] = (int32_t)(c0 + pp);
    osc[j] = sc[pp];
  }
}

// Step 3 (CSA): top-k over all chunk candidates (ascending entry order).
__global__ void __launch_bounds__(kSelThreads) topk_merge_kernel(
    csa_cache_desc d, const int64_t* __restrict__ pos, int nchunks,
    const float* __restrict__ cand_score, const int32_t* __restrict__ cand_idx,
    int32_t* __restrict__ sel) {
  __shared__ SelectShared<kSelThreads> sh;
  const int64_t b = blockIdx.x;
  const int64_t t = pos[b];
  const int64_t V = min((t + 1) / d.m, d.capacity);
  int32_t* out = sel + b * d.k;
  if (t < 0 || V <= d.k) {
    for (int j = threadIdx.x; j < d.k; j += blockDim.x) out[j] = j < V ? j : -1;
    return;
  }
  const int64_t N = (int64_t)nchunks * d.k;
  const float* s = cand_score + b * N;
  const int32_t* id = cand_idx + b * N;
  block_select_topk<kSelThreads>(CandidatesInGlobal{s, id}, N, d.k, out, id, sh);
}

// Step 3' (CSA, tensor-core indexer), capacities beyond the cluster top-k:
// top-k over one sequence's score array in global memory.
__global__ void __launch_bounds__(kDecSelThreads) decode_select_kernel(
    csa_cache_desc d, const int64_t* __restrict__ pos, const float* __restrict__ scores,
    int32_t* __restrict__ sel) {
  __shared__ SelectShared<kDecSelThreads> sh;
  const int64_t b = blockIdx.x;
  const int64_t t = pos[b];
  const int64_t V = t < 0 ? 0 : min((t + 1) / d.m, d.capacity);
  int32_t* out = sel + b * d.k;
  if (V <= d.k) {
    for (int j = threadIdx.x; j < d.k; j += kDecSelThreads) out[j] = j < V ? j : -1;
    return;
  }
  block_select_topk<kDecSelThreads>(ScoresIn{scores + b * d.capacity}, V, d.k, out, nullptr, sh);
}

// ---------------------------------------------------------------------------
// Steps 4-5: split attention over (selected | all visible) entries + window.
// ---------------------------------------------------------------------------
constexpr int kDecHG = 8;   // heads per block (one warp each)
constexpr int kDecTE = 32;  // entries per tile

__global__ void __launch_bounds__(256) attn_split_kernel(
    csa_cache_desc d, CacheView cv, const int64_t* __restrict__ pos,
    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ sel, float scale,
    int nsplit, float* __restrict__ part_o, float* __restrict__ part_ms) {
  extern __shared__ float smem[];
  const int c = d.c, ld = c + 1;
  float* Es = smem;                      // [kDecTE][c+1]
  float* Qs = Es + kDecTE * ld;          // [kDecHG][c]
  float* Ps = Qs + kDecHG * c;           // [kDecHG][kDecTE]
  int64_t* rows = reinterpret_cast<int64_t*>(Ps + kDecHG * kDecTE);  // [kDecTE]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, h0 = blockIdx.y * kDecHG;
  const int64_t b = blockIdx.z;
  const int64_t t = max(pos[b], (int64_t)-1);  // t = -1: nothing to attend
  const int64_t V = max((int64_t)0, min((t + 1) / d.m, d.capacity));
  const int64_t w0 = max((int64_t)0, t - d.window + 1);
  const int64_t n_comp = t < 0 ? 0 : (d.is_hca ? V : (int64_t)d.k);
  const int64_t N = n_comp + max((int64_t)0, t - w0 + 1);
  const int64_t j_lo = N * split / nsplit, j_hi = N * (split + 1) / nsplit;
  const float qscale = scale * kLog2e;
  for (int e = tid; e < kDecHG * c; e += 256) {
    const int h = e / c, dd = e % c;
    Qs[e] = (h0 + h < d.nh) ? __bfloat162float(q[(b * d.nh + h0 + h) * c + dd]) * qscale : 0.f;
  }
  const int body = c - d.rope_dims;
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.f;
  float run_max = kNegInf, run_sum = 0.f;
  for (int64_t j0 = j_lo; j0 < j_hi; j0 += kDecTE) {
    __syncthreads();
    if (tid < kDecTE) {
      const int64_t j = j0 + tid;
      int64_t row = -1;
      if (j < j_hi) {
        if (j < n_comp) {
          const int64_t s = d.is_hca ? j : (int64_t)sel[b * d.k + j];
          if (s >= 0 && s < V) row = s;
        } else {
          row = d.capacity + (w0 + (j - n_comp)) % d.window;  // ring slot, offset
        }
      }
      rows[tid] = row;
    }
    __syncthreads();
    const int per_row = c / 8;
    for (int e = tid; e < kDecTE * per_row; e += 256) {
      const int r = e / per_row, dd = (e % per_row) * 8;
      const int64_t row = rows[r];
      float v[8];
      if (row < 0) {
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = 0.f;
      } else if (row < d.capacity) {
        const int64_t es = entry_row(cv, b, row, d.capacity);
        if (es < 0) {
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = 0.f;
        } else if (dd < body) {
          const float sc = cv.entry_scale[es];
          const uint2 raw = *reinterpret_cast<const uint2*>(cv.entry_fp8 + es * body + dd);
          const uint8_t* by = reinterpret_cast<const uint8_t*>(&raw);
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = e4m3_value(by[u]) * sc;
        } else {
          load8_cg(cv.entry_rope + es * d.rope_dims + (dd - body), v);
        }
      } else {
        load8_cg(cv.window + (b * d.window + (row - d.capacity)) * c + dd, v);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) Es[r * ld + dd + u] = v[u];
    }
    __syncthreads();
    {
      const float* qh = Qs + warp * c;
      const float* er = Es + lane * ld;
      float dot = 0.f;
      for (int dd = 0; dd < c; ++dd) dot = fmaf(qh[dd], er[dd], dot);
      const float l = rows[lane] >= 0 ? dot : kNegInf;
      float mx = l;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float new_max = fmaxf(run_max, mx);
      const float pj = new_max == kNegInf ? 0.f : ex2(l - new_max);
      float ps = pj;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      const float f = run_max == kNegInf ? 0.f : ex2(run_max - new_max);
      run_sum = run_sum * f + ps;
      run_max = new_max;
      Ps[warp * kDecTE + lane] = pj;
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] *= f;
    }
    __syncwarp();
    const int nd = c / 32;
    for (int e = 0; e < kDecTE; ++e) {
      const float pj = Ps[warp * kDecTE + e];
      const float* er = Es + e * ld + lane;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < nd) acc[j] = fmaf(pj, er[32 * j], acc[j]);
    }
  }
  const int h = h0 + warp;
  if (h < d.nh) {
    const int64_t base = (b * nsplit + split) * d.nh + h;
    float* o = part_o + base * c;
    const int nd = c / 32;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < nd) o[lane + 32 * j] = acc[j];
    if (lane == 0) {
      part_ms[base * 2 + 0] = run_max;
      part_ms[base * 2 + 1] = run_sum;
    }
  }
}

__global__ void __launch_bounds__(256) attn_combine_kernel(
    csa_cache_desc d, const float* __restrict__ sink, int nsplit, const float* __restrict__ part_o,
    const float* __restrict__ part_ms, __nv_bfloat16* __restrict__ out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t b = blockIdx.x;
  const int h = blockIdx.y * 8 + warp;
  if (h >= d.nh) return;
  const int c = d.c;
  float M = sink ? sink[h] * kLog2e : kNegInf;
  for (int sp = 0; sp < nsplit; ++sp)
    M = fmaxf(M, part_ms[((b * nsplit + sp) * d.nh + h) * 2]);
  float den = sink ? ex2(sink[h] * kLog2e - M) : 0.f;
  for (int dd = lane; dd < c; dd += 32) {
    float o = 0.f;
    for (int sp = 0; sp < nsplit; ++sp) {
      const int64_t base = (b * nsplit + sp) * d.nh + h;
      const float mi = part_ms[base * 2];
      if (mi == kNegInf) continue;
      o = fmaf(ex2(mi - M), part_o[base * c + dd], o);
    }
    if (dd == lane) {  // first pass also sums the denominators (same for all dd)
      float s = 0.f;
      for (int sp = 0; sp < nsplit; ++sp) {
        const int64_t base = (b * nsplit + sp) * d.nh + h;
        const float mi = part_ms[base * 2];
        if (mi != kNegInf) s = fmaf(ex2(mi - M), part_ms[base * 2 + 1], s);
      }
      den += s;
    }
    out[(b * d.nh + h) * c + dd] = __float2bfloat16_rn(o / den);
  }
}

// ---------------------------------------------------------------------------
struct DecodeWs {
  int nchunks, nsplit;
  bool tc_index, tc_attn, hist_select, attn_select;
  size_t cand_score, cand_idx, scores, qop, sel, part_o, part_ms, select, total;
};

static DecodeWs decode_ws_layout(const csa_cache_desc& d) {
  DecodeWs w;
  w.tc_index = decode_index_tc_supported(d);
  w.nchunks = (d.is_hca || w.tc_index) ? 0 : (int)((d.capacity + kDecChunk - 1) / kDecChunk);
  const int64_t max_slots = (d.is_hca ? d.capacity : (int64_t)d.k) + d.window;
  w.tc_attn = decode_attn_tc_supported(d);
  w.nsplit = w.tc_attn ? decode_attn_splits(d)
                       : (int)std::min<int64_t>(128, std::max<int64_t>(1, (max_slots + 63) / 64));
  const size_t B = (size_t)d.batch;
  size_t off = 0;
  w.cand_score = off; off = align256(off + B * w.nchunks * d.k * 4);
  w.cand_idx = off;   off = align256(off + B * w.nchunks * d.k * 4);
  w.scores = off;     off = align256(off + (w.tc_index ? B * (size_t)d.capacity * 4 : 0));
  w.qop = off;        off = align256(off + (w.tc_index ? B * decode_qop_bytes(d.nh_i) : 0));
  w.sel = off;        off = align256(off + B * (d.is_hca ? 0 : d.k) * 4);
  w.part_o = off;     off = align256(off + B * w.nsplit * d.nh * (size_t)d.c * 4);
  w.part_ms = off;    off = align256(off + B * w.nsplit * d.nh * 2 * 4);
  w.hist_select = w.tc_index && decode_select_supported(d);
  // the attention kernel takes the top-k itself where the scores fit its
  // shared memory; the selection kernel otherwise
  w.attn_select = w.hist_select && w.tc_attn && decode_attn_selects(d);
  size_t sel_bytes = 0;
  if (w.hist_select) decode_select_ws(d, nullptr, &sel_bytes);
  w.select = off;     off = align256(off + sel_bytes);
  w.total = off;
  return w;
}

size_t decode_workspace(const csa_cache_desc& d) { return decode_ws_layout(d).total; }

cudaError_t launch_decode_step(const csa_cache_desc& d, const CacheView& cv, const int64_t* pos,
                               const csa_rows& rows, const csa_decode_params& p, const void* q,
                               const void* q_i, const float* w_i, void* out, void* ws,
                               cudaStream_t s) {
  const DecodeWs w = decode_ws_layout(d);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  float* cand_score = reinterpret_cast<float*>(wb + w.cand_score);
  int32_t* cand_idx = reinterpret_cast<int32_t*>(wb + w.cand_idx);
  int32_t* sel = p.sel_out != nullptr ? p.sel_out : reinterpret_cast<int32_t*>(wb + w.sel);
  float* part_o = reinterpret_cast<float*>(wb + w.part_o);
  float* part_ms = reinterpret_cast<float*>(wb + w.part_ms);

  // one thread per emitted dim (c + c_i of them), 256 to 1024 threads; with
  // the indexer's query operand, a second block per sequence builds it (one
  // half-warp per head)
  const int dims = d.c + (d.is_hca ? 0 : d.c_i);
  uint8_t* qop = w.tc_index ? wb + w.qop : nullptr;
  const int want = std::max(dims, qop != nullptr ? d.nh_i * 16 : 0);
  const unsigned emit_threads = (unsigned)std::min(1024, std::max(256, (want + 31) / 32 * 32));
  const size_t emit_smem = sizeof(float) * (dims + 32);
  size_t sel_bytes = 0;
  const DecodeSelectWs sws =
      decode_select_ws(d, w.hist_select ? wb + w.select : nullptr, &sel_bytes);
  cudaError_t err = launch_pdl(append_emit_kernel,
                               dim3((unsigned)d.batch, qop != nullptr ? 2u : 1u),
                               dim3(emit_threads), emit_smem, s, d, cv, pos, rows, p,
                               (const __nv_bfloat16*)q_i, w_i, qop, sws.ghist, sws.done,
                               sws.idx_done, sws.list_ready);
  if (err != cudaSuccess) return err;
  if (!d.is_hca && w.tc_index) {
    float* scores = p.scores_out != nullptr ? p.scores_out : reinterpret_cast<float*>(wb + w.scores);
    unsigned int* flag = device_timeout_flag();
    if (flag == nullptr) return cudaErrorUnknown;
    // (sws.ghist is NULL when the selection below does not use it: the
    // indexer then keeps no histogram)
    err = launch_decode_index_tc(d, cv, pos, qop, scores, sws.ghist,
                                 w.attn_select ? sws.idx_done : nullptr, flag, s);
    if (err != cudaSuccess) return err;
    if (w.attn_select) {
      err = cudaSuccess;  // the attention kernel selects
    } else if (w.hist_select) {
      err = launch_decode_select(d, pos, scores, sws, sel, s);
    } else {
      decode_select_kernel<<<(unsigned)d.batch, kDecSelThreads, 0, s>>>(d, pos, scores, sel);
      err = cudaGetLastError();
    }
    if (err != cudaSuccess) return err;
  } else if (!d.is_hca) {
    const size_t smem = sizeof(SelectShared<kSelThreads>) + (size_t)kDecChunk * 8 +
                        (size_t)((d.k + 3) & ~3) * 4 + (size_t)d.c_i * d.nh_i * 4 +
                        (size_t)d.nh_i * 4;
    cudaFuncSetAttribute(index_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    index_chunk_kernel<<<dim3(w.nchunks, (unsigned)d.batch), kSelThreads, smem, s>>>(
        d, cv, pos, (const __nv_bfloat16*)q_i, w_i, w.nchunks, cand_score, cand_idx);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    topk_merge_kernel<<<(unsigned)d.batch, kSelThreads, 0, s>>>(d, pos, w.nchunks, cand_score,
                                                                cand_idx, sel);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  const unsigned hgroups = (unsigned)((d.nh + kDecHG - 1) / kDecHG);
  if (w.tc_attn) {
    unsigned int* flag = device_timeout_flag();
    if (flag == nullptr) return cudaErrorUnknown;
    const float* ascores = nullptr;
    if (w.attn_select)
      ascores = p.scores_out != nullptr ? p.scores_out : reinterpret_cast<float*>(wb + w.scores);
    return launch_decode_attn_tc(d, cv, pos, q, w.attn_select ? nullptr : sel, p.sink, p.scale,
                                 w.nsplit, out, part_o, part_ms, ascores,
                                 w.attn_select ? sws.ghist : nullptr,
                                 w.attn_select ? p.sel_out : nullptr,
                                 w.attn_select ? sws.idx_done : nullptr,
                                 decode_index_tile_keys(d),
                                 w.attn_select ? reinterpret_cast<int32_t*>(wb + w.sel) : nullptr,
                                 w.attn_select ? sws.list_ready : nullptr, flag, s);
  }
  const size_t asmem = sizeof(float) * ((size_t)kDecTE * (d.c + 1) + (size_t)kDecHG * d.c +
                                        kDecHG * kDecTE) + sizeof(int64_t) * kDecTE;
  cudaFuncSetAttribute(attn_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)asmem);
  attn_split_kernel<<<dim3(w.nsplit, hgroups, (unsigned)d.batch), 256, asmem, s>>>(
      d, cv, pos, (const __nv_bfloat16*)q, sel, p.scale, w.nsplit, part_o, part_ms);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  attn_combine_kernel<<<dim3((unsigned)d.batch, hgroups), 256, 0, s>>>(
      d, p.sink, w.nsplit, part_o, part_ms, (__nv_bfloat16*)out);
  return cudaGetLastError();
}

}  // namespace csa
