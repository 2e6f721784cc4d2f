// Core attention on CUDA cores: shared-KV MQA over an explicit entry set with
// the attention sink in the softmax denominator (fp32 path and the shapes the
// tcgen05 kernel in attn_tc.cu does not take).
//
// For query t and head h, E_t is (CSA) the selected compressed entries
// idx[t, :] that are visible (0 <= s < floor((t+1)/m)), or (HCA) every
// visible compressed entry, followed by the raw window rows
// max(0, t-W+1) .. t.  Every entry is both key and value:
//   o = sum_j exp(l_j) e_j / (exp(sink_h) + sum_j exp(l_j)),  l_j = scale q.e_j
// (sections 4.3 and 4.5 of "DeepSeek-V4: million-token context"; B9 of the
// "Core formulas chapter"; one softmax for window, compressed entries and
// sink, as the reader's notes stress in section 1).
//
// One block = one query x 8 heads (one warp per head).  Entries are gathered
// 32 at a time into shared memory; the softmax is online (running max/sum per
// head) in the log2 domain (q is pre-scaled by scale*log2(e)).
#include "common.cuh"
#include "launch.h"
#include "rope.cuh"

namespace csa {

constexpr int kAttnThreads = 256;
constexpr int kAttnHG = kAttnThreads / 32;  // heads per block
constexpr int kAttnTE = 32;                 // entries per tile

template <typename T>
__global__ void __launch_bounds__(kAttnThreads) attn_kernel(
    const T* __restrict__ q, const T* __restrict__ kv_comp, const int32_t* __restrict__ idx,
    int k, const T* __restrict__ kv_win, int window, const float* __restrict__ sink,
    float scale, int64_t n, int nh, int c, int m, int64_t E, QNormRope qn,
    T* __restrict__ out) {
  extern __shared__ float smem[];
  const int ld = c + 1;
  float* Es = smem;                              // [kAttnTE][c+1]
  float* Qs = Es + kAttnTE * ld;                 // [kAttnHG][c]
  float* Ps = Qs + kAttnHG * c;                  // [kAttnHG][kAttnTE]
  int64_t* rows = reinterpret_cast<int64_t*>(Ps + kAttnHG * kAttnTE);  // [kAttnTE] (-1 = skip)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t = blockIdx.x, b = blockIdx.z;
  const int h0 = blockIdx.y * kAttnHG;
  const int64_t V = min((t + 1) / m, E);
  const int64_t w0 = max((int64_t)0, t - window + 1);
  const int64_t n_comp = idx ? (int64_t)k : V;   // compressed slots
  const int64_t N = n_comp + (t - w0 + 1);       // total slots

  const float qscale = scale * kLog2e;
  for (int e = tid; e < kAttnHG * c; e += kAttnThreads) {
    const int h = e / c, d = e % c;
    const float x = (h0 + h < nh) ? to_f32(q[((b * n + t) * nh + h0 + h) * c + d]) : 0.f;
    Qs[e] = qn.gamma != nullptr ? x : x * qscale;
  }
  const int my_h = h0 + warp;
  if (qn.gamma != nullptr) {
    // the query head's RMSNorm and rotation for position t (warp = head)
    __syncthreads();
    float* qh = Qs + warp * c;
    float ss = 0.f;
    for (int d = lane; d < c; d += 32) ss = fmaf(qh[d], qh[d], ss);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = 1.f / sqrtf(ss / (float)c + qn.eps);
    __syncwarp();
    for (int d = lane; d < c; d += 32) qh[d] = qh[d] * inv * __ldg(qn.gamma + d);
    __syncwarp();
    for (int j = lane; j < qn.rope_dims / 2; j += 32) {
      float cs, sn;
      rope_cos_sin(t, j, qn.rope_dims, qn.base, cs, sn);
      const int d = c - qn.rope_dims + 2 * j;
      rope_turn(qh[d], qh[d + 1], cs, sn);
    }
    __syncwarp();
    for (int d = lane; d < c; d += 32) qh[d] *= qscale;
  }
  const int nd = c / 32;  // dims per thread (c % 32 == 0 here; see launcher)
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.f;
  float run_max = kNegInf, run_sum = 0.f;

  for (int64_t j0 = 0; j0 < N; j0 += kAttnTE) {
    __syncthreads();  // previous tile consumed
    if (tid < kAttnTE) {
      const int64_t j = j0 + tid;
      int64_t row = -1;
      if (j < N) {
        if (j < n_comp) {
          const int64_t s = idx ? (int64_t)idx[(b * n + t) * k + j] : j;
          if (s >= 0 && s < V) row = s;                // compressed entry s
        } else {
          row = E + w0 + (j - n_comp);                 // window row, offset by E
        }
      }
      rows[tid] = row;
    }
    __syncthreads();
    // gather the tile (8 elements per thread per step)
    const int per_row = c / 8;
    for (int e = tid; e < kAttnTE * per_row; e += kAttnThreads) {
      const int r = e / per_row, d = (e % per_row) * 8;
      const int64_t row = rows[r];
      float v[8];
      if (row < 0) {
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) v[q8] = 0.f;
      } else if (row < E) {
        load8(kv_comp + (b * E + row) * c + d, v);
      } else {
        load8(kv_win + (b * n + (row - E)) * c + d, v);
      }
#pragma unroll
      for (int q8 = 0; q8 < 8; ++q8) Es[r * ld + d + q8] = v[q8];
    }
    __syncthreads();
    // logits: warp = head, lane = entry
    {
      const float* qh = Qs + warp * c;
      const float* er = Es + lane * ld;
      float dot = 0.f;
      for (int d = 0; d < c; ++d) dot = fmaf(qh[d], er[d], dot);
      const float l = rows[lane] >= 0 ? dot : kNegInf;
      float mx = l;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float new_max = fmaxf(run_max, mx);
      const float p = new_max == kNegInf ? 0.f : ex2(l - new_max);
      float ps = p;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      const float f = run_max == kNegInf ? 0.f : ex2(run_max - new_max);
      run_sum = run_sum * f + ps;
      run_max = new_max;
      Ps[warp * kAttnTE + lane] = p;
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] *= f;
    }
    __syncwarp();
    // accumulate o[h][lane + 32 j] += sum_e p_e * E[e][lane + 32 j]
    for (int e = 0; e < kAttnTE; ++e) {
      const float p = Ps[warp * kAttnTE + e];
      const float* er = Es + e * ld + lane;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < nd) acc[j] = fmaf(p, er[32 * j], acc[j]);
    }
  }
  if (my_h < nh) {
    const float z = sink ? sink[my_h] * kLog2e : kNegInf;
    const float den = run_sum + (z == kNegInf ? 0.f : ex2(z - run_max));
    const float inv = 1.f / den;
    T* o = out + ((b * n + t) * nh + my_h) * c;
    if (qn.gamma != nullptr && qn.rope_dims > 0) {
      // the output's trailing dims turned back by position -t: dims lane + 32 j
      // pair with their neighbour lane (lane ^ 1)
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int d = lane + 32 * j;
        const float other = __shfl_xor_sync(0xffffffffu, acc[j], 1);
        if (j < nd && d >= c - qn.rope_dims) {
          float cs, sn;
          rope_cos_sin(-t, (d - (c - qn.rope_dims)) >> 1, qn.rope_dims, qn.base, cs, sn);
          acc[j] = (lane & 1) == 0 ? acc[j] * cs - other * sn : other * sn + acc[j] * cs;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < nd) from_f32(o[lane + 32 * j], acc[j] * inv);
  }
}

cudaError_t launch_attn(const void* q, const void* kv_comp, const int32_t* idx, int k,
                        const void* kv_win, int window, const float* sink, float scale,
                        int64_t batch, int64_t n, int nh, int c, int m, csa_dtype dt,
                        const csa_norm_rope* q_nr, void* out, cudaStream_t s) {
  const int64_t E = n / m;
  const QNormRope qn = q_nr != nullptr
                           ? QNormRope{q_nr->gamma, q_nr->eps, q_nr->rope_dims, q_nr->rope_base}
                           : QNormRope{nullptr, 0.f, 0, 0.f};
  if (attn_tc_supported(nh, c, idx ? k : 0, dt, q, kv_comp ? kv_comp : q, kv_win,
                        qn.gamma != nullptr ? qn.rope_dims : 0)) {
    unsigned int* err = device_timeout_flag();
    if (err == nullptr) return cudaErrorUnknown;
    return launch_attn_tc(q, kv_comp, idx, k, kv_win, window, sink, scale, batch, n, m, qn, out,
                          err, s);
  }
  const size_t smem = sizeof(float) * ((size_t)kAttnTE * (c + 1) + (size_t)kAttnHG * c +
                                       kAttnHG * kAttnTE) + sizeof(int64_t) * kAttnTE;
  dim3 grid((unsigned)n, (unsigned)((nh + kAttnHG - 1) / kAttnHG), (unsigned)batch);
  if (dt == CSA_F32) {
    auto kern = attn_kernel<float>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kAttnThreads, smem, s>>>((const float*)q, (const float*)kv_comp, idx, k,
                                          (const float*)kv_win, window, sink, scale, n, nh, c,
                                          m, E, qn, (float*)out);
  } else {
    auto kern = attn_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kAttnThreads, smem, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)kv_comp, idx, k,
        (const __nv_bfloat16*)kv_win, window, sink, scale, n, nh, c, m, E, qn,
        (__nv_bfloat16*)out);
  }
  return cudaGetLastError();
}

}  // namespace csa
