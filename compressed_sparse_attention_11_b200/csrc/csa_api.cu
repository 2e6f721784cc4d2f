// C ABI of the CSA/HCA attention layer: argument checks, then launches.
// Every entry point validates before enqueuing anything on the stream and
// never allocates, frees or synchronises.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "launch.h"

using namespace csa;

namespace {

thread_local char g_err[512] = "";

csa_status fail(csa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

csa_status ok() {
  g_err[0] = '\0';
  return CSA_OK;
}

csa_status cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return ok();
  return fail(CSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE(cond, ...) \
  do { if (!(cond)) return fail(CSA_ERR_INVALID_ARG, __VA_ARGS__); } while (0)
#define REQUIRE_PTR(p) \
  do { \
    if ((p) == nullptr) return fail(CSA_ERR_INVALID_ARG, "%s is NULL", #p); \
    if (!aligned16(p)) return fail(CSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
  } while (0)
#define REQUIRE_OPT_PTR(p) \
  do { \
    if ((p) != nullptr && !aligned16(p)) \
      return fail(CSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
  } while (0)

bool valid_dt(csa_dtype dt) { return dt == CSA_F32 || dt == CSA_BF16; }

constexpr size_t kMaxSmem = 227 * 1024;

csa_status check_attn_common(const void* q, const void* kv_comp, const void* kv_win, int window,
                             float scale, int64_t batch, int64_t n, int nh, int c, int m,
                             csa_dtype dt, const void* out, const float* sink) {
  REQUIRE(valid_dt(dt), "dt must be CSA_F32 or CSA_BF16");
  REQUIRE(batch >= 0 && n >= 0, "batch and n must be >= 0");
  REQUIRE(nh >= 1, "nh must be >= 1");
  REQUIRE(c >= 8 && c % 8 == 0, "c must be a positive multiple of 8");
  REQUIRE(m >= 1, "m must be >= 1");
  REQUIRE(window >= 1, "window must be >= 1");
  REQUIRE(scale == scale && scale > -3.4e38f && scale < 3.4e38f, "scale must be finite");
  if (batch == 0 || n == 0) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(kv_win);
  REQUIRE_PTR(out);
  REQUIRE_OPT_PTR(sink);
  if (n / m > 0) REQUIRE_PTR(kv_comp);
  if (c % 32 != 0 || c > 512) return fail(CSA_ERR_UNSUPPORTED, "attention needs c %% 32 == 0 and c <= 512");
  return ok();
}

csa_status check_desc(const csa_cache_desc* d) {
  REQUIRE(d != nullptr, "desc is NULL");
  REQUIRE(d->batch >= 1 && d->capacity >= 1, "batch and capacity must be >= 1");
  REQUIRE(d->c >= 32 && d->c % 32 == 0, "c must be a positive multiple of 32");
  REQUIRE(d->rope_dims >= 0 && d->rope_dims < d->c && d->rope_dims % 8 == 0,
          "rope_dims must be in [0, c) and a multiple of 8");
  REQUIRE((d->c - d->rope_dims) % 16 == 0, "c - rope_dims must be a multiple of 16");
  REQUIRE(d->m >= 1, "m must be >= 1");
  REQUIRE(d->window >= 1, "window must be >= 1");
  REQUIRE(d->nh >= 1, "nh must be >= 1");
  REQUIRE(d->is_hca == 0 || d->is_hca == 1, "is_hca must be 0 or 1");
  if (!d->is_hca) {
    REQUIRE(d->c_i >= 16 && d->c_i % 16 == 0, "c_i must be a positive multiple of 16");
    REQUIRE(d->nh_i >= 1, "nh_i must be >= 1");
    REQUIRE(d->k >= 1, "k must be >= 1");
  }
  if (d->c > 512) return fail(CSA_ERR_UNSUPPORTED, "decode attention needs c <= 512");
  return ok();
}

csa_status check_norm_rope(const csa_norm_rope* nr, int c) {
  REQUIRE(nr != nullptr, "nr is NULL");
  REQUIRE_PTR(nr->gamma);
  REQUIRE(nr->eps >= 0.f && nr->eps < 3.4e38f, "eps must be finite and >= 0");
  REQUIRE(nr->rope_dims >= 0 && nr->rope_dims <= c && nr->rope_dims % 8 == 0,
          "rope_dims must be a multiple of 8 in [0, c]");
  REQUIRE(nr->rope_base > 1.f && nr->rope_base < 3.4e38f, "rope_base must be finite and > 1");
  return ok();
}

}  // namespace

namespace {
// Set (bit OR) by kernels whose bounded waits expired; read by csa_check.
static __device__ unsigned int g_timeout_flag;
constexpr int kMaxDev = 64;
std::mutex g_flag_mu;
unsigned int* g_flag_ptr[kMaxDev] = {};
}  // namespace

unsigned int* csa::device_timeout_flag() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  std::lock_guard<std::mutex> lock(g_flag_mu);
  if (g_flag_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_timeout_flag) != cudaSuccess) return nullptr;
    g_flag_ptr[dev] = static_cast<unsigned int*>(p);
  }
  return g_flag_ptr[dev];
}

csa_status csa::set_last_error(csa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

extern "C" {

const char* csa_status_string(int status) {
  switch (status) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID_ARG: return "CSA_ERR_INVALID_ARG";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED";
    case CSA_ERR_WORKSPACE: return "CSA_ERR_WORKSPACE";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA";
    case CSA_ERR_TIMEOUT: return "CSA_ERR_TIMEOUT";
    default: return "CSA_ERR_UNKNOWN";
  }
}

const char* csa_last_error(void) { return g_err; }

int csa_abi_version(void) { return 2; }

csa_status csa_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e, "csa_check");
  unsigned int* flag = device_timeout_flag();
  if (flag == nullptr) return fail(CSA_ERR_CUDA, "csa_check: no device flag");
  unsigned int v = 0;
  e = cudaMemcpy(&v, flag, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_status(e, "csa_check");
  if (v != 0) {
    const unsigned int zero = 0;
    cudaMemcpy(flag, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    return fail(CSA_ERR_TIMEOUT, "a kernel gave up a bounded wait; its outputs are invalid");
  }
  return ok();
}

csa_status csa_selftest_wait(uint32_t limit_us, int arrive, void* stream) {
  if (limit_us < 1 || limit_us > 2000000u)
    return fail(CSA_ERR_INVALID_ARG, "csa_selftest_wait: limit_us out of range");
  unsigned int* flag = device_timeout_flag();
  if (flag == nullptr) return fail(CSA_ERR_CUDA, "csa_selftest_wait: no device flag");
  return cuda_status(launch_selftest_wait(limit_us, arrive != 0, flag, (cudaStream_t)stream),
                     "csa_selftest_wait");
}

csa_status csa_compress(const void* ca, const void* cb, const void* za, const void* zb,
                        const float* ba, const float* bb, int64_t batch, int64_t n, int c,
                        int m, int overlap, csa_dtype dt, void* out, void* stream) {
  REQUIRE(valid_dt(dt), "dt must be CSA_F32 or CSA_BF16");
  REQUIRE(batch >= 0 && n >= 0, "batch and n must be >= 0");
  REQUIRE(c >= 8 && c % 8 == 0, "c must be a positive multiple of 8");
  REQUIRE(m >= 1, "m must be >= 1");
  REQUIRE(overlap == 0 || overlap == 1, "overlap must be 0 or 1");
  if (!overlap)
    REQUIRE(cb == nullptr && zb == nullptr && bb == nullptr,
            "cb, zb and bb must be NULL when overlap == 0");
  if (batch == 0 || n / m == 0) return ok();
  REQUIRE_PTR(ca);
  REQUIRE_PTR(za);
  REQUIRE_PTR(ba);
  REQUIRE_PTR(out);
  if (overlap) {
    REQUIRE_PTR(cb);
    REQUIRE_PTR(zb);
    REQUIRE_PTR(bb);
  }
  return cuda_status(launch_compress(ca, cb, za, zb, ba, bb, batch, n, c, m, overlap, dt, nullptr, out,
                                     (cudaStream_t)stream),
                     "csa_compress");
}

size_t csa_index_topk_workspace(int64_t batch, int64_t n, int nh_i, int c_i, int m, int k) {
  (void)nh_i; (void)c_i; (void)k;
  if (batch <= 0 || n <= 0 || m <= 0) return 0;
  const int64_t E = n / m;
  return (size_t)batch * (size_t)n * (size_t)E * sizeof(float);
}

csa_status csa_index_topk(const void* q_i, const float* w_i, const void* k_i, int64_t batch,
                          int64_t n, int nh_i, int c_i, int m, int k, csa_dtype dt,
                          int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
  REQUIRE(valid_dt(dt), "dt must be CSA_F32 or CSA_BF16");
  REQUIRE(batch >= 0 && n >= 0, "batch and n must be >= 0");
  REQUIRE(nh_i >= 1, "nh_i must be >= 1");
  REQUIRE(c_i >= 8 && c_i % 8 == 0, "c_i must be a positive multiple of 8");
  REQUIRE(m >= 1, "m must be >= 1");
  REQUIRE(k >= 1, "k must be >= 1");
  if (batch == 0 || n == 0) return ok();
  REQUIRE_PTR(idx);
  const int64_t E = n / m;
  if (E > 0) {
    REQUIRE_PTR(q_i);
    REQUIRE_PTR(w_i);
    REQUIRE_PTR(k_i);
    const int nh_pad = (nh_i + 31) / 32 * 32;
    if ((size_t)c_i * (128 + nh_pad) * 4 > kMaxSmem)
      return fail(CSA_ERR_UNSUPPORTED, "indexer tile for c_i=%d, nh_i=%d exceeds shared memory",
                  c_i, nh_i);
    const size_t need = csa_index_topk_workspace(batch, n, nh_i, c_i, m, k);
    if (ws_bytes < need || ws == nullptr)
      return fail(CSA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, need);
    REQUIRE_PTR(ws);
  }
  cudaStream_t s = (cudaStream_t)stream;
  float* scores = static_cast<float*>(ws);
  if (E > 0) {
    cudaError_t e = launch_index_scores(q_i, w_i, k_i, batch, n, nh_i, c_i, m, dt, scores, E, s);
    if (e != cudaSuccess) return cuda_status(e, "csa_index_topk (scores)");
  }
  return cuda_status(launch_topk_rows(scores, E, batch, n, m, E, k, idx, s),
                     "csa_index_topk (top-k)");
}

namespace {
// Workspace regions of the low-precision indexer (byte offsets, 256-aligned).
struct LowpWs {
  size_t scores, q8, qs, k8, ks, total;
};
LowpWs lowp_ws(int64_t batch, int64_t n, int nh_i, int c_i, int m, int flags) {
  LowpWs w{};
  const int64_t E = n / m;
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  size_t off = 0;
  w.scores = off;
  off = al(off + (size_t)batch * n * E * ((flags & CSA_INDEX_BF16_SCORES) ? 2 : 4));
  if (flags & CSA_INDEX_FP8_QK) {
    w.q8 = off; off = al(off + (size_t)batch * n * nh_i * c_i);
    w.qs = off; off = al(off + (size_t)batch * n * nh_i * 4);
    w.k8 = off; off = al(off + (size_t)batch * E * c_i);
    w.ks = off; off = al(off + (size_t)batch * E * 4);
  }
  w.total = off;
  return w;
}
}  // namespace

size_t csa_index_topk_lowp_workspace(int64_t batch, int64_t n, int nh_i, int c_i, int m, int k,
                                     int flags) {
  (void)k;
  if (batch <= 0 || n <= 0 || m <= 0 || nh_i <= 0 || c_i <= 0 || flags < 1 || flags > 3) return 0;
  return lowp_ws(batch, n, nh_i, c_i, m, flags).total;
}

csa_status csa_index_topk_lowp(const void* q_i, const float* w_i, const void* k_i, int64_t batch,
                               int64_t n, int nh_i, int c_i, int m, int k, csa_dtype dt,
                               int flags, int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
  REQUIRE(valid_dt(dt), "dt must be CSA_F32 or CSA_BF16");
  REQUIRE(batch >= 0 && n >= 0, "batch and n must be >= 0");
  REQUIRE(nh_i >= 1, "nh_i must be >= 1");
  REQUIRE(c_i >= 8 && c_i % 8 == 0, "c_i must be a positive multiple of 8");
  REQUIRE(m >= 1, "m must be >= 1");
  REQUIRE(k >= 1, "k must be >= 1");
  REQUIRE(flags >= 1 && flags <= 3, "flags must combine CSA_INDEX_FP8_QK and CSA_INDEX_BF16_SCORES");
  const bool fp8 = (flags & CSA_INDEX_FP8_QK) != 0, bf16s = (flags & CSA_INDEX_BF16_SCORES) != 0;
  if (dt != CSA_BF16) return fail(CSA_ERR_UNSUPPORTED, "the low-precision indexer takes bf16 inputs");
  if (fp8 && !index_fp8_supported(nh_i, c_i))
    return fail(CSA_ERR_UNSUPPORTED, "the FP8 indexer needs c_i = 128 and nh_i in {16, 32, 64, 128}");
  const int64_t E = n / m;
  if (bf16s && E > 32768)
    return fail(CSA_ERR_UNSUPPORTED, "bf16 scores need n/m <= 32768");
  if (batch == 0 || n == 0) return ok();
  REQUIRE_PTR(idx);
  if (bf16s && !fp8 && !index_scores_tc_supported(nh_i, c_i, dt, q_i, k_i))
    return fail(CSA_ERR_UNSUPPORTED, "bf16 scores need the tensor-core indexer shape");
  if (E > 0) {
    REQUIRE_PTR(q_i);
    REQUIRE_PTR(w_i);
    REQUIRE_PTR(k_i);
    const size_t need = csa_index_topk_lowp_workspace(batch, n, nh_i, c_i, m, k, flags);
    if (ws_bytes < need || ws == nullptr)
      return fail(CSA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, need);
    REQUIRE_PTR(ws);
  }
  cudaStream_t s = (cudaStream_t)stream;
  const LowpWs L = lowp_ws(batch, n, nh_i, c_i, m, flags);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  if (E > 0) {
    unsigned int* flag = device_timeout_flag();
    if (flag == nullptr) return fail(CSA_ERR_CUDA, "csa_index_topk_lowp: no device flag");
    cudaError_t e;
    if (fp8) {
      uint8_t* q8 = wb + L.q8;
      float* qs = reinterpret_cast<float*>(wb + L.qs);
      uint8_t* k8 = wb + L.k8;
      float* ks = reinterpret_cast<float*>(wb + L.ks);
      if ((e = launch_quantize_rows_fp8(q_i, batch * n * nh_i, q8, qs, s)) != cudaSuccess ||
          (e = launch_quantize_rows_fp8(k_i, batch * E, k8, ks, s)) != cudaSuccess)
        return cuda_status(e, "csa_index_topk_lowp (quantize)");
      e = launch_index_scores_fp8(q8, qs, k8, ks, w_i, batch, n, nh_i, m, wb + L.scores, bf16s, E,
                                  flag, s);
    } else {
      e = launch_index_scores_tc(q_i, w_i, k_i, batch, n, nh_i, c_i, m, wb + L.scores, true, E,
                                 flag, s);
    }
    if (e != cudaSuccess) return cuda_status(e, "csa_index_topk_lowp (scores)");
  }
  if (bf16s)
    return cuda_status(launch_topk_rows_bf16(reinterpret_cast<const __nv_bfloat16*>(wb + L.scores),
                                             E, batch, n, m, E, k, idx, s),
                       "csa_index_topk_lowp (top-k)");
  return cuda_status(launch_topk_rows(reinterpret_cast<const float*>(wb + L.scores), E, batch, n,
                                      m, E, k, idx, s),
                     "csa_index_topk_lowp (top-k)");
}

csa_status csa_sparse_attn(const void* q, const void* kv_comp, const int32_t* idx, int k,
                           const void* kv_win, int window, const float* sink, float scale,
                           int64_t batch, int64_t n, int nh, int c, int m, csa_dtype dt,
                           void* out, void* stream) {
  REQUIRE(k >= 1, "k must be >= 1");
  csa_status st = check_attn_common(q, kv_comp, kv_win, window, scale, batch, n, nh, c, m, dt,
                                    out, sink);
  if (st != CSA_OK || batch == 0 || n == 0) return st;
  REQUIRE_PTR(idx);
  return cuda_status(launch_attn(q, kv_comp, idx, k, kv_win, window, sink, scale, batch, n, nh,
                                 c, m, dt, nullptr, out, (cudaStream_t)stream),
                     "csa_sparse_attn");
}

csa_status hca_attn(const void* q, const void* kv_comp, const void* kv_win, int window,
                    const float* sink, float scale, int64_t batch, int64_t n, int nh, int c,
                    int m_heavy, csa_dtype dt, void* out, void* stream) {
  csa_status st = check_attn_common(q, kv_comp, kv_win, window, scale, batch, n, nh, c, m_heavy,
                                    dt, out, sink);
  if (st != CSA_OK || batch == 0 || n == 0) return st;
  return cuda_status(launch_attn(q, kv_comp, nullptr, 0, kv_win, window, sink, scale, batch, n,
                                 nh, c, m_heavy, dt, nullptr, out, (cudaStream_t)stream),
                     "hca_attn");
}

csa_status csa_norm_rope_rows(const void* x, int64_t batch, int64_t n, int heads, int c,
                              int64_t pos_mul, const csa_norm_rope* nr, csa_dtype dt, void* out,
                              void* stream) {
  REQUIRE(valid_dt(dt), "dt must be CSA_F32 or CSA_BF16");
  REQUIRE(batch >= 0 && n >= 0, "batch and n must be >= 0");
  REQUIRE(heads >= 1, "heads must be >= 1");
  REQUIRE(c >= 8 && c % 8 == 0, "c must be a positive multiple of 8");
  REQUIRE(pos_mul >= 0, "pos_mul must be >= 0");
  csa_status st = check_norm_rope(nr, c);
  if (st != CSA_OK) return st;
  if (c > 1024) return fail(CSA_ERR_UNSUPPORTED, "csa_norm_rope_rows needs c <= 1024");
  if (batch == 0 || n == 0) return ok();
  REQUIRE_PTR(x);
  REQUIRE_PTR(out);
  return cuda_status(launch_norm_rope_rows(x, batch, n, heads, c, pos_mul, nr, dt, out,
                                           (cudaStream_t)stream),
                     "csa_norm_rope_rows");
}

csa_status csa_compress_norm_rope(const void* ca, const void* cb, const void* za,
                                  const void* zb, const float* ba, const float* bb,
                                  int64_t batch, int64_t n, int c, int m, int overlap,
                                  csa_dtype dt, const csa_norm_rope* nr, void* out,
                                  void* stream) {
  REQUIRE(valid_dt(dt), "dt must be CSA_F32 or CSA_BF16");
  REQUIRE(batch >= 0 && n >= 0, "batch and n must be >= 0");
  REQUIRE(c >= 8 && c % 8 == 0, "c must be a positive multiple of 8");
  REQUIRE(m >= 1, "m must be >= 1");
  REQUIRE(overlap == 0 || overlap == 1, "overlap must be 0 or 1");
  if (!overlap)
    REQUIRE(cb == nullptr && zb == nullptr && bb == nullptr,
            "cb, zb and bb must be NULL when overlap == 0");
  csa_status st = check_norm_rope(nr, c);
  if (st != CSA_OK) return st;
  if (c > 1024) return fail(CSA_ERR_UNSUPPORTED, "the entry norm needs c <= 1024");
  if (batch == 0 || n / m == 0) return ok();
  REQUIRE_PTR(ca);
  REQUIRE_PTR(za);
  REQUIRE_PTR(ba);
  REQUIRE_PTR(out);
  if (overlap) {
    REQUIRE_PTR(cb);
    REQUIRE_PTR(zb);
    REQUIRE_PTR(bb);
  }
  return cuda_status(launch_compress(ca, cb, za, zb, ba, bb, batch, n, c, m, overlap, dt, nr,
                                     out, (cudaStream_t)stream),
                     "csa_compress_norm_rope");
}

csa_status csa_sparse_attn_norm_rope(const void* q, const void* kv_comp, const int32_t* idx,
                                     int k, const void* kv_win, int window, const float* sink,
                                     float scale, int64_t batch, int64_t n, int nh, int c, int m,
                                     csa_dtype dt, const csa_norm_rope* nr, void* out,
                                     void* stream) {
  REQUIRE(k >= 1, "k must be >= 1");
  csa_status st = check_attn_common(q, kv_comp, kv_win, window, scale, batch, n, nh, c, m, dt,
                                    out, sink);
  if (st != CSA_OK) return st;
  if ((st = check_norm_rope(nr, c)) != CSA_OK) return st;
  if (batch == 0 || n == 0) return ok();
  REQUIRE_PTR(idx);
  return cuda_status(launch_attn(q, kv_comp, idx, k, kv_win, window, sink, scale, batch, n, nh,
                                 c, m, dt, nr, out, (cudaStream_t)stream),
                     "csa_sparse_attn_norm_rope");
}

csa_status hca_attn_norm_rope(const void* q, const void* kv_comp, const void* kv_win, int window,
                              const float* sink, float scale, int64_t batch, int64_t n, int nh,
                              int c, int m_heavy, csa_dtype dt, const csa_norm_rope* nr,
                              void* out, void* stream) {
  csa_status st = check_attn_common(q, kv_comp, kv_win, window, scale, batch, n, nh, c, m_heavy,
                                    dt, out, sink);
  if (st != CSA_OK) return st;
  if ((st = check_norm_rope(nr, c)) != CSA_OK) return st;
  if (batch == 0 || n == 0) return ok();
  return cuda_status(launch_attn(q, kv_comp, nullptr, 0, kv_win, window, sink, scale, batch, n,
                                 nh, c, m_heavy, dt, nr, out, (cudaStream_t)stream),
                     "hca_attn_norm_rope");
}

size_t csa_grouped_out_proj_workspace(int64_t rows, int groups, int d_g) {
  if (rows <= 0 || groups <= 0 || d_g <= 0) return 0;
  return (size_t)rows * groups * d_g * 2;
}

csa_status csa_grouped_out_proj(const void* o, int64_t rows, int nh, int c, int groups, int d_g,
                                int d, const void* w1, const void* w2, void* ws,
                                size_t ws_bytes, void* y, void* stream) {
  REQUIRE(rows >= 0, "rows must be >= 0");
  REQUIRE(nh >= 1 && c >= 1 && groups >= 1 && d_g >= 1 && d >= 1,
          "nh, c, groups, d_g and d must be >= 1");
  REQUIRE(nh % groups == 0, "nh must be a multiple of groups");
  if ((int64_t)(nh / groups) * c % 64 != 0 || d_g % 256 != 0 || d % 256 != 0)
    return fail(CSA_ERR_UNSUPPORTED,
                "grouped projection needs (nh/groups)*c %% 64 == 0, d_g %% 256 == 0, d %% 256 == 0");
  if (rows == 0) return ok();
  REQUIRE_PTR(o);
  REQUIRE_PTR(w1);
  REQUIRE_PTR(w2);
  REQUIRE_PTR(y);
  const size_t need = csa_grouped_out_proj_workspace(rows, groups, d_g);
  if (ws == nullptr || ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, need);
  REQUIRE_PTR(ws);
  return cuda_status(launch_grouped_out_proj(o, rows, nh, c, groups, d_g, d, w1, w2, ws, y,
                                             (cudaStream_t)stream),
                     "csa_grouped_out_proj");
}

}  // extern "C"

namespace {

csa_status check_paging(const csa_cache_desc* d, const csa_paging* pg) {
  if (pg == nullptr) return ok();
  REQUIRE(pg->block_tokens >= d->m && pg->block_tokens % d->m == 0,
          "block_tokens must be a positive multiple of m");
  const int epb = pg->block_tokens / d->m;
  REQUIRE((epb & (epb - 1)) == 0, "block_tokens / m must be a power of two");
  REQUIRE(pg->num_blocks >= 1 && pg->max_blocks >= 1, "num_blocks and max_blocks must be >= 1");
  REQUIRE(d->capacity == pg->max_blocks * epb, "capacity must equal max_blocks * block_tokens / m");
  REQUIRE(pg->num_blocks * (int64_t)epb < ((int64_t)1 << 31), "the pool must hold < 2^31 entries");
  REQUIRE_PTR(pg->block_table);
  if (!d->is_hca && epb < 32)
    return fail(CSA_ERR_UNSUPPORTED, "a paged CSA layer needs at least 32 entries per block");
  return ok();
}

csa_status cache_layout_impl(const csa_cache_desc* desc, const csa_paging* pg,
                             csa_cache_layout_t* layout) {
  csa_status st = check_desc(desc);
  if (st != CSA_OK) return st;
  if ((st = check_paging(desc, pg)) != CSA_OK) return st;
  REQUIRE(layout != nullptr, "layout is NULL");
  cache_layout(*desc, layout, pg);
  return ok();
}

csa_status store_entries_impl(const csa_cache_desc* desc, const csa_paging* pg, void* cache,
                              int64_t first, int64_t count, const void* kv, const void* ikey,
                              csa_dtype dt, void* stream) {
  csa_status st = check_desc(desc);
  if (st != CSA_OK) return st;
  if ((st = check_paging(desc, pg)) != CSA_OK) return st;
  REQUIRE(valid_dt(dt), "dt must be CSA_F32 or CSA_BF16");
  REQUIRE(first >= 0 && count >= 0 && first + count <= desc->capacity,
          "entries [first, first+count) must lie within [0, capacity)");
  if (count == 0) return ok();
  REQUIRE_PTR(cache);
  REQUIRE_PTR(kv);
  if (!desc->is_hca) REQUIRE_PTR(ikey);
  return cuda_status(launch_store_entries(*desc, cache_view(*desc, cache, pg), first, count, kv,
                                          ikey, dt, (cudaStream_t)stream),
                     "csa_cache_store_entries");
}

static csa_status check_rows(const csa_cache_desc* d, const csa_rows* rows) {
  REQUIRE(rows != nullptr, "rows is NULL");
  REQUIRE_PTR(rows->ca);
  REQUIRE_PTR(rows->za);
  REQUIRE_PTR(rows->kv_win);
  if (!d->is_hca) {
    REQUIRE_PTR(rows->cb);
    REQUIRE_PTR(rows->zb);
    REQUIRE_PTR(rows->ica);
    REQUIRE_PTR(rows->icb);
    REQUIRE_PTR(rows->iza);
    REQUIRE_PTR(rows->izb);
  }
  return ok();
}

csa_status write_rows_impl(const csa_cache_desc* desc, const csa_paging* pg, void* cache,
                           int64_t first_pos, int64_t count, const csa_rows* rows, void* stream) {
  csa_status st = check_desc(desc);
  if (st != CSA_OK) return st;
  if ((st = check_paging(desc, pg)) != CSA_OK) return st;
  REQUIRE(first_pos >= 0 && count >= 0, "first_pos and count must be >= 0");
  if (count == 0) return ok();
  REQUIRE_PTR(cache);
  if ((st = check_rows(desc, rows)) != CSA_OK) return st;
  return cuda_status(launch_write_rows(*desc, cache_view(*desc, cache, pg), first_pos, count,
                                       *rows, (cudaStream_t)stream),
                     "csa_cache_write_rows");
}

csa_status decode_step_impl(const csa_cache_desc* desc, const csa_paging* pg, void* cache,
                            const int64_t* pos, const csa_rows* rows,
                            const csa_decode_params* params, const void* q, const void* q_i,
                            const float* w_i, void* out, void* ws, size_t ws_bytes,
                            void* stream) {
  csa_status st = check_desc(desc);
  if (st != CSA_OK) return st;
  if ((st = check_paging(desc, pg)) != CSA_OK) return st;
  REQUIRE_PTR(cache);
  REQUIRE_PTR(pos);
  if ((st = check_rows(desc, rows)) != CSA_OK) return st;
  REQUIRE(params != nullptr, "params is NULL");
  REQUIRE_PTR(params->ba);
  REQUIRE_OPT_PTR(params->sink);
  REQUIRE(params->scale == params->scale, "scale must not be NaN");
  REQUIRE_PTR(q);
  REQUIRE_PTR(out);
  if (!desc->is_hca) {
    REQUIRE_PTR(params->bb);
    REQUIRE_PTR(params->iba);
    REQUIRE_PTR(params->ibb);
    REQUIRE_PTR(q_i);
    REQUIRE_PTR(w_i);
  }
  REQUIRE_OPT_PTR(params->sel_out);
  REQUIRE_OPT_PTR(params->scores_out);
  if (!desc->is_hca && params->scores_out != nullptr && !decode_index_tc_supported(*desc))
    return fail(CSA_ERR_UNSUPPORTED,
                "scores_out needs the tensor-core indexer shape (c_i = 128, nh_i 64 or 128)");
  const size_t need = decode_workspace(*desc);
  if (ws == nullptr || ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, need);
  REQUIRE_PTR(ws);
  return cuda_status(launch_decode_step(*desc, cache_view(*desc, cache, pg), pos, *rows, *params,
                                        q, q_i, w_i, out, ws, (cudaStream_t)stream),
                     "csa_decode_step");
}

}  // namespace

extern "C" {

csa_status csa_cache_layout(const csa_cache_desc* desc, csa_cache_layout_t* layout) {
  return cache_layout_impl(desc, nullptr, layout);
}
csa_status csa_paged_cache_layout(const csa_cache_desc* desc, const csa_paging* paging,
                                  csa_cache_layout_t* layout) {
  REQUIRE(paging != nullptr, "paging is NULL");
  return cache_layout_impl(desc, paging, layout);
}

csa_status csa_cache_store_entries(const csa_cache_desc* desc, void* cache, int64_t first,
                                   int64_t count, const void* kv, const void* ikey,
                                   csa_dtype dt, void* stream) {
  return store_entries_impl(desc, nullptr, cache, first, count, kv, ikey, dt, stream);
}
csa_status csa_paged_cache_store_entries(const csa_cache_desc* desc, const csa_paging* paging,
                                         void* cache, int64_t first, int64_t count,
                                         const void* kv, const void* ikey, csa_dtype dt,
                                         void* stream) {
  REQUIRE(paging != nullptr, "paging is NULL");
  return store_entries_impl(desc, paging, cache, first, count, kv, ikey, dt, stream);
}

csa_status csa_cache_write_rows(const csa_cache_desc* desc, void* cache, int64_t first_pos,
                                int64_t count, const csa_rows* rows, void* stream) {
  return write_rows_impl(desc, nullptr, cache, first_pos, count, rows, stream);
}
csa_status csa_paged_cache_write_rows(const csa_cache_desc* desc, const csa_paging* paging,
                                      void* cache, int64_t first_pos, int64_t count,
                                      const csa_rows* rows, void* stream) {
  REQUIRE(paging != nullptr, "paging is NULL");
  return write_rows_impl(desc, paging, cache, first_pos, count, rows, stream);
}

size_t csa_decode_workspace(const csa_cache_desc* desc) {
  if (check_desc(desc) != CSA_OK) return 0;
  return decode_workspace(*desc);
}

csa_status csa_decode_step(const csa_cache_desc* desc, void* cache, const int64_t* pos,
                           const csa_rows* rows, const csa_decode_params* params,
                           const void* q, const void* q_i, const float* w_i, void* out,
                           void* ws, size_t ws_bytes, void* stream) {
  return decode_step_impl(desc, nullptr, cache, pos, rows, params, q, q_i, w_i, out, ws,
                          ws_bytes, stream);
}
csa_status csa_paged_decode_step(const csa_cache_desc* desc, const csa_paging* paging,
                                 void* cache, const int64_t* pos, const csa_rows* rows,
                                 const csa_decode_params* params, const void* q,
                                 const void* q_i, const float* w_i, void* out, void* ws,
                                 size_t ws_bytes, void* stream) {
  REQUIRE(paging != nullptr, "paging is NULL");
  return decode_step_impl(desc, paging, cache, pos, rows, params, q, q_i, w_i, out, ws, ws_bytes,
                          stream);
}

}  // extern "C"
