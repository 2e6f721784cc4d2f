// Host-side launch functions, one per kernel family.  Arguments are already
// validated by the C ABI layer (csa_api.cu); these only size grids and launch.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>
#include <utility>

#include "../../include/csa.h"

namespace csa {

// Launches `kern` with programmatic stream serialization: its CTAs may be
// scheduled while the previous kernel on `s` drains; the kernel itself
// waits (griddepcontrol.wait) before touching anything that kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Number of SMs of the current device (cached per device).
int sm_count();

// Records a one-line reason for `st` (read back by csa_last_error) and returns st.
csa_status set_last_error(csa_status st, const char* fmt, ...);

// Device word that kernels with bounded waits OR a bit into when a wait
// expires (per current device; csa_check reads and clears it).
unsigned int* device_timeout_flag();

// tcgen05 indexer (bf16, c_i in {64, 128}, nh_i in {16, 32, 64, 128}).
bool index_scores_tc_supported(int nh_i, int c_i, csa_dtype dt, const void* q_i, const void* k_i);
// scores: fp32, or bf16 when bf16_scores.
cudaError_t launch_index_scores_tc(const void* q_i, const float* w_i, const void* k_i,
                                   int64_t batch, int64_t n, int nh_i, int c_i, int m,
                                   void* scores, bool bf16_scores, int64_t ld, unsigned int* err,
                                   cudaStream_t s);

// Low-precision indexer: E4M3 codes + fp32 scale of rows of 128 bf16 values,
// and the FP8 x FP8 tcgen05 scores (c_i = 128, nh_i in {16, 32, 64, 128}).
bool index_fp8_supported(int nh_i, int c_i);
cudaError_t launch_quantize_rows_fp8(const void* x, int64_t rows, uint8_t* codes, float* scales,
                                     cudaStream_t s);
cudaError_t launch_index_scores_fp8(const uint8_t* q8, const float* qs, const uint8_t* k8,
                                    const float* ks, const float* w_i, int64_t batch, int64_t n,
                                    int nh_i, int m, void* scores, bool bf16_scores, int64_t ld,
                                    unsigned int* err, cudaStream_t s);
// Top-k rows over bf16 scores (rows of at most 32768 keys).
cudaError_t launch_topk_rows_bf16(const __nv_bfloat16* scores, int64_t ld, int64_t batch,
                                  int64_t n, int m, int64_t E, int k, int32_t* idx,
                                  cudaStream_t s);

// tcgen05 attention (bf16, 64 heads of dim 512, up to 2048 selected entries).
bool attn_tc_supported(int nh, int c, int k, csa_dtype dt, const void* q, const void* kv_comp,
                       const void* kv_win, int rope_dims);
// One warp waits on a barrier that is completed first (arrive) or never; the
// wait gives up after limit_us and sets *err.
cudaError_t launch_selftest_wait(uint32_t limit_us, bool arrive, unsigned int* err,
                                 cudaStream_t s);
// Query RMSNorm + rotation and output rotation of the attention kernels
// (gamma == NULL: off).
struct QNormRope {
  const float* gamma;
  float eps;
  int rope_dims;
  float base;
};
cudaError_t launch_attn_tc(const void* q, const void* kv_comp, const int32_t* idx, int k,
                           const void* kv_win, int window, const float* sink, float scale,
                           int64_t batch, int64_t n, int m, const QNormRope& qn, void* out,
                           unsigned int* err, cudaStream_t s);

// tcgen05 decode indexer over FP8 keys (c_i = 128, nh_i in {64, 128}), persistent.
struct CacheView;
bool decode_index_tc_supported(const csa_cache_desc& d);
// Bytes of one sequence's indexer query operand: the swizzled hi / lo E4M3
// image (2 H rows of 128 bytes) followed by H fp32 weights.
__host__ __device__ inline size_t decode_qop_bytes(int nh_i) { return (size_t)nh_i * (2 * 128 + 4); }
// Row of head h's hi (part 0) or lo (part 1) FP8 half in the query operand.
// With 64 heads the operand is the M side of the indexer MMA and its rows
// are ordered for the 16-lane TMEM loads of the epilogue: in each block of 16
// rows, rows 0-7 hold the hi halves and rows 8-15 the lo halves of 8 heads
// (row 16 (h / 8) + 8 part + h % 8).  Otherwise the H hi rows come first,
// then the H lo rows.
__host__ __device__ inline int decode_qop_row(int h, int part, int H) {
  return H == 64 ? ((h >> 3) << 4) + (part << 3) + (h & 7) : part * H + h;
}
// qop: [batch] query operands (written by the append step); scores
// [batch][capacity] fp32, written for s < V of each sequence.
// ghist [batch][kDecHistBins]: each sequence's score histogram (added to).
// idx_done [batch] (optional): each CTA adds, once its scores and histogram
// counts of a sequence are written (fenced), the number of the sequence's
// key tiles it scored, so a later kernel can start on a sequence as soon as
// the count reaches decode_index_tiles(d, pos) without waiting for the grid.
cudaError_t launch_decode_index_tc(const csa_cache_desc& d, const CacheView& cv,
                                   const int64_t* pos, const uint8_t* qop, float* scores,
                                   uint32_t* ghist, uint32_t* idx_done, unsigned int* err,
                                   cudaStream_t s);
// Keys per indexer tile of launch_decode_index_tc for this cache.
int decode_index_tile_keys(const csa_cache_desc& d);

// Histogram of each sequence's indexer scores over the top kDecHistShift..31
// bits of their order keys, written by the indexer for the selection step.
constexpr int kDecHistBins = 4096;
constexpr int kDecHistShift = 20;
constexpr int kDecMaxSlices = 512;  // 4096-score slices per sequence (2M entries)

// Selection scratch inside the decode workspace (see decode_select_ws).
struct DecodeSelectWs {
  uint32_t* ghist;     // [batch][kDecHistBins]  zeroed by the append step
  uint32_t* done;      // [batch]                finished slices; zeroed by the append step
  uint32_t* idx_done;  // [batch]                key tiles the indexer has scored and counted
                       //                        in ghist (released); zeroed by the append step
  uint32_t* list_ready;  // [batch]              the attention's selection is published;
                         //                      zeroed by the append step
  uint32_t* bitmap;    // [batch][words]         chosen entries, one bit each
  uint32_t* cand_key;  // [batch][capacity]      threshold-bin candidates, per slice
  int32_t* cand_idx;
  uint32_t* cand_cnt;  // [batch][kDecMaxSlices]
  uint32_t* cc_key;    // [batch][capacity]      the candidates gathered in index order
  int32_t* cc_idx;
  int64_t words;
};
// Layout of the scratch at `base` (NULL: only the size); *bytes its size.
DecodeSelectWs decode_select_ws(const csa_cache_desc& d, uint8_t* base, size_t* bytes);
// Exact top-k from the indexer's scores and histogram: many CTAs per
// sequence, the last of them writing sel [batch][k] (ascending, -1 padded
// when V <= k).
bool decode_select_supported(const csa_cache_desc& d);
cudaError_t launch_decode_select(const csa_cache_desc& d, const int64_t* pos, const float* scores,
                                 const DecodeSelectWs& ws, int32_t* sel, cudaStream_t s);

// tcgen05 decode attention (64 heads x 512, FP8/bf16 cache): one 128-entry
// tile per CTA (ntile = decode_attn_splits), merged by a combine kernel.
bool decode_attn_tc_supported(const csa_cache_desc& d);
int decode_attn_splits(const csa_cache_desc& d);
// With scores != NULL (CSA, decode_attn_selects(d)) the kernel takes the
// top-k itself from the indexer's scores and histogram (sel unused) and, if
// sel_out != NULL, writes the selection there; with idx_done != NULL it
// starts on a sequence once the indexer's tile count for it is complete
// (tiles of idx_tile keys) instead of waiting for the indexer's whole grid.
// With several CTAs per sequence only split 0 selects: it publishes the
// selection in xlist [batch][k] and sets list_ready[b] (zeroed by the append
// step); the others process their window-only tiles meanwhile.
bool decode_attn_selects(const csa_cache_desc& d);
cudaError_t launch_decode_attn_tc(const csa_cache_desc& d, const CacheView& cv,
                                  const int64_t* pos, const void* q, const int32_t* sel,
                                  const float* sink, float scale, int nsplit, void* out,
                                  float* part_o, float* part_ms, const float* scores,
                                  const uint32_t* ghist, int32_t* sel_out,
                                  const uint32_t* idx_done, int idx_tile, int32_t* xlist,
                                  uint32_t* list_ready, unsigned int* err, cudaStream_t s);

// nr != NULL: each entry i RMSNorm-ed and its trailing dims rotated for
// position m * i as it is written (or by a second in-place pass).
cudaError_t launch_compress(const void* ca, const void* cb, const void* za, const void* zb,
                            const float* ba, const float* bb, int64_t batch, int64_t n, int c,
                            int m, int overlap, csa_dtype dt, const csa_norm_rope* nr, void* out,
                            cudaStream_t s);
// Rows [batch, n, heads, c]: RMSNorm + rotation of the trailing dims for
// position t * pos_mul (t the row's token); out may equal x.
cudaError_t launch_norm_rope_rows(const void* x, int64_t batch, int64_t n, int heads, int c,
                                  int64_t pos_mul, const csa_norm_rope* nr, csa_dtype dt,
                                  void* out, cudaStream_t s);

// fp32 scores[b][t][s] (row stride `ld`) for s < V(t); entries beyond V(t) untouched.
cudaError_t launch_index_scores(const void* q_i, const float* w_i, const void* k_i,
                                int64_t batch, int64_t n, int nh_i, int c_i, int m,
                                csa_dtype dt, float* scores, int64_t ld, cudaStream_t s);

// Top-k rows: row r of `rows` has V(r) candidates; writes idx[r][0..k).
cudaError_t launch_topk_rows(const float* scores, int64_t ld, int64_t batch, int64_t n,
                             int m, int64_t E, int k, int32_t* idx, cudaStream_t s);

// q_nr != NULL: each query head RMSNorm-ed and rotated for position t before
// the logits, and the output's trailing dims rotated by -t (the entries are
// taken as given: already normed and rotated).
cudaError_t launch_attn(const void* q, const void* kv_comp, const int32_t* idx, int k,
                        const void* kv_win, int window, const float* sink, float scale,
                        int64_t batch, int64_t n, int nh, int c, int m, csa_dtype dt,
                        const csa_norm_rope* q_nr, void* out, cudaStream_t s);

// Grouped output projection: z = grouped o W1^T (bf16 [rows, G dg]), y = z W2^T.
cudaError_t launch_grouped_out_proj(const void* o, int64_t rows, int nh, int c, int G, int dg,
                                    int d, const void* w1, const void* w2, void* z, void* y,
                                    cudaStream_t s);

// ---- decode --------------------------------------------------------------
struct CacheView {
  uint8_t* entry_fp8;
  float* entry_scale;
  __nv_bfloat16* entry_rope;
  uint8_t* ikey_fp8;
  float* ikey_scale;
  __nv_bfloat16* window;
  __nv_bfloat16* state;
  __nv_bfloat16* istate;
  // paged classical cache: entry s of sequence b sits in physical block
  // btab[b][s >> epb_shift] of the pool, row s & (epb - 1); NULL btab: the
  // contiguous [batch][capacity] form
  const int32_t* btab;
  int64_t bt_stride;   // block-table row length
  int64_t nblocks;     // blocks in the pool
  int epb_shift;       // log2(entries per block)
};

// Row of entry s of sequence b in the entry regions, or -1 when its block is
// absent from the pool (such entries read as zero and are not written).
__host__ __device__ __forceinline__ int64_t entry_row(const CacheView& cv, int64_t b, int64_t s,
                                                      int64_t cap) {
  if (cv.btab == nullptr) return b * cap + s;
  const int64_t blk = cv.btab[b * cv.bt_stride + (s >> cv.epb_shift)];
  if (blk < 0 || blk >= cv.nblocks) return -1;
  return (blk << cv.epb_shift) + (s & ((int64_t(1) << cv.epb_shift) - 1));
}

// Paging of the classical cache (NULL: contiguous).
CacheView cache_view(const csa_cache_desc& d, void* cache, const csa_paging* pg = nullptr);
void cache_layout(const csa_cache_desc& d, csa_cache_layout_t* L, const csa_paging* pg = nullptr);

cudaError_t launch_store_entries(const csa_cache_desc& d, const CacheView& cv, int64_t first,
                                 int64_t count, const void* kv, const void* ikey, csa_dtype dt,
                                 cudaStream_t s);
cudaError_t launch_write_rows(const csa_cache_desc& d, const CacheView& cv, int64_t first_pos,
                              int64_t count, const csa_rows& rows, cudaStream_t s);
size_t decode_workspace(const csa_cache_desc& d);
cudaError_t launch_decode_step(const csa_cache_desc& d, const CacheView& cv, const int64_t* pos,
                               const csa_rows& rows, const csa_decode_params& p, const void* q,
                               const void* q_i, const float* w_i, void* out, void* ws,
                               cudaStream_t s);

}  // namespace csa
