/*
 * csa.h -- C ABI of the CSA / HCA attention layer for one NVIDIA B200 (sm_100a).
 *
 * The layer (DeepSeek-V4 hybrid attention) has four parts:
 *   1. a token-level KV compressor (overlapped for CSA, single-stream for HCA),
 *   2. a lightning indexer that scores visible compressed entries, plus top-k,
 *   3. shared-KV multi-query attention over the selected entries and a causal
 *      sliding window of raw rows,
 *   4. a per-head attention sink inside the same softmax denominator.
 *
 * Sources, cited by page title and section:
 *   [Formulas B9]  "Core formulas chapter" (polysight, 06-formulas), B9 CSA + HCA.
 *   [Walk-through] "DeepSeek-V4: million-token context" (songhuiming.github.io),
 *                  sections 4.1-4.5 (CSA) and 5.1-5.2 (HCA).
 *   [Analysis]     "DeepSeek paper-feature analysis" (deepseek-paper-analysis.md),
 *                  sections 7.1-7.3 and "Inference KV Cache".
 *   [Notes]        "DeepSeek-V4 reader's notes" (cooking-agi, deepseek-v4.html),
 *                  section 2 (ledger) and section 3 (completion rule).
 *
 * Conventions shared by every entry point
 *   - Memory: the caller owns every buffer (inputs, outputs, cache, workspace),
 *     all of them device memory unless stated.  The library never allocates,
 *     frees or synchronises; all work is enqueued on `stream` (a cudaStream_t
 *     passed as void*, NULL = legacy default stream).
 *   - Layout: dense row-major, innermost dimension last, no padding.  Tensor
 *     pointers must be 16-byte aligned.
 *   - Numbers: CSA_F32 / CSA_BF16 select the element type of the activation
 *     tensors; all arithmetic is fp32.  Biases, head weights and sinks are fp32.
 *   - Positions are 0-based.  A query at position t may read the compressed
 *     entries s < floor((t+1)/m) ([Notes] section 3: (pos+1)//m entries are
 *     complete) and the raw window rows max(0, t-W+1) .. t.
 *   - Errors: arguments are checked before anything is launched; a bad
 *     argument returns CSA_ERR_INVALID_ARG and launches nothing.  A failed
 *     launch returns CSA_ERR_CUDA.  csa_last_error() gives a one-line reason
 *     (thread-local, valid until the next call on the same thread).
 *   - Empty work (batch == 0 or n == 0) returns CSA_OK without a launch.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = -1, /* bad size, null or misaligned pointer, bad enum   */
  CSA_ERR_UNSUPPORTED = -2, /* valid but not built for (e.g. a dim too large)    */
  CSA_ERR_WORKSPACE = -3,   /* workspace smaller than the *_workspace() figure    */
  CSA_ERR_CUDA = -4,        /* a CUDA launch or API call failed                   */
  CSA_ERR_TIMEOUT = -5      /* a bounded device-side wait gave up                 */
} csa_status;

typedef enum { CSA_F32 = 0, CSA_BF16 = 1 } csa_dtype;

/* Human-readable name of a status code (static string). */
const char* csa_status_string(int status);
/* Reason for the last non-OK status returned on this thread ("" if none). */
const char* csa_last_error(void);
/* ABI version, bumped on any signature or layout change (2: csa_decode_params
 * gained scores_out; the norm / RoPE calls were added). */
int csa_abi_version(void);
/* Synchronises `stream`, then returns CSA_ERR_TIMEOUT if any kernel of this
 * library on the current device gave up a bounded wait since the last check,
 * and clears that record.  While the record is set, every later kernel of the
 * library on that device skips or cuts short its work, so the outputs of ALL
 * launches on the device since the last check are invalid, not only those of
 * the launch that gave up.  The one entry point that synchronises. */
csa_status csa_check(void* stream);
/* Exercises the bounded-wait path on the device (no counterpart on the
 * pages; a library self-test).  One warp waits on a shared-memory barrier;
 * if `arrive` is non-zero the barrier is completed first and the wait
 * succeeds, otherwise nothing completes it and the wait gives up after
 * `limit_us` microseconds (1 .. 2,000,000), recording the timeout exactly as
 * a kernel of the layer would: the next csa_check on that device returns
 * CSA_ERR_TIMEOUT.  No fault, trap or hang is involved; the context stays
 * usable.  Returns CSA_ERR_INVALID_ARG for a limit out of range. */
csa_status csa_selftest_wait(uint32_t limit_us, int arrive, void* stream);

/* ------------------------------------------------------------------------
 * csa_compress -- token-level KV compressor ([Formulas B9] CSA and HCA
 * compressor equations; [Walk-through] 4.1 overlapped compression and 5.1
 * non-overlapped compression; [Analysis] 7.1, 7.2).
 *
 * overlap = 1 (CSA): entry i, dimension d, joins 2m logits
 *     Za[m*i+j, d] + Ba[j, d]        (own block, j = 0..m-1)
 *     Zb[m*(i-1)+j, d] + Bb[j, d]    (previous block)
 *   in one softmax S, and out[i, d] = sum_j Sa_j Ca[m*i+j, d]
 *   + sum_j Sb_j Cb[m*(i-1)+j, d].  For i = 0 the previous-block logits are
 *   -inf and its rows zero.
 * overlap = 0 (HCA): out[i, d] = sum_j softmax_j(Z[m*i+j, d] + B[j, d]) C[m*i+j, d];
 *   pass C as `ca`, Z as `za`, B as `ba`; `cb`, `zb`, `bb` must be NULL.
 *
 *   ca, cb, za, zb : [batch, n, c] of `dt`
 *   ba, bb         : [m, c] fp32
 *   out            : [batch, n/m, c] of `dt` (n/m rounded down; rows past the
 *                    last full block are the not-yet-compressed tail)
 * Constraints: c % 8 == 0, m >= 1.  Also used for the indexer keys (c = c_i).
 * ------------------------------------------------------------------------ */
csa_status csa_compress(const void* ca, const void* cb, const void* za, const void* zb,
                        const float* ba, const float* bb, int64_t batch, int64_t n, int c,
                        int m, int overlap, csa_dtype dt, void* out, void* stream);

/* ------------------------------------------------------------------------
 * csa_index_topk -- lightning indexer + top-k ([Formulas B9] I_{t,s};
 * [Walk-through] 4.2 steps 3-4; [Analysis] 7.1 "Lightning Indexer").
 *
 *   I[t, s] = sum_h w_i[t, h] * ReLU(q_i[t, h, :] . k_i[s, :]),  s < V(t),
 *   V(t) = min(floor((t+1)/m), n/m).
 *   idx[t, :] = the min(k, V(t)) entries with the largest I[t, s] (ties: the
 *   smaller s), listed in ascending order, then -1 padding up to k.
 *
 *   q_i : [batch, n, nh_i, c_i] of `dt`     w_i : [batch, n, nh_i] fp32
 *   k_i : [batch, n/m, c_i] of `dt` (compressed index keys)
 *   idx : [batch, n, k] int32
 *   ws  : device workspace of at least csa_index_topk_workspace(...) bytes
 *         (holds fp32 scores; contents undefined on return).
 * Constraints: c_i % 8 == 0, nh_i >= 1, k >= 1.
 * ------------------------------------------------------------------------ */
size_t csa_index_topk_workspace(int64_t batch, int64_t n, int nh_i, int c_i, int m, int k);
csa_status csa_index_topk(const void* q_i, const float* w_i, const void* k_i, int64_t batch,
                          int64_t n, int nh_i, int c_i, int m, int k, csa_dtype dt,
                          int32_t* idx, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * csa_index_topk_noalloc -- csa_index_topk for callers that cannot allocate
 * device memory (no counterpart on the pages; a library convenience).
 *
 * Same arguments, results and errors as csa_index_topk, without `ws`: the
 * score scratch is a fixed array inside the library (8 MiB per device, held
 * by every GPU that loads the library until the process exits).  Arguments
 * are checked first (CSA_ERR_INVALID_ARG as for csa_index_topk); a valid
 * call that needs more than 2^21 fp32 scores (batch * n * floor(n/m),
 * computed without overflow) returns CSA_ERR_UNSUPPORTED and launches
 * nothing.  All calls share that array, so calls whose work overlaps on the
 * GPU race on it.  The first call on a device looks up the array's address
 * (cudaGetSymbolAddress with that device current); with the CUDA runtime's
 * lazy module loading that lookup may load the library's device code and
 * the array itself (a device allocation made by the runtime, which may
 * synchronise), so make the first call before any stream capture.  Calls
 * after cudaDeviceReset of that device are unsupported (the cached address
 * is stale).  The entry point itself calls no allocator.
 * ------------------------------------------------------------------------ */
csa_status csa_index_topk_noalloc(const void* q_i, const float* w_i, const void* k_i,
                                  int64_t batch, int64_t n, int nh_i, int c_i, int m, int k,
                                  csa_dtype dt, int32_t* idx, void* stream);

/* ------------------------------------------------------------------------
 * csa_index_topk_lowp -- the lightning indexer + top-k in low precision
 * ([Analysis] "Lightning Indexer": a few heads and FP8 keep the indexer
 * cheap, the ReLU suits FP8; [Analysis] "FP4 Quantization-Aware Training":
 * index scores kept in BF16 instead of FP32).  `flags`:
 *   CSA_INDEX_FP8_QK     every query head q_i[t, h, :] and every key
 *                        k_i[s, :] is quantised to E4M3 with one fp32 scale
 *                        (amax / 448; 1 when amax = 0; code = E4M3(x / scale),
 *                        round to nearest even, saturating) and scored on the
 *                        FP8 tensor cores: I[t, s] is the indexer formula on
 *                        the dequantised vectors (fp32 accumulation);
 *   CSA_INDEX_BF16_SCORES the scores are stored as bf16 (rounded to nearest
 *                        even) and the top-k is taken over those values
 *                        (ties: the smaller s).
 * Either or both.  The selection then approximates csa_index_topk's; its
 * recall against it is what the two forms trade for speed and traffic.
 * Arguments as csa_index_topk; dt must be CSA_BF16, the FP8 form needs
 * c_i = 128 and nh_i in {16, 32, 64, 128}, the bf16-score form n/m <= 32768
 * (and c_i in {64, 128} with those nh_i when not FP8), else
 * CSA_ERR_UNSUPPORTED.  ws: csa_index_topk_lowp_workspace(...) bytes.
 * ------------------------------------------------------------------------ */
enum { CSA_INDEX_FP8_QK = 1, CSA_INDEX_BF16_SCORES = 2 };
size_t csa_index_topk_lowp_workspace(int64_t batch, int64_t n, int nh_i, int c_i, int m, int k,
                                     int flags);
csa_status csa_index_topk_lowp(const void* q_i, const float* w_i, const void* k_i, int64_t batch,
                               int64_t n, int nh_i, int c_i, int m, int k, csa_dtype dt,
                               int flags, int32_t* idx, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * csa_sparse_attn -- CSA core attention: shared-KV MQA over the selected
 * compressed entries plus the sliding window, with the sink in the same
 * denominator ([Walk-through] 4.3 shared-KV MQA, 4.5 sliding window and
 * attention sink; [Formulas B9]; [Notes] section 1).
 *
 *   E_t = { kv_comp[s] : s in idx[t, :], 0 <= s < V(t) }
 *         U { kv_win[u] : max(0, t-W+1) <= u <= t }
 *   l_hj = scale * q[t, h, :] . e_j
 *   out[t, h, :] = sum_j exp(l_hj) e_j / (exp(sink[h]) + sum_j exp(l_hj))
 *   Entries of idx outside [0, V(t)) (e.g. -1 padding) are skipped.
 *   sink == NULL means no sink term (plain softmax).
 *
 *   q : [batch, n, nh, c]   kv_comp : [batch, n/m, c]   idx : [batch, n, k] int32
 *   kv_win : [batch, n, c]  sink : [nh] fp32            out : [batch, n, nh, c]
 * Constraints: c % 8 == 0, window >= 1, k >= 1, nh >= 1.
 * ------------------------------------------------------------------------ */
csa_status csa_sparse_attn(const void* q, const void* kv_comp, const int32_t* idx, int k,
                           const void* kv_win, int window, const float* sink, float scale,
                           int64_t batch, int64_t n, int nh, int c, int m, csa_dtype dt,
                           void* out, void* stream);

/* ------------------------------------------------------------------------
 * hca_attn -- HCA core attention: dense shared-KV MQA over every visible
 * compressed entry (m = m_heavy) plus the window, sink in the denominator
 * ([Formulas B9] HCA; [Walk-through] 5.2).  Same tensors as csa_sparse_attn
 * without idx; kv_comp is [batch, n/m_heavy, c].
 * ------------------------------------------------------------------------ */
csa_status hca_attn(const void* q, const void* kv_comp, const void* kv_win, int window,
                    const float* sink, float scale, int64_t batch, int64_t n, int nh, int c,
                    int m_heavy, csa_dtype dt, void* out, void* stream);

/* ------------------------------------------------------------------------
 * RMSNorm and partial RoPE around core attention ([Walk-through] 4.5 "other
 * details": query / KV entry normalisation and partial RoPE; 7.1 Partial
 * RoPE; 7.4 Query/KV Entry Normalization).  Every query head and every KV
 * entry is RMSNorm-ed before core attention; the trailing `rope_dims` dims of
 * queries and entries are rotated for their position; since each entry is
 * both key and value, the attention output's trailing dims are rotated back
 * by position -t, so the output depends on relative positions only.
 *
 *   RMSNorm(x) = x / sqrt(mean(x^2) + eps) * gamma      (over the c dims)
 *   RoPE_p(x):   pair j = dims (c - R + 2j, c - R + 2j + 1), j < R/2, turns
 *                by angle p * rope_base^(-2j/R)
 * Positions: a query or window row of token t sits at t; compressed entry s
 * at m * s (its block's first token).  Angles are reduced in double
 * precision, so positions of millions keep float-accurate rotations.
 * ------------------------------------------------------------------------ */
typedef struct {
  const float* gamma; /* [c] fp32 RMSNorm weight (device, 16-byte aligned)   */
  float eps;          /* >= 0, finite                                          */
  int32_t rope_dims;  /* R: 0 <= R <= c, R % 8 == 0 (0: no rotation)          */
  float rope_base;    /* > 1 and finite                                        */
} csa_norm_rope;

/* out[b, t, h, :] = RoPE_{t * pos_mul}(RMSNorm(x[b, t, h, :])) for rows
 * [batch, n, heads, c] of `dt` (queries: heads = nh, pos_mul = 1; window
 * rows: heads = 1, pos_mul = 1; compressed entries: n = entries, heads = 1,
 * pos_mul = m).  out may equal x (in place).  c % 8 == 0, c <= 1024. */
csa_status csa_norm_rope_rows(const void* x, int64_t batch, int64_t n, int heads, int c,
                              int64_t pos_mul, const csa_norm_rope* nr, csa_dtype dt, void* out,
                              void* stream);

/* csa_compress followed by RMSNorm + RoPE of each entry i at position m * i
 * (gamma = the KV entries' weight), done as the entries are written (one
 * kernel) wherever an entry's dims tile a block, else as a second in-place
 * pass over the compressed output.  Same arguments and errors as
 * csa_compress, plus `nr` (required). */
csa_status csa_compress_norm_rope(const void* ca, const void* cb, const void* za,
                                  const void* zb, const float* ba, const float* bb,
                                  int64_t batch, int64_t n, int c, int m, int overlap,
                                  csa_dtype dt, const csa_norm_rope* nr, void* out, void* stream);

/* csa_sparse_attn / hca_attn with the query RMSNorm + RoPE (nr->gamma = the
 * query weight) applied in the kernel's prologue and the output's trailing
 * dims rotated by -t in its epilogue.  The entries (kv_comp, kv_win) are
 * taken as given: pass them already normed and rotated (csa_compress_norm_rope
 * and csa_norm_rope_rows).  Same arguments and errors as the plain calls,
 * plus `nr` (required; the tensor-core path takes rope_dims <= 64). */
csa_status csa_sparse_attn_norm_rope(const void* q, const void* kv_comp, const int32_t* idx,
                                     int k, const void* kv_win, int window, const float* sink,
                                     float scale, int64_t batch, int64_t n, int nh, int c, int m,
                                     csa_dtype dt, const csa_norm_rope* nr, void* out,
                                     void* stream);
csa_status hca_attn_norm_rope(const void* q, const void* kv_comp, const void* kv_win, int window,
                              const float* sink, float scale, int64_t batch, int64_t n, int nh,
                              int c, int m_heavy, csa_dtype dt, const csa_norm_rope* nr,
                              void* out, void* stream);

/* ------------------------------------------------------------------------
 * csa_grouped_out_proj -- grouped output projection after core attention
 * ([Walk-through] 4.4: the n_h heads form G groups; each group's
 * concatenated head outputs are projected to d_g, and the G results,
 * concatenated, to the model dim d; [Formulas B9] gives V4-Flash n_h = 64,
 * g = 8, d_g = 1024, d = 4096).  All bf16, fp32 accumulation:
 *   z[r, g d_g + j] = sum_k o[r, g (nh/G) c + k] w1[g, j, k]   (o as [rows, nh c])
 *   y[r, j]         = sum_k z[r, k] w2[j, k]
 *   o : [rows, nh, c]   w1 : [G, d_g, (nh/G) c]   w2 : [d, G d_g]   y : [rows, d]
 *   ws: the intermediate z, [rows, G d_g] bf16 (csa_grouped_out_proj_workspace
 *       bytes; rounded to bf16 between the two products).
 * Needs nh % G == 0, (nh/G) c % 64 == 0, d_g % 256 == 0, d % 256 == 0, else
 * CSA_ERR_UNSUPPORTED.  Pointers 16-byte aligned.
 * ------------------------------------------------------------------------ */
size_t csa_grouped_out_proj_workspace(int64_t rows, int groups, int d_g);
csa_status csa_grouped_out_proj(const void* o, int64_t rows, int nh, int c, int groups, int d_g,
                                int d, const void* w1, const void* w2, void* ws,
                                size_t ws_bytes, void* y, void* stream);

/* ------------------------------------------------------------------------
 * Decode over a persistent cache ([Analysis] "Inference KV Cache": a state
 * cache with the sliding-window rows and the tail waiting for compression,
 * and a classical cache of compressed entries; [Analysis] 7.3 mixed
 * precision: RoPE dims in BF16, the rest in FP8; [Notes] section 2: the
 * tail plus the previous block's overlap state).
 *
 * One cache describes one layer for `batch` sequences.  All decode tensors
 * are bf16 except biases, head weights and sinks (fp32).
 *
 * Cache regions (byte offsets from csa_cache_layout, each 256-byte aligned):
 *   entry_fp8   [batch][capacity][c - rope_dims] u8  E4M3 codes
 *   entry_scale [batch][capacity] fp32              per-entry scale
 *   entry_rope  [batch][capacity][rope_dims] bf16   trailing (RoPE) dims
 *   ikey_fp8    [batch][capacity][c_i] u8           index keys (CSA only)
 *   ikey_scale  [batch][capacity] fp32              (CSA only)
 *   window      [batch][window][c] bf16             raw row of position u at slot u % window
 *   state       raw rows of the compressor tail, bf16:
 *               CSA: [batch][2][4][m][c] then [batch][2][4][m][c_i]
 *                    (block parity (u/m)%2, stream ca/cb/za/zb, row u%m)
 *               HCA: [batch][2][m][c]  (stream C/Z, row u%m)
 * Entry quantisation: scale = amax/448 over the FP8 dims (1 if amax == 0),
 * code = E4M3 round-to-nearest-even saturating of (x / scale); the last
 * rope_dims dims are stored as bf16.  Index keys: c_i FP8 dims, own scale.
 * ------------------------------------------------------------------------ */
typedef struct {
  int64_t batch;     /* sequences                                           */
  int64_t capacity;  /* compressed entries each sequence can hold            */
  int32_t c;         /* entry dim (= head dim)                               */
  int32_t rope_dims; /* trailing dims kept in bf16 (0 <= rope_dims < c)      */
  int32_t c_i;       /* index-key dim (CSA); ignored for HCA                 */
  int32_t m;         /* compression ratio (4 CSA, 128 HCA)                   */
  int32_t window;    /* sliding-window rows                                  */
  int32_t nh;        /* query heads                                          */
  int32_t nh_i;      /* indexer heads (CSA)                                  */
  int32_t k;         /* top-k (CSA)                                          */
  int32_t is_hca;    /* 0: CSA layer (overlap, indexer, top-k); 1: HCA layer  */
} csa_cache_desc;

typedef struct {
  size_t entry_fp8, entry_scale, entry_rope, ikey_fp8, ikey_scale, window, state, istate;
  size_t total_bytes;
} csa_cache_layout_t;

/* Raw per-position rows, each [batch][count][dim] bf16 (dim = c, or c_i for
 * the index streams).  HCA uses ca (= C), za (= Z) and kv_win only. */
typedef struct {
  const void *ca, *cb, *za, *zb;     /* compressor streams, dim c          */
  const void *ica, *icb, *iza, *izb; /* index-key compressor streams, c_i  */
  const void* kv_win;                /* sliding-window rows, dim c          */
} csa_rows;

typedef struct {
  const float *ba, *bb;   /* [m][c] compressor biases (HCA: ba only)        */
  const float *iba, *ibb; /* [m][c_i] index-key compressor biases (CSA)      */
  const float* sink;      /* [nh] sink logits, or NULL                       */
  float scale;            /* logit scale                                     */
  int32_t* sel_out;       /* CSA, optional: [batch][k] int32 device array that
                           * receives each sequence's selected entry indices
                           * (ascending, -1 padded when V <= k); NULL keeps
                           * them in the workspace.  Ignored for HCA.        */
  float* scores_out;      /* CSA, optional: [batch][capacity] fp32 device
                           * array that receives each sequence's indexer
                           * scores I[s] for s < V (the rest untouched); NULL
                           * keeps them in the workspace.  Needs the
                           * tensor-core indexer shape (c_i = 128, nh_i 64 or
                           * 128), else CSA_ERR_UNSUPPORTED.  Ignored for HCA. */
} csa_decode_params;

/* Offsets and total size of a cache for `desc`. Host-only, no launch. */
csa_status csa_cache_layout(const csa_cache_desc* desc, csa_cache_layout_t* layout);

/* Quantise `count` compressed entries per sequence into slots
 * first .. first+count-1 (the hand-off from prefill compression).
 *   kv   : [batch][count][c] of `dt`;  ikey : [batch][count][c_i] of `dt` (CSA; NULL for HCA) */
csa_status csa_cache_store_entries(const csa_cache_desc* desc, void* cache, int64_t first,
                                   int64_t count, const void* kv, const void* ikey,
                                   csa_dtype dt, void* stream);

/* Write raw rows of positions first_pos .. first_pos+count-1 (the same for
 * every sequence) into the window ring and the compressor state, without
 * emitting entries (the hand-off of a prompt's tail to decode). */
csa_status csa_cache_write_rows(const csa_cache_desc* desc, void* cache, int64_t first_pos,
                                int64_t count, const csa_rows* rows, void* stream);

/* Workspace bytes csa_decode_step needs for `desc`. */
size_t csa_decode_workspace(const csa_cache_desc* desc);

/* One decode token per sequence, sequence b at position pos[b] (device
 * int64 [batch]).  In order: (1) write the token's raw rows (count = 1) into
 * the window ring and the compressor state; (2) if (pos+1) % m == 0, compress
 * entry pos/m from the state (CSA: own block + previous block; HCA: own
 * block), quantise it and store it (CSA: also its index key); (3) CSA: score
 * the V = (pos+1)/m visible entries with the indexer and keep the top k;
 * (4) attend over the selected (CSA) or all visible (HCA) entries plus the
 * window with the sink, writing out[b][nh][c] bf16.
 * The cache must already hold entries 0 .. pos/m - 1 and the raw rows of
 * positions pos-window+1 .. pos-1 and of the current and previous block.
 *   q : [batch][nh][c]   q_i : [batch][nh_i][c_i]   w_i : [batch][nh_i] fp32 (CSA) */
csa_status csa_decode_step(const csa_cache_desc* desc, void* cache, const int64_t* pos,
                           const csa_rows* rows, const csa_decode_params* params,
                           const void* q, const void* q_i, const float* w_i, void* out,
                           void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Paged classical cache ([Analysis] "Inference KV Cache": the compressed
 * entries live in a classical cache of blocks allocated per request, each
 * block covering lcm(m, m') raw tokens -- 128 for V4's m = 4 and m' = 128,
 * i.e. 32 CSA entries or 1 HCA entry per block -- so CSA and HCA layers of a
 * sequence share one block table; the state cache (window ring and
 * compressor tail) stays per sequence).  DSA is the special case m = 1 (one
 * entry per token, 128 per block).
 *
 * The entry regions (entry_fp8, entry_scale, entry_rope, ikey_fp8,
 * ikey_scale) then hold num_blocks * (block_tokens / m) rows instead of
 * batch * capacity: entry s of sequence b is row
 *   block_table[b][s / epb] * epb + s % epb,   epb = block_tokens / m.
 * Entries whose block is absent (-1 or >= num_blocks) read as zero and are
 * not written; the caller allocates a sequence's blocks before it reaches
 * them.  desc->capacity must equal max_blocks * epb.  epb must be a power of
 * two, and at least 32 for CSA layers.
 * ------------------------------------------------------------------------ */
typedef struct {
  int32_t block_tokens;        /* raw tokens per block (a multiple of m)          */
  int64_t num_blocks;          /* blocks in the pool                              */
  int64_t max_blocks;          /* block-table row length                          */
  const int32_t* block_table;  /* device [batch][max_blocks] int32 (-1: absent)    */
} csa_paging;

/* The paged forms of csa_cache_layout, csa_cache_store_entries,
 * csa_cache_write_rows and csa_decode_step: same arguments and results,
 * plus the paging; csa_decode_workspace applies unchanged. */
csa_status csa_paged_cache_layout(const csa_cache_desc* desc, const csa_paging* paging,
                                  csa_cache_layout_t* layout);
csa_status csa_paged_cache_store_entries(const csa_cache_desc* desc, const csa_paging* paging,
                                         void* cache, int64_t first, int64_t count,
                                         const void* kv, const void* ikey, csa_dtype dt,
                                         void* stream);
csa_status csa_paged_cache_write_rows(const csa_cache_desc* desc, const csa_paging* paging,
                                      void* cache, int64_t first_pos, int64_t count,
                                      const csa_rows* rows, void* stream);
csa_status csa_paged_decode_step(const csa_cache_desc* desc, const csa_paging* paging,
                                 void* cache, const int64_t* pos, const csa_rows* rows,
                                 const csa_decode_params* params, const void* q,
                                 const void* q_i, const float* w_i, void* out, void* ws,
                                 size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
