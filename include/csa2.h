/*
 * csa2.h -- C ABI of the CSA2 hot path on B200 (sm_100a).
 *
 * CSA2 is compressed sparse attention over a global KV cache that several
 * layers share, stored in four-bit numbers ("DeepSeek-V4.1 模型结构（0）", 延伸解读
 * "CSA2 共享池：四种层模式如何分工"; "从V4到V4.1 Flash：架构的激进进化", section
 * "CSA2架构：跨层压缩的创新方案").  Each layer runs in one of three modes:
 *   Full    -- score every cache entry with the lightning indexer, keep top-k;
 *   Reindex -- reuse the shared cache, score only a candidate pool with the
 *              layer's own indexer query, keep top-k inside the pool;
 *   Reuse   -- reuse the shared cache and the given top-k indices, no indexer.
 * A 128-token sliding-window (SWA) branch over a per-layer FP8 cache runs beside
 * it and the two are combined by log-sum-exp.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every pointer argument is a DEVICE pointer owned by the caller unless the
 *    comment says "host".  The library never allocates or frees memory; calls
 *    that need scratch take a caller workspace sized by csa2_workspace_size().
 *  - Every compute call is asynchronous on `stream` (0 = legacy default stream)
 *    and returns a csa2_status for the host-side checks and the launch itself.
 *  - Errors found on the device (an index or page outside the cache) never trap:
 *    the kernel skips the bad access and stores the status code into *err (a
 *    caller-owned device int32, first error wins), read back by csa2_check().
 *  - A call with no work (a batch, token, row or query count of 0) returns CSA2_OK
 *    without reading any pointer or launching anything; negative sizes are errors.
 *  - bf16 tensors are passed as `const uint16_t*` (raw bf16 bits).
 *  - Fixed dimensions: main-KV and query head dim 512, indexer dim 128,
 *    query heads H = 64, indexer heads H_I = 64.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *csa2_stream_t; /* a cudaStream_t */

typedef enum {
  CSA2_OK = 0,
  CSA2_ERR_INVALID_ARG = 1, /* null pointer, bad enum, negative size */
  CSA2_ERR_SHAPE = 2,       /* sizes inconsistent with each other or the cache */
  CSA2_ERR_UNSUPPORTED = 3, /* a valid request this build does not implement */
  CSA2_ERR_CUDA = 4,        /* launch or runtime error (see csa2_last_error_string) */
  CSA2_ERR_INDEX = 5,       /* device side: an index or page outside the cache */
  CSA2_ERR_TIMEOUT = 6      /* device side: a bounded wait gave up */
} csa2_status;

/* CSA2_MODE_DENSE attends every visible entry (no indexer, no indices): the
 * predecessor's heavily compressed attention ("DeepSeek V4.1 Flash 深度解析",
 * 本专栏篇目 "前代 · HCA": 128-fold compression, then dense attention). */
typedef enum {
  CSA2_MODE_FULL = 0,
  CSA2_MODE_REINDEX = 1,
  CSA2_MODE_REUSE = 2,
  CSA2_MODE_DENSE = 3
} csa2_mode;
typedef enum { CSA2_F32 = 0, CSA2_BF16 = 1 } csa2_dtype;

enum {
  CSA2_MAIN_DIM = 512,        /* values per main-KV entry */
  CSA2_MAIN_CODE_BYTES = 256, /* two e2m1 codes per byte, element 2i in the low nibble */
  CSA2_MAIN_SCALE_BYTES = 32, /* one E4M3 scale per block of 16 values */
  CSA2_IX_DIM = 128,          /* values per indexer key */
  CSA2_IX_CODE_BYTES = 64,    /* two e2m1 codes per byte */
  CSA2_IX_SCALE_BYTES = 4,    /* one E8M0 exponent per block of 32 values */
  CSA2_SWA_DIM = 512,         /* E4M3 codes per SWA token, plus one fp32 scale */
  CSA2_HEADS = 64,            /* query heads H */
  CSA2_IX_HEADS = 64          /* indexer heads H_I */
};

/*
 * The shared global KV cache ("DeepSeek-V4.1 模型结构（0）", Q&A "890 字节全局 KV
 * 是怎么算出来的": a main-KV entry is 512 four-bit numbers plus 32 bytes of scale,
 * 288 bytes; an indexer-K entry is 128 four-bit numbers plus 4 bytes of scale,
 * 68 bytes).  The four byte planes are kept apart (structure of arrays) so that
 * every row starts 16-byte aligned; bytes per entry are still 288 + 68.
 *
 * Physical slot of entry n of sequence b:
 *   contiguous (page_table == NULL): b * seq_stride + n, with n < seq_stride;
 *   paged: page_table[b * max_pages + n / page_size] * page_size + n % page_size.
 * Row s of a plane starts at plane + s * (row bytes).  num_slots bounds every slot.
 * ratio is the compression ratio of the layer that wrote the cache: an entry
 * pools `ratio` tokens, so a query at position p sees entries
 * n < min(num_entries[b], (p + 1) / ratio).
 */
typedef struct {
  uint8_t *kv_codes;          /* [num_slots][256] */
  uint8_t *kv_scales;         /* [num_slots][32]  */
  uint8_t *ix_codes;          /* [num_slots][64]  */
  uint8_t *ix_scales;         /* [num_slots][4]   */
  const int32_t *page_table;  /* [batch][max_pages] or NULL (contiguous) */
  const int32_t *num_entries; /* [batch] entries present per sequence */
  int64_t num_slots;          /* rows allocated in each plane */
  int32_t batch;              /* sequences described by this cache */
  int32_t ratio;              /* tokens per entry, >= 1 */
  int32_t seq_stride;         /* contiguous layout: slots per sequence */
  int32_t page_size;          /* paged layout: entries per page (power of two) */
  int32_t max_pages;          /* paged layout: page-table row length */
} csa2_cache;

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int csa2_version(void);

/* Text of the last host-side error on this thread ("" if none).  Static storage. */
const char *csa2_last_error_string(void);

/*
 * Synchronises `stream`, reads the caller's device error word and returns it as
 * a csa2_status (CSA2_OK when zero).  Does not clear it.
 */
csa2_status csa2_check(const int32_t *err, csa2_stream_t stream);

/*
 * Bytes of workspace csa2_sparse_attn needs for these sizes (0 for Reuse, and for
 * Dense up to 4096 entries).  max_entries bounds num_entries[b]; pool_k is the
 * candidate-pool size (0 if none).  Full mode with B * Q >= 1024 query rows and no
 * pool (a prefill chunk), and Reindex over a pool of at most 16384 candidates, select
 * without materialising scores and need only the B * Q * k selection.
 */
size_t csa2_workspace_size(csa2_mode mode, int32_t B, int32_t Q, int32_t max_entries,
                           int32_t k, int32_t pool_k);

/*
 * Token compressor + packer: writes floor(T / ratio) new entries per sequence.
 * ("从V4到V4.1 Flash", section 编码器层: about two tokens per main-KV entry in
 * the encoder; section 解码器层: ratio 1 in the decoder; "DeepSeek-V4.1 模型结构（0）",
 * Q&A on the 890 bytes: entry formats.)
 *   lat_kv  [B][T][512] and lat_ix [B][T][128] in `dtype` (fp32 or bf16);
 *   pool_w  [B][T] fp32 pooling weights, or NULL for fp32(1/ratio);
 *   entry j of sequence b = sum over t in [j*r, j*r + r) of pool_w * lat, fp32,
 *   left to right; then per block of 16 an E4M3 scale = RNE(amax / 6) and e2m1
 *   codes RNE(x / scale); per block of 32 of the indexer key an E8M0 exponent
 *   ceil(log2(amax / 6)) and e2m1 codes.  A block with a zero scale has zero codes.
 *   first_entry [B] (device): entry index of the first new entry of sequence b.
 * Writes the four planes only; the caller updates num_entries.
 * Device errors: a slot outside the cache -> CSA2_ERR_INDEX in *err, entry skipped.
 */
csa2_status csa2_pack_kv(const void *lat_kv, const void *lat_ix, csa2_dtype dtype,
                         const float *pool_w, int32_t B, int32_t T, const int32_t *first_entry,
                         const csa2_cache *cache, int32_t *err, csa2_stream_t stream);

/*
 * csa2_pack_kv with a learned (gated) pooling: the encoder pools about two tokens
 * per entry ("从V4到V4.1 Flash", section 编码器层) by a rule the pages do not give;
 * this call reads it as a gated sum.  For each channel d of entry j,
 *   x_d = sum over t in the group of softmax_t(g_t,d) * lat_t,d,
 * the softmax taken over the group's r tokens: m = max g, e_t = exp(g_t,d - m),
 * weights e_t / (sum of e, left to right), products summed left to right, every step
 * one fp32 operation and exp evaluated by a fixed fp32 sequence (2^f by its degree-7
 * Taylor polynomial after n = rint(x log2 e)), so the codes do not depend on a math
 * library.  Then quantised as csa2_pack_kv.
 *   gate_kv [B][T][512], gate_ix [B][T][128] fp32 gate logits (computed by the model);
 *   the other arguments as csa2_pack_kv.  Equal logits give csa2_pack_kv's mean.
 */
csa2_status csa2_pack_kv_gated(const void *lat_kv, const void *lat_ix, csa2_dtype dtype,
                               const float *gate_kv, const float *gate_ix, int32_t B, int32_t T,
                               const int32_t *first_entry, const csa2_cache *cache, int32_t *err,
                               csa2_stream_t stream);

/*
 * SWA packer: per token an fp32 scale = amax / 448 and 512 E4M3 codes RNE(x / scale)
 * (saturating), stored in a per-layer ring at slot pos mod R.  ("DeepSeek V4.1 Flash
 * 深度解析", 本专栏篇目 "FP4 从权重走进 KV 缓存": the sliding-window cache stays FP8;
 * "从V4到V4.1 Flash", section "SWA 有界重放": the window keeps the last 128 tokens.)
 *   x [B][T][512] in `dtype`; pos [B][T] absolute positions (device), a negative
 *   position marks a padding token that is skipped;
 *   swa_codes [B][R][512] u8; swa_scale [B][R] fp32.
 * Positions of one sequence's tokens in a call are consecutive, so only the
 * last R tokens of the call are stored (earlier ones would be overwritten).
 */
csa2_status csa2_pack_swa(const void *x, csa2_dtype dtype, int32_t B, int32_t T,
                          const int32_t *pos, uint8_t *swa_codes, float *swa_scale, int32_t R,
                          int32_t *err, csa2_stream_t stream);

/*
 * Lightning-indexer scores ("DeepSeek V4.1 Flash 深度解析", 本专栏篇目 "前代 · CSA":
 * an FP4 lightning indexer picks top-512; the score formula is the weighted-ReLU
 * form s_n = sum_h w_h * relu(q^_h . k^_n) with q^ the per-32 E8M0/e2m1
 * quantisation of the query heads).
 *   q_ix [B][Q][64][128] bf16; w [B][Q][64] bf16; q_pos [B][Q] positions;
 *   cand [B][Q][P] entry indices (-1 = none) or NULL to score entries 0..N-1;
 *   scores [B][Q][N_out] fp32 with N_out = P when cand != NULL else max_entries.
 * Entries not visible to the query (see csa2_cache) and -1 candidates score -inf.
 * Device errors: a candidate >= num_entries[b] or a bad page -> CSA2_ERR_INDEX, -inf;
 * without candidates, a query that sees more than max_entries entries ->
 * CSA2_ERR_SHAPE (only its first max_entries entries are scored).
 */
csa2_status csa2_index_score(const uint16_t *q_ix, const uint16_t *w, int32_t B, int32_t Q,
                             const int32_t *q_pos, const int32_t *cand, int32_t P,
                             int32_t max_entries, const csa2_cache *cache, float *scores,
                             int32_t *err, csa2_stream_t stream);

/*
 * Top-k of each row ("DeepSeek-V4.1 模型结构（0）", 延伸解读 CSA2 共享池: top-512;
 * "从V4到V4.1 Flash", section 解码器层: a candidate pool, then top-512 inside it).
 *   scores [R][N] fp32; n_valid [R] (device) or NULL = N: candidates are positions
 *   j < n_valid[r] whose score is not -inf, ordered by score descending, then j
 *   ascending.  idx [R][k] receives the first k positions in ascending order,
 *   padded with -1; val [R][k] (optional) their scores (-inf for pads).
 *   A second selection of the same rows (k2 > 0 with idx2 [R][k2], val2 optional),
 *   e.g. the candidate pool, is computed in the same passes; k2 = 0 for none.
 *   No workspace is needed.  NaN scores give an unspecified selection.
 */
csa2_status csa2_topk(const float *scores, const int32_t *n_valid, int32_t R, int32_t N,
                      int32_t k, int32_t *idx, float *val, int32_t k2, int32_t *idx2, float *val2,
                      csa2_stream_t stream);

/*
 * The Full-mode selection of a chunk of query tokens without materialising scores
 * ("DeepSeek V4.1 Flash 深度解析", 序: prefill compute, HBM and SSD capacity are the
 * bottlenecks; "从V4到V4.1 Flash", 编码器层: prefill runs the encoder's CSA2 layers over
 * the whole prompt).  For every query: the scores of csa2_index_score over the entries
 * it sees, then the top-k of csa2_topk -- the same selection, bit for bit.  Three
 * query tokens share each key tile loaded; each keeps a running top-k on chip.
 *   q_ix [B][Q][64][128], w [B][Q][64] bf16; q_pos [B][Q]; idx [B][Q][k] int32,
 *   ascending entries, -1 padded; k <= 512.  No workspace.
 * Efficient for hundreds of query tokens or more (a prefill chunk); decode rows are
 * better served by csa2_index_score + csa2_topk, which spread one row over the GPU.
 * Device errors: a query that sees more than max_entries entries -> CSA2_ERR_SHAPE
 * (only the first max_entries are scored); a bad page -> CSA2_ERR_INDEX.
 */
csa2_status csa2_index_topk(const uint16_t *q_ix, const uint16_t *w, int32_t B, int32_t Q,
                            const int32_t *q_pos, int32_t k, int32_t max_entries,
                            const csa2_cache *cache, int32_t *idx, int32_t *err,
                            csa2_stream_t stream);

/*
 * Sparse attention of one CSA2 layer ("从V4到V4.1 Flash", section CSA2架构: the
 * Full, Reindex and Reuse modes; section 解码器层: the hierarchical pool).
 *   q [B][Q][64][512] bf16 query heads; q_pos [B][Q]; softmax_scale tau.
 *   FULL:    q_ix, w (as csa2_index_score) select top-k of all visible entries;
 *            if pool_k > 0 the top-pool_k entries are written to pool_io [B][Q][pool_k].
 *            With B * Q >= 1024 rows and pool_k = 0 (prefill) the indexer scores three
 *            query tokens per key tile and keeps each one's running top-k on chip
 *            ("DeepSeek V4.1 Flash 深度解析", 序: prefill compute is the bottleneck);
 *            the selection is the same as scoring and csa2_topk would give.
 *   REINDEX: q_ix, w score the entries listed in pool_io [B][Q][pool_k]; top-k of them
 *            (ties: the earlier candidate).  Pools of at most 16384: one launch per row
 *            group, each row's scores gathered in one CTA's shared memory and selected
 *            there (the same selection as scoring and csa2_topk with the pool as map).
 *   REUSE:   idx_in [B][Q][k] given entry indices (-1 = none; order free).
 *   DENSE:   every visible entry (q_ix, w, k, pool and indices unused); the caches of
 *            the predecessor's 128-fold compressed layers are read this way.  Any
 *            number of entries: beyond one segment of 4096 or 8192 entries the
 *            segments' partial results are merged through the workspace.
 *   idx_out [B][Q][k] (optional, FULL/REINDEX) receives the chosen entries, ascending.
 *   k <= 512 (FULL, REINDEX, REUSE).
 * The bf16 query enters the tensor cores scaled by a power of two per head, so every
 * value within a factor 2^32 of its head's largest is used exactly.
 * Per head: logits tau * q . v_j over the chosen entries, v_j the dequantised
 * 512-d main entry used as key and value; o [B][Q][64][512] fp32 = softmax-weighted
 * sum, lse [B][Q][64] fp32 natural-log normaliser; no entries -> o = 0, lse = -inf.
 * Optional sliding-window branch in the same call: when swa_codes != NULL the
 * window of each query (as csa2_swa_attn: ring [B][R], window <= 128) joins the
 * same softmax, so o / lse are the log-sum-exp merge of the two branches
 * (what csa2_merge of the separate results gives).  swa_codes = NULL: none.
 * swa_new [B][1][512] bf16 (decode, Q == 1, with the window branch; NULL: none): this step's
 * token of each sequence for the window, quantised inside the launch exactly as csa2_pack_swa
 * quantises it, written to ring slot q_pos mod R (codes and scale) and used as the window's last
 * key -- csa2_pack_swa followed by this call, in one launch ("从V4到V4.1 Flash", SWA 有界重放).
 * 8-byte aligned.
 * ws: csa2_workspace_size(mode, ...) bytes (may be NULL for REUSE).
 * Device errors: an index outside the visible entries -> CSA2_ERR_INDEX, skipped;
 * FULL or DENSE with a query that sees more than max_entries entries -> CSA2_ERR_SHAPE
 * (max_entries must bound the visible entries; the tail is left out).
 */
csa2_status csa2_sparse_attn(csa2_mode mode, const uint16_t *q, int32_t B, int32_t Q,
                             const int32_t *q_pos, float softmax_scale, const uint16_t *q_ix,
                             const uint16_t *w, int32_t k, int32_t pool_k, int32_t *pool_io,
                             const int32_t *idx_in, int32_t *idx_out, int32_t max_entries,
                             const csa2_cache *cache, const uint8_t *swa_codes,
                             const float *swa_scale, int32_t R, int32_t window,
                             const uint16_t *swa_new, float *o, float *lse, void *ws,
                             size_t ws_bytes, int32_t *err, csa2_stream_t stream);

/*
 * Sliding-window branch ("从V4到V4.1 Flash", sections "CSA2 机制下的全局 KV 共享与局部
 * 滑动窗口隔离" (per-layer SWA cache) and "SWA 有界重放" (128 tokens)).
 *   Window of a query at p: positions max(0, p - window + 1) .. p, read from the
 *   ring written by csa2_pack_swa (slot t mod R, R >= window, window <= 128).
 *   Keys = values = E4M3 code * fp32 scale.  Same o / lse as csa2_sparse_attn.
 */
csa2_status csa2_swa_attn(const uint16_t *q, int32_t B, int32_t Q, const int32_t *q_pos,
                          const uint8_t *swa_codes, const float *swa_scale, int32_t R,
                          int32_t window, float softmax_scale, float *o, float *lse,
                          int32_t *err, csa2_stream_t stream);

/*
 * Log-sum-exp merge of the sparse and sliding-window branches ("从V4到V4.1 Flash",
 * section 移除混合注意力机制: CSA mixed with SWA): m = max(l1, l2),
 * o = (e^(l1-m) o1 + e^(l2-m) o2) / (e^(l1-m) + e^(l2-m)), lse = m + log(...).
 *   o1, o2, o [rows][D] fp32; l1, l2, lse [rows].  o may alias o1 or o2 and lse
 *   may alias l1 or l2.  Both -inf -> o = 0, lse = -inf.
 */
csa2_status csa2_merge(const float *o1, const float *l1, const float *o2, const float *l2,
                       int64_t rows, int32_t D, float *o, float *lse, csa2_stream_t stream);

/*
 * Decode-time append of one token per sequence to a cache written at ratio r
 * ("从V4到V4.1 Flash", section 编码器层: the encoder pools about two tokens per entry;
 * section 解码器层: the decoder keeps ratio 1).  The token at position pos[b] is kept,
 * in fp32, in row pos % r of the sequence's staging buffer; when it completes a group
 * of r tokens, the group is pooled and packed exactly as csa2_pack_kv does (fp32, left
 * to right, weight fp32(1/r)) into entry pos / r, and cache->num_entries[b] is raised
 * to pos / r + 1 (this call writes num_entries on the device).
 *   lat_kv [B][512], lat_ix [B][128] in `dtype`; pos [B] (negative: skip the row);
 *   stage [B][r][640] fp32 (512 main then 128 indexer values), may be NULL when r = 1;
 *   it carries the incomplete group from call to call.
 * Device errors: an entry outside the cache -> CSA2_ERR_INDEX, skipped.
 */
csa2_status csa2_append_kv(const void *lat_kv, const void *lat_ix, csa2_dtype dtype, int32_t B,
                           const int32_t *pos, float *stage, const csa2_cache *cache, int32_t *err,
                           csa2_stream_t stream);

/*
 * Multi-layer decode: one token per sequence through a stack of layers.
 * ("DeepSeek-V4.1 模型结构（0）", Q&A "DeepSeek-V4.1-Flash 的 40 层具体如何排布？": layers
 * 0-1 use only the sliding window, 2 / 8 / 14 / 20 are Full, 24 / 28 / 32 / 36 Reindex,
 * the other 30 Reuse; 延伸解读 "CSA2 共享池": only the Full layers produce global KV;
 * "从V4到V4.1 Flash", 解码器层: the decoder's first layer keeps a candidate pool that the
 * later layers search.)
 * A layer's plan: its mode (a csa2_mode or CSA2_LAYER_SWA), the earlier layer it takes
 * its entries from (Reuse) or whose pool it searches (Reindex, a Full layer), and the
 * global cache it reads (Full: the one it writes).
 */
#define CSA2_LAYER_SWA 4
typedef struct {
  int32_t mode;
  int32_t source; /* -1 unless Reuse or Reindex */
  int32_t cache;  /* index into the step's caches, -1 for CSA2_LAYER_SWA */
} csa2_layer_plan;

/*
 * The pages' 40-layer plan into plan[0..39] (host) and, if cache_ratio (host [4]) is
 * given, its caches' ratios: caches 0-2 are written by the encoder's Full layers 2, 8, 14
 * at ratio 2, cache 3 by the decoder's Full layer 20 at ratio 1, whose pool the Reindex
 * layers search; every Reuse layer takes the nearest earlier Full or Reindex layer's
 * entries.  Returns 40 (and writes nothing when max_layers < 40).
 */
int32_t csa2_plan_v41(csa2_layer_plan *plan, int32_t max_layers, int32_t *cache_ratio);

/*
 * One decode step.  Host fields: n_layers, plan, n_caches, caches, max_entries and the
 * sizes; every other pointer is device memory, layer-major.  For each layer l:
 *   q [L][B][64][512], q_ix [L][B][64][128], w [L][B][64] bf16 (q_ix / w are read only
 *   for Full and Reindex layers); swa_x [L][B][512] bf16, this token's hidden state for
 *   the layer's ring swa_codes [L][B][R][512] / swa_scale [L][B][R] (quantised as
 *   csa2_pack_swa does and stored by the layer's attention launch);
 *   idx [L][B][k]: Full and Reindex layers write the entries they chose (a Reuse layer
 *   attends its source's row); o [L][B][64][512], lse [L][B][64] fp32 as csa2_sparse_attn
 *   with the window merged.
 * Caches: new_kv [n_caches][B][512] and new_ix [n_caches][B][128] bf16 are this token's
 * latents per cache (NULL: no append), appended as csa2_append_kv does before the first
 * layer that reads the cache, with staging kv_stage [n_caches][B][rmax][640] fp32 (rmax =
 * the largest ratio); pool [n_caches][B][pool_k] holds the pool of the cache's Full layer
 * when a Reindex layer searches it.  max_entries [n_caches] (host) bounds each cache's
 * entries after the append.
 * The layers run in order, each with its own launches (a Full layer: indexer scan, top-k,
 * attention; Reindex the same over the pool; Reuse and window-only layers: one attention
 * launch), on `stream` without synchronising or allocating (capturable in a CUDA graph).
 * Dense layers hold at most one segment (4096 entries).
 */
typedef struct {
  int32_t n_layers;
  const csa2_layer_plan *plan;
  int32_t n_caches;
  const csa2_cache *caches;
  const int32_t *max_entries;
  int32_t B;
  const int32_t *pos; /* [B] position of this step's token */
  float softmax_scale;
  int32_t k, pool_k;
  const uint16_t *q, *q_ix, *w;
  const uint16_t *new_kv, *new_ix;
  float *kv_stage;
  const uint16_t *swa_x;
  uint8_t *swa_codes;
  float *swa_scale;
  int32_t R, window;
  int32_t *idx, *pool;
  float *o, *lse;
} csa2_decode_args;

/* Workspace bytes csa2_decode_step needs: the largest Full layer's fp32 scores (and a
 * Reindex layer's, for pools above 16384); 0 when no layer needs any (ws may be NULL). */
size_t csa2_decode_workspace_size(const csa2_decode_args *args);
csa2_status csa2_decode_step(const csa2_decode_args *args, void *ws, size_t ws_bytes, int32_t *err,
                             csa2_stream_t stream);

/*
 * csa2_sparse_attn without a caller workspace.  (The pages have no counterpart:
 * this is a convenience of this library.)  For callers that cannot allocate
 * device memory -- e.g. an engine whose pool already holds the whole device, or
 * a serving loop that forbids cudaMalloc/cudaFree on its hot path because they
 * synchronise the device.  Same arguments and results as csa2_sparse_attn minus
 * ws / ws_bytes.  Scratch comes from a fixed array inside the library of
 * CSA2_NOALLOC_SCRATCH_BYTES (8 MiB; every GPU that loads the library holds it
 * until the process exits); calls whose csa2_workspace_size exceeds it return
 * CSA2_ERR_UNSUPPORTED with a message.  It allocates nothing itself.
 *   - Every call looks up the array's device address on the current device (the
 *     lookup loads the library's module on a device's first call, so make that
 *     first call before any stream capture); nothing is cached, so the entry
 *     point stays valid after a device reset.
 *   - All calls on a device share the one array and each call overwrites it
 *     (no part of it needs to start at zero); calls that overlap on the GPU --
 *     on different streams, or from different host threads -- race.
 */
#define CSA2_NOALLOC_SCRATCH_BYTES (8u << 20)
size_t csa2_noalloc_scratch_bytes(void);
csa2_status csa2_sparse_attn_noalloc(csa2_mode mode, const uint16_t *q, int32_t B, int32_t Q,
                                     const int32_t *q_pos, float softmax_scale,
                                     const uint16_t *q_ix, const uint16_t *w, int32_t k,
                                     int32_t pool_k, int32_t *pool_io, const int32_t *idx_in,
                                     int32_t *idx_out, int32_t max_entries,
                                     const csa2_cache *cache, const uint8_t *swa_codes,
                                     const float *swa_scale, int32_t R, int32_t window, float *o,
                                     float *lse, int32_t *err, csa2_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */
