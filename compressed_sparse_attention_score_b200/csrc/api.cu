// The C ABI of the CSA2 library: argument checks, workspace carving, launches.
#include <cuda_runtime.h>

#include <cstdio>
#include <string>

#include "../../include/csa2.h"
#include "kernels.cuh"

#define CSA2_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

thread_local std::string g_last_error;

csa2_status fail(csa2_status s, const char *msg) {
  g_last_error = msg;
  return s;
}

csa2_status launched(const char *what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
    return CSA2_ERR_CUDA;
  }
  g_last_error.clear();
  return CSA2_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

csa2_status check_cache(const csa2_cache *c, int B) {
  if (!c) return fail(CSA2_ERR_INVALID_ARG, "cache is NULL");
  if (!c->kv_codes || !c->kv_scales || !c->ix_codes || !c->ix_scales || !c->num_entries)
    return fail(CSA2_ERR_INVALID_ARG, "cache plane or num_entries is NULL");
  if (!aligned16(c->kv_codes) || !aligned16(c->ix_codes) || !aligned16(c->kv_scales) || (reinterpret_cast<uintptr_t>(c->ix_scales) & 3))
    return fail(CSA2_ERR_INVALID_ARG, "cache planes must be 16-byte aligned (ix_scales 4-byte)");
  if (c->ratio < 1) return fail(CSA2_ERR_INVALID_ARG, "cache ratio must be >= 1");
  if (c->num_slots < 0 || c->batch < 0) return fail(CSA2_ERR_INVALID_ARG, "negative cache size");
  if (B > c->batch) return fail(CSA2_ERR_SHAPE, "B exceeds cache batch");
  if (c->page_table) {
    if (c->page_size <= 0 || (c->page_size & (c->page_size - 1)) || c->max_pages <= 0)
      return fail(CSA2_ERR_INVALID_ARG, "paged cache needs a power-of-two page_size and max_pages > 0");
  } else if (c->seq_stride <= 0) {
    return fail(CSA2_ERR_INVALID_ARG, "contiguous cache needs seq_stride > 0");
  }
  return CSA2_OK;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Dense attention runs over segments of csa2::attn_dense_segment() entries (8192, or 4096 on a
// device that cannot hold a 16-CTA cluster); the workspace is sized for the smaller.
constexpr int kDenseMinSegment = 4096;

// Full mode with this many query rows or more (a prefill chunk) and no pool selects with the
// fused prefill indexer: each CTA serves 3 query tokens over every key tile they see, so there
// must be enough of them to fill the device; the scores are never materialised.
constexpr int64_t kFusedPrefillRows = 1024;
bool fused_prefill(int64_t rows, int32_t pool_k) { return rows >= kFusedPrefillRows && pool_k == 0; }

}  // namespace

namespace csa2 {
// Lets other translation units of the library set the thread's error text.
void set_last_error(const char *msg) { g_last_error = msg; }
}  // namespace csa2

CSA2_EXPORT int csa2_version(void) { return 100; }

CSA2_EXPORT const char *csa2_last_error_string(void) { return g_last_error.c_str(); }

CSA2_EXPORT csa2_status csa2_check(const int32_t *err, csa2_stream_t stream) {
  if (!err) return fail(CSA2_ERR_INVALID_ARG, "err is NULL");
  int32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, err, sizeof(h), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) {
    g_last_error = std::string("csa2_check: ") + cudaGetErrorString(e);
    return CSA2_ERR_CUDA;
  }
  return csa2_status(h);
}

CSA2_EXPORT size_t csa2_workspace_size(csa2_mode mode, int32_t B, int32_t Q, int32_t max_entries, int32_t k,
                                       int32_t pool_k) {
  if (B < 0 || Q < 0 || max_entries < 0 || k < 0 || pool_k < 0) return 0;
  const size_t rows = size_t(B) * Q;
  switch (mode) {
    case CSA2_MODE_FULL:
      return (fused_prefill(int64_t(rows), pool_k) ? 0 : round256(rows * max_entries * 4)) + round256(rows * k * 4);
    case CSA2_MODE_REINDEX:  // pools of at most REINDEX_SELECT_MAX: scores never leave the chip
      return (pool_k <= csa2::REINDEX_SELECT_MAX ? 0 : round256(rows * pool_k * 4)) + round256(rows * k * 4);
    case CSA2_MODE_DENSE:  // partial (o, lse) of one key segment beyond the first
      return max_entries > kDenseMinSegment ? round256(rows * CSA2_HEADS * CSA2_MAIN_DIM * 4) +
                                                  round256(rows * CSA2_HEADS * 4)
                                            : 0;
    default: return 0;
  }
}

CSA2_EXPORT csa2_status csa2_pack_kv(const void *lat_kv, const void *lat_ix, csa2_dtype dtype, const float *pool_w,
                                     int32_t B, int32_t T, const int32_t *first_entry, const csa2_cache *cache,
                                     int32_t *err, csa2_stream_t stream) {
  if (B < 0 || T < 0) return fail(CSA2_ERR_INVALID_ARG, "negative size");
  if (B == 0 || T == 0) return CSA2_OK;
  if (csa2_status s = check_cache(cache, B)) return s;
  if (!lat_kv || !lat_ix || !first_entry) return fail(CSA2_ERR_INVALID_ARG, "NULL input");
  if (dtype != CSA2_F32 && dtype != CSA2_BF16) return fail(CSA2_ERR_INVALID_ARG, "bad dtype");
  if (!aligned16(lat_kv) || (reinterpret_cast<uintptr_t>(lat_ix) & 7)) return fail(CSA2_ERR_INVALID_ARG, "latents misaligned");
  csa2::launch_pack_kv(lat_kv, lat_ix, dtype, pool_w, nullptr, nullptr, B, T, first_entry, *cache, err, stream);
  return launched("csa2_pack_kv");
}

CSA2_EXPORT csa2_status csa2_pack_kv_gated(const void *lat_kv, const void *lat_ix, csa2_dtype dtype,
                                           const float *gate_kv, const float *gate_ix, int32_t B, int32_t T,
                                           const int32_t *first_entry, const csa2_cache *cache, int32_t *err,
                                           csa2_stream_t stream) {
  if (B < 0 || T < 0) return fail(CSA2_ERR_INVALID_ARG, "negative size");
  if (B == 0 || T == 0) return CSA2_OK;
  if (csa2_status s = check_cache(cache, B)) return s;
  if (!lat_kv || !lat_ix || !gate_kv || !gate_ix || !first_entry) return fail(CSA2_ERR_INVALID_ARG, "NULL input");
  if (dtype != CSA2_F32 && dtype != CSA2_BF16) return fail(CSA2_ERR_INVALID_ARG, "bad dtype");
  if (!aligned16(lat_kv) || (reinterpret_cast<uintptr_t>(lat_ix) & 7) || !aligned16(gate_kv) || !aligned16(gate_ix))
    return fail(CSA2_ERR_INVALID_ARG, "latents or gates misaligned");
  csa2::launch_pack_kv(lat_kv, lat_ix, dtype, nullptr, gate_kv, gate_ix, B, T, first_entry, *cache, err, stream);
  return launched("csa2_pack_kv_gated");
}

CSA2_EXPORT csa2_status csa2_pack_swa(const void *x, csa2_dtype dtype, int32_t B, int32_t T, const int32_t *pos,
                                      uint8_t *swa_codes, float *swa_scale, int32_t R, int32_t *err,
                                      csa2_stream_t stream) {
  if (B < 0 || T < 0 || R < 1) return fail(CSA2_ERR_INVALID_ARG, "bad size");
  if (B == 0 || T == 0) return CSA2_OK;
  if (!x || !pos || !swa_codes || !swa_scale) return fail(CSA2_ERR_INVALID_ARG, "NULL input");
  if (dtype != CSA2_F32 && dtype != CSA2_BF16) return fail(CSA2_ERR_INVALID_ARG, "bad dtype");
  if (!aligned16(x) || !aligned16(swa_codes)) return fail(CSA2_ERR_INVALID_ARG, "x / swa_codes misaligned");
  csa2::launch_pack_swa(x, dtype, B, T, pos, B, swa_codes, swa_scale, R, err, stream);
  return launched("csa2_pack_swa");
}

CSA2_EXPORT csa2_status csa2_index_score(const uint16_t *q_ix, const uint16_t *w, int32_t B, int32_t Q,
                                         const int32_t *q_pos, const int32_t *cand, int32_t P, int32_t max_entries,
                                         const csa2_cache *cache, float *scores, int32_t *err,
                                         csa2_stream_t stream) {
  if (B < 0 || Q < 0 || max_entries < 0 || (cand && P <= 0)) return fail(CSA2_ERR_INVALID_ARG, "bad size");
  if (B == 0 || Q == 0) return CSA2_OK;
  if (csa2_status s = check_cache(cache, B)) return s;
  if (!q_ix || !w || !q_pos || !scores) return fail(CSA2_ERR_INVALID_ARG, "NULL input");
  if (!aligned16(q_ix)) return fail(CSA2_ERR_INVALID_ARG, "q_ix misaligned");
  const int n_out = cand ? P : max_entries;
  if (size_t(B) * Q > 65535) return fail(CSA2_ERR_UNSUPPORTED, "more than 65535 query rows per call");
  csa2::launch_index_score_mma(q_ix, w, B, Q, q_pos, cand, P, n_out, *cache, scores, err, stream);
  return launched("csa2_index_score");
}

CSA2_EXPORT csa2_status csa2_index_topk(const uint16_t *q_ix, const uint16_t *w, int32_t B, int32_t Q,
                                        const int32_t *q_pos, int32_t k, int32_t max_entries,
                                        const csa2_cache *cache, int32_t *idx, int32_t *err, csa2_stream_t stream) {
  if (B < 0 || Q < 0 || max_entries < 0 || k < 1) return fail(CSA2_ERR_INVALID_ARG, "bad size");
  if (B == 0 || Q == 0) return CSA2_OK;
  if (csa2_status s = check_cache(cache, B)) return s;
  if (!q_ix || !w || !q_pos || !idx) return fail(CSA2_ERR_INVALID_ARG, "NULL input");
  if (k > 512) return fail(CSA2_ERR_UNSUPPORTED, "k > 512");
  if (!aligned16(q_ix)) return fail(CSA2_ERR_INVALID_ARG, "q_ix misaligned");
  if (B > 65535) return fail(CSA2_ERR_UNSUPPORTED, "more than 65535 sequences per call");
  csa2::launch_prefill_index(q_ix, w, B, Q, q_pos, k, max_entries, *cache, idx, err, stream);
  return launched("csa2_index_topk");
}

CSA2_EXPORT csa2_status csa2_topk(const float *scores, const int32_t *n_valid, int32_t R, int32_t N, int32_t k,
                                  int32_t *idx, float *val, int32_t k2, int32_t *idx2, float *val2,
                                  csa2_stream_t stream) {
  if (R < 0 || N < 0 || k < 1 || k2 < 0) return fail(CSA2_ERR_INVALID_ARG, "bad size");
  if (R == 0) return CSA2_OK;
  if (!scores || !idx) return fail(CSA2_ERR_INVALID_ARG, "NULL input");
  if (k2 > 0 && !idx2) return fail(CSA2_ERR_INVALID_ARG, "k2 > 0 needs idx2");
  if (int64_t(R) * 16 > INT32_MAX) return fail(CSA2_ERR_UNSUPPORTED, "too many rows");
  csa2::launch_topk_cluster(scores, n_valid, R, N, k, idx, val, k2, k2 > 0 ? idx2 : nullptr, val2, nullptr, stream);
  return launched("csa2_topk");
}

CSA2_EXPORT csa2_status csa2_sparse_attn(csa2_mode mode, const uint16_t *q, int32_t B, int32_t Q,
                                         const int32_t *q_pos, float softmax_scale, const uint16_t *q_ix,
                                         const uint16_t *w, int32_t k, int32_t pool_k, int32_t *pool_io,
                                         const int32_t *idx_in, int32_t *idx_out, int32_t max_entries,
                                         const csa2_cache *cache, const uint8_t *swa_codes, const float *swa_scale,
                                         int32_t R, int32_t window, const uint16_t *swa_new, float *o, float *lse,
                                         void *ws, size_t ws_bytes, int32_t *err, csa2_stream_t stream) {
  if (B < 0 || Q < 0 || k < 1 || pool_k < 0 || max_entries < 0) return fail(CSA2_ERR_INVALID_ARG, "bad size");
  if (B == 0 || Q == 0) return CSA2_OK;
  if (csa2_status s = check_cache(cache, B)) return s;
  if (!q || !q_pos || !o || !lse) return fail(CSA2_ERR_INVALID_ARG, "NULL input");
  if (k > 512 && mode != CSA2_MODE_DENSE) return fail(CSA2_ERR_UNSUPPORTED, "k > 512");
  if (!aligned16(q)) return fail(CSA2_ERR_INVALID_ARG, "q misaligned");
  if (swa_codes) {
    if (!swa_scale || window < 1 || window > 128 || R < window) return fail(CSA2_ERR_INVALID_ARG, "need 1 <= window <= 128, window <= R");
    if (!aligned16(swa_codes)) return fail(CSA2_ERR_INVALID_ARG, "swa_codes misaligned");
  }
  if (swa_new) {
    if (!swa_codes || Q != 1) return fail(CSA2_ERR_INVALID_ARG, "swa_new needs the window branch and Q == 1");
    if (reinterpret_cast<uintptr_t>(swa_new) & 7) return fail(CSA2_ERR_INVALID_ARG, "swa_new misaligned");
  }
  if (int64_t(B) * Q > 65535 * 16) return fail(CSA2_ERR_UNSUPPORTED, "too many query rows per call");
  const int rows = B * Q;
  const int32_t *idx = nullptr;
  if (mode == CSA2_MODE_DENSE) {
    // every visible entry, in segments of at most `seg` entries; the partials of the segments
    // after the first go through the workspace and are merged into o / lse in place
    const int seg = csa2::attn_dense_segment();
    if (max_entries > seg) {
      if (!ws || ws_bytes < csa2_workspace_size(mode, B, Q, max_entries, k, pool_k))
        return fail(CSA2_ERR_INVALID_ARG, "workspace too small");
    }
    float *po = static_cast<float *>(ws);
    float *pl = reinterpret_cast<float *>(static_cast<char *>(ws) + round256(size_t(rows) * CSA2_HEADS * CSA2_MAIN_DIM * 4));
    for (int s = 0, e0 = 0; s == 0 || e0 < max_entries; ++s, e0 += seg) {
      const int e1 = e0 + seg < max_entries ? e0 + seg : max_entries;
      csa2::launch_attn_mma(q, B, Q, q_pos, softmax_scale, nullptr, 0, true, e0, e1, max_entries, cache,
                            s == 0 ? swa_codes : nullptr, s == 0 && swa_codes ? swa_scale : nullptr, R, window,
                            s == 0 ? o : po, s == 0 ? lse : pl, err, stream, s == 0 ? swa_new : nullptr);
      if (s > 0) csa2::launch_merge(o, lse, po, pl, int64_t(rows) * CSA2_HEADS, CSA2_MAIN_DIM, o, lse, stream);
    }
    return launched("csa2_sparse_attn");
  }
  if (mode == CSA2_MODE_REUSE) {
    if (!idx_in) return fail(CSA2_ERR_INVALID_ARG, "REUSE needs idx_in");
    idx = idx_in;
  } else if (mode == CSA2_MODE_FULL || mode == CSA2_MODE_REINDEX) {
    if (!q_ix || !w) return fail(CSA2_ERR_INVALID_ARG, "FULL/REINDEX need q_ix and w");
    if (!aligned16(q_ix)) return fail(CSA2_ERR_INVALID_ARG, "q_ix misaligned");
    if (mode == CSA2_MODE_REINDEX && (!pool_io || pool_k < 1)) return fail(CSA2_ERR_INVALID_ARG, "REINDEX needs pool_io and pool_k");
    if (mode == CSA2_MODE_FULL && pool_k > 0 && !pool_io) return fail(CSA2_ERR_INVALID_ARG, "pool_k > 0 needs pool_io");
    const size_t need = csa2_workspace_size(mode, B, Q, max_entries, k, pool_k);
    if (!ws || ws_bytes < need) return fail(CSA2_ERR_INVALID_ARG, "workspace too small");
    if (mode == CSA2_MODE_FULL && fused_prefill(rows, pool_k)) {
      // a prefill chunk: fused indexer + causal top-k, no score matrix
      int32_t *sel = idx_out ? idx_out : static_cast<int32_t *>(ws);
      csa2::launch_prefill_index(q_ix, w, B, Q, q_pos, k, max_entries, *cache, sel, err, stream);
      csa2::launch_attn_mma(q, B, Q, q_pos, softmax_scale, sel, k, false, 0, 0, 0, cache, swa_codes,
                            swa_codes ? swa_scale : nullptr, R, window, o, lse, err, stream, swa_new);
      return launched("csa2_sparse_attn");
    }
    const int n_out = mode == CSA2_MODE_FULL ? max_entries : pool_k;
    if (rows > 65535) return fail(CSA2_ERR_UNSUPPORTED, "more than 65535 query rows per call");
    const bool fused_select = mode == CSA2_MODE_REINDEX && pool_k <= csa2::REINDEX_SELECT_MAX;
    float *scores = static_cast<float *>(ws);
    int32_t *sel = reinterpret_cast<int32_t *>(static_cast<char *>(ws) +
                                               (fused_select ? 0 : round256(size_t(rows) * n_out * 4)));
    if (idx_out) sel = idx_out;
    if (mode == CSA2_MODE_FULL) {
      csa2::launch_index_score_mma(q_ix, w, B, Q, q_pos, nullptr, 0, max_entries, *cache, scores, err, stream);
      csa2::launch_topk_cluster(scores, nullptr, rows, max_entries, k, sel, nullptr, pool_k,
                                pool_k > 0 ? pool_io : nullptr, nullptr, nullptr, stream);
    } else if (fused_select) {
      csa2::launch_reindex_select(q_ix, w, B, Q, q_pos, pool_io, pool_k, k, *cache, sel, err, stream);
    } else {
      csa2::launch_index_score_mma(q_ix, w, B, Q, q_pos, pool_io, pool_k, pool_k, *cache, scores, err, stream);
      csa2::launch_topk_cluster(scores, nullptr, rows, pool_k, k, sel, nullptr, 0, nullptr, nullptr, pool_io, stream);
    }
    idx = sel;
  } else {
    return fail(CSA2_ERR_INVALID_ARG, "bad mode");
  }
  // (a programmatic dependent launch after the selection measured no faster here: 0.390 against
  // 0.389 ms on the hier1m step, 62 against 53 us on one-query Full decode)
  csa2::launch_attn_mma(q, B, Q, q_pos, softmax_scale, idx, k, false, 0, 0, 0, cache, swa_codes,
                        swa_codes ? swa_scale : nullptr, R, window, o, lse, err, stream, swa_new);
  return launched("csa2_sparse_attn");
}

CSA2_EXPORT csa2_status csa2_swa_attn(const uint16_t *q, int32_t B, int32_t Q, const int32_t *q_pos,
                                      const uint8_t *swa_codes, const float *swa_scale, int32_t R, int32_t window,
                                      float softmax_scale, float *o, float *lse, int32_t *err, csa2_stream_t stream) {
  if (B < 0 || Q < 0 || window < 1 || R < window) return fail(CSA2_ERR_INVALID_ARG, "need 1 <= window <= R");
  if (B == 0 || Q == 0) return CSA2_OK;
  if (!q || !q_pos || !swa_codes || !swa_scale || !o || !lse) return fail(CSA2_ERR_INVALID_ARG, "NULL input");
  if (window > 128) return fail(CSA2_ERR_UNSUPPORTED, "window > 128");
  if (!aligned16(swa_codes) || !aligned16(q)) return fail(CSA2_ERR_INVALID_ARG, "swa_codes / q misaligned");
  if (int64_t(B) * Q > 65535 * 16) return fail(CSA2_ERR_UNSUPPORTED, "too many query rows per call");
  csa2::launch_attn_mma(q, B, Q, q_pos, softmax_scale, nullptr, 0, false, 0, 0, 0, nullptr, swa_codes, swa_scale, R,
                        window, o, lse, err, stream);
  return launched("csa2_swa_attn");
}

CSA2_EXPORT csa2_status csa2_merge(const float *o1, const float *l1, const float *o2, const float *l2, int64_t rows,
                                   int32_t D, float *o, float *lse, csa2_stream_t stream) {
  if (rows < 0 || D < 4 || (D & 3)) return fail(CSA2_ERR_INVALID_ARG, "D must be a positive multiple of 4");
  if (rows == 0) return CSA2_OK;
  if (!o1 || !l1 || !o2 || !l2 || !o || !lse) return fail(CSA2_ERR_INVALID_ARG, "NULL input");
  if (!aligned16(o1) || !aligned16(o2) || !aligned16(o)) return fail(CSA2_ERR_INVALID_ARG, "o misaligned");
  csa2::launch_merge(o1, l1, o2, l2, rows, D, o, lse, stream);
  return launched("csa2_merge");
}
