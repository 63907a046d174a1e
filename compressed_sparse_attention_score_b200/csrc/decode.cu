// The multi-layer decode driver: one token per sequence through a stack of CSA2 layers.
//
// A plan gives each layer its mode, the layer it takes indices or a pool from, and the global
// cache it reads.  csa2_decode_step runs the plan on one stream with no host synchronisation
// and no allocation, so a caller can capture it in a CUDA graph.  The layers run strictly in
// order, each with its own launches, as they would between the other blocks of a model:
//   - the first layer that reads a cache appends this step's token to it (once its group of
//     `ratio` tokens is complete);
//   - a Full layer scans its cache with the indexer and keeps its top-k (and the pool a
//     Reindex layer will search); a Reindex layer scans that pool; then top-k;
//   - every layer packs its own sliding-window token, then one attention launch computes the
//     sparse branch (its own entries, or for a Reuse layer the nearest selecting layer's), the
//     window branch and their merge.
// The pages' 40-layer plan comes from csa2_plan_v41 ("DeepSeek-V4.1 模型结构（0）", Q&A
// "DeepSeek-V4.1-Flash 的 40 层具体如何排布？"; "从V4到V4.1 Flash", 编码器层 and 解码器层).
#include <cuda_runtime.h>

#include <algorithm>
#include <string>

#include "../../include/csa2.h"
#include "kernels.cuh"

#define CSA2_EXPORT extern "C" __attribute__((visibility("default")))

namespace csa2 {
void set_last_error(const char *msg);  // api.cu
}

namespace {

csa2_status fail(csa2_status s, const std::string &msg) {
  csa2::set_last_error(msg.c_str());
  return s;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kV41Layers = 40;

// Checks the plan; returns the failing layer's message or "".
std::string check_plan(const csa2_decode_args &a) {
  for (int l = 0; l < a.n_layers; ++l) {
    const csa2_layer_plan &p = a.plan[l];
    const std::string at = "layer " + std::to_string(l) + ": ";
    if (p.mode == CSA2_LAYER_SWA) continue;
    if (p.mode < CSA2_MODE_FULL || p.mode > CSA2_MODE_DENSE) return at + "bad mode";
    if (p.cache < 0 || p.cache >= a.n_caches) return at + "cache id out of range";
    if (p.mode == CSA2_MODE_REUSE || p.mode == CSA2_MODE_REINDEX) {
      if (p.source < 0 || p.source >= l) return at + "source must be an earlier layer";
      const int sm = a.plan[p.source].mode;
      if (p.mode == CSA2_MODE_REINDEX && sm != CSA2_MODE_FULL) return at + "a Reindex source must be a Full layer";
      if (p.mode == CSA2_MODE_REUSE && sm != CSA2_MODE_FULL && sm != CSA2_MODE_REINDEX)
        return at + "a Reuse source must be a Full or Reindex layer";
      if (a.plan[p.source].cache != p.cache) return at + "source reads another cache";
    }
  }
  return "";
}

// Does some Reindex layer search the pool of Full layer l?
bool keeps_pool(const csa2_decode_args &a, int l) {
  for (int j = l + 1; j < a.n_layers; ++j)
    if (a.plan[j].mode == CSA2_MODE_REINDEX && a.plan[j].source == l) return true;
  return false;
}

size_t scores_bytes(const csa2_decode_args &a) {
  size_t n = 0;
  for (int l = 0; l < a.n_layers; ++l) {
    const int m = a.plan[l].mode;
    if (m == CSA2_MODE_FULL) n = std::max(n, size_t(a.max_entries[a.plan[l].cache]));
    if (m == CSA2_MODE_REINDEX && a.pool_k > csa2::REINDEX_SELECT_MAX) n = std::max(n, size_t(a.pool_k));
  }
  return round256(size_t(a.B) * n * 4);
}

}  // namespace

CSA2_EXPORT int32_t csa2_plan_v41(csa2_layer_plan *plan, int32_t max_layers, int32_t *cache_ratio) {
  if (!plan || max_layers < kV41Layers) return kV41Layers;
  // Full layers and the caches they write: the encoder's at ratio 2, the decoder's at ratio 1.
  const int full_layer[4] = {2, 8, 14, 20};
  const int ratio[4] = {2, 2, 2, 1};
  const int reindex_layer[4] = {24, 28, 32, 36};
  int src = -1, cache = -1;
  for (int l = 0; l < kV41Layers; ++l) {
    csa2_layer_plan p{CSA2_LAYER_SWA, -1, -1};
    bool head = false;
    for (int c = 0; c < 4; ++c)
      if (l == full_layer[c]) p = {CSA2_MODE_FULL, -1, c}, head = true, cache = c;
    for (int r = 0; r < 4; ++r)
      if (l == reindex_layer[r]) p = {CSA2_MODE_REINDEX, full_layer[3], 3}, head = true, cache = 3;
    if (head) {
      src = l;
    } else if (src >= 0) {
      p = {CSA2_MODE_REUSE, src, cache};  // the nearest earlier Full or Reindex layer
    }
    plan[l] = p;
  }
  if (cache_ratio)
    for (int c = 0; c < 4; ++c) cache_ratio[c] = ratio[c];
  return kV41Layers;
}

CSA2_EXPORT size_t csa2_decode_workspace_size(const csa2_decode_args *a) {
  if (!a || !a->plan || a->n_layers <= 0 || a->B <= 0 || !a->max_entries) return 0;
  return scores_bytes(*a);
}

CSA2_EXPORT csa2_status csa2_decode_step(const csa2_decode_args *a, void *ws, size_t ws_bytes, int32_t *err,
                                         csa2_stream_t stream) {
  if (!a) return fail(CSA2_ERR_INVALID_ARG, "args is NULL");
  if (a->n_layers < 0 || a->B < 0 || a->n_caches < 0) return fail(CSA2_ERR_INVALID_ARG, "negative size");
  if (a->n_layers == 0 || a->B == 0) return CSA2_OK;
  if (!a->plan || !a->pos || !a->q || !a->o || !a->lse || !a->idx) return fail(CSA2_ERR_INVALID_ARG, "NULL input");
  if (a->n_caches > 0 && (!a->caches || !a->max_entries)) return fail(CSA2_ERR_INVALID_ARG, "NULL caches");
  if (a->k < 1 || a->k > 512 || a->pool_k < 0) return fail(CSA2_ERR_INVALID_ARG, "need 1 <= k <= 512");
  if (!a->swa_x || !a->swa_codes || !a->swa_scale || a->window < 1 || a->window > 128 || a->R < a->window)
    return fail(CSA2_ERR_INVALID_ARG, "every layer needs its SWA ring (1 <= window <= 128 <= R)");
  if (a->B > 65535) return fail(CSA2_ERR_UNSUPPORTED, "too many sequences per step");
  const std::string bad = check_plan(*a);
  if (!bad.empty()) return fail(CSA2_ERR_INVALID_ARG, bad);
  bool need_ix = false, need_pool = false;
  for (int l = 0; l < a->n_layers; ++l) {
    const int m = a->plan[l].mode;
    need_ix |= m == CSA2_MODE_FULL || m == CSA2_MODE_REINDEX;
    need_pool |= m == CSA2_MODE_REINDEX;
    if (m == CSA2_MODE_DENSE && a->max_entries[a->plan[l].cache] > csa2::attn_dense_segment())
      return fail(CSA2_ERR_UNSUPPORTED, "a Dense layer of the decode driver holds one segment of entries");
  }
  if (need_ix && (!a->q_ix || !a->w)) return fail(CSA2_ERR_INVALID_ARG, "Full/Reindex layers need q_ix and w");
  if (need_pool && (!a->pool || a->pool_k < a->k)) return fail(CSA2_ERR_INVALID_ARG, "Reindex needs pool, pool_k >= k");
  const size_t need_ws = scores_bytes(*a);
  if (need_ws > 0 && (!ws || ws_bytes < need_ws)) return fail(CSA2_ERR_INVALID_ARG, "workspace too small");
  int rmax = 1;
  for (int c = 0; c < a->n_caches; ++c) rmax = std::max(rmax, int(a->caches[c].ratio));
  if (a->new_kv && (!a->new_ix || (rmax > 1 && !a->kv_stage)))
    return fail(CSA2_ERR_INVALID_ARG, "new_kv needs new_ix and (ratio > 1) kv_stage");

  const int B = a->B, L = a->n_layers;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t qrow = size_t(CSA2_HEADS) * CSA2_MAIN_DIM, ixrow = size_t(CSA2_IX_HEADS) * CSA2_IX_DIM;
  float *scores = static_cast<float *>(ws);
  bool appended[64] = {};
  if (a->n_caches > 64) return fail(CSA2_ERR_UNSUPPORTED, "more than 64 caches");

  bool launched_any = false;  // has this call launched a kernel yet
  for (int l = 0; l < L; ++l) {
    const csa2_layer_plan &p = a->plan[l];
    const int c = p.cache;
    // this step's token joins the cache before the first layer that reads it
    if (c >= 0 && a->new_kv && !appended[c]) {
      const csa2_cache &cc = a->caches[c];
      csa2::launch_append_kv(a->new_kv + size_t(c) * B * CSA2_MAIN_DIM, a->new_ix + size_t(c) * B * CSA2_IX_DIM,
                             CSA2_BF16, B, a->pos, a->kv_stage ? a->kv_stage + size_t(c) * B * rmax * 640 : nullptr,
                             int64_t(rmax) * 640, cc, const_cast<int32_t *>(cc.num_entries), err, st);
      appended[c] = true;
      launched_any = true;
    }
    int32_t *idx_l = a->idx + size_t(l) * B * a->k;
    const int32_t *idx = nullptr;
    if (p.mode == CSA2_MODE_FULL || p.mode == CSA2_MODE_REINDEX) {
      const csa2_cache &cc = a->caches[c];
      const uint16_t *qix = a->q_ix + size_t(l) * B * ixrow;
      const uint16_t *w = a->w + size_t(l) * B * CSA2_IX_HEADS;
      int32_t *pool_c = a->pool ? a->pool + size_t(c) * B * a->pool_k : nullptr;
      if (p.mode == CSA2_MODE_FULL) {
        const int me = a->max_entries[c];
        const bool pool = keeps_pool(*a, l);
        csa2::launch_index_score_mma(qix, w, B, 1, a->pos, nullptr, 0, me, cc, scores, err, st);
        csa2::launch_topk_cluster(scores, nullptr, B, me, a->k, idx_l, nullptr, pool ? a->pool_k : 0,
                                  pool ? pool_c : nullptr, nullptr, nullptr, st);
      } else if (a->pool_k <= csa2::REINDEX_SELECT_MAX) {
        csa2::launch_reindex_select(qix, w, B, 1, a->pos, pool_c, a->pool_k, a->k, cc, idx_l, err, st);
      } else {
        csa2::launch_index_score_mma(qix, w, B, 1, a->pos, pool_c, a->pool_k, a->pool_k, cc, scores, err, st);
        csa2::launch_topk_cluster(scores, nullptr, B, a->pool_k, a->k, idx_l, nullptr, 0, nullptr, nullptr, pool_c,
                                  st);
      }
      idx = idx_l;
      launched_any = true;
    } else if (p.mode == CSA2_MODE_REUSE) {
      idx = a->idx + size_t(p.source) * B * a->k;
    }
    // one launch: the layer's own window token quantised into its ring, then its attention
    // (sparse or dense branch + window + merge)
    uint8_t *codes_l = a->swa_codes + size_t(l) * B * a->R * CSA2_SWA_DIM;
    float *scale_l = a->swa_scale + size_t(l) * B * a->R;
    const csa2_cache *cc = c >= 0 ? &a->caches[c] : nullptr;
    const int me = c >= 0 ? a->max_entries[c] : 0;
    // every attention launch but the call's first starts early and waits on the device for the
    // launch before it (everything else it reads was written before this call): 1.269 against
    // 1.295 ms on the 40-layer step
    csa2::launch_attn_mma(a->q + size_t(l) * B * qrow, B, 1, a->pos, a->softmax_scale, idx, a->k,
                          p.mode == CSA2_MODE_DENSE, 0, me, me, cc, codes_l, scale_l, a->R, a->window,
                          a->o + size_t(l) * B * qrow, a->lse + size_t(l) * B * CSA2_HEADS, err, st,
                          a->swa_x + size_t(l) * B * CSA2_SWA_DIM, launched_any);
    launched_any = true;
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(CSA2_ERR_CUDA, std::string("csa2_decode_step: ") + cudaGetErrorString(e));
  csa2::set_last_error("");
  return CSA2_OK;
}

CSA2_EXPORT csa2_status csa2_append_kv(const void *lat_kv, const void *lat_ix, csa2_dtype dtype, int32_t B,
                                       const int32_t *pos, float *stage, const csa2_cache *cache, int32_t *err,
                                       csa2_stream_t stream) {
  if (B < 0) return fail(CSA2_ERR_INVALID_ARG, "negative size");
  if (B == 0) return CSA2_OK;
  if (!cache || !lat_kv || !lat_ix || !pos || !cache->num_entries) return fail(CSA2_ERR_INVALID_ARG, "NULL input");
  if (dtype != CSA2_F32 && dtype != CSA2_BF16) return fail(CSA2_ERR_INVALID_ARG, "bad dtype");
  if (cache->ratio < 1 || B > cache->batch) return fail(CSA2_ERR_SHAPE, "bad ratio or B exceeds cache batch");
  if (cache->ratio > 1 && !stage) return fail(CSA2_ERR_INVALID_ARG, "ratio > 1 needs a staging buffer");
  if ((reinterpret_cast<uintptr_t>(lat_kv) & 15) || (reinterpret_cast<uintptr_t>(lat_ix) & 7) ||
      (reinterpret_cast<uintptr_t>(stage) & 15))
    return fail(CSA2_ERR_INVALID_ARG, "latents or stage misaligned");
  csa2::launch_append_kv(lat_kv, lat_ix, dtype, B, pos, stage, int64_t(cache->ratio) * 640, *cache,
                         const_cast<int32_t *>(cache->num_entries), err, reinterpret_cast<cudaStream_t>(stream));
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(CSA2_ERR_CUDA, std::string("csa2_append_kv: ") + cudaGetErrorString(e));
  return CSA2_OK;
}
