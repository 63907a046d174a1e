// Host-side launchers of the CSA2 kernels (internal to the library).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

// Raise a kernel's dynamic shared-memory limit once per device.
template <typename F>
inline void set_smem_limit(F *func, size_t bytes) {
  static bool done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || done[dev]) return;
  cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
  done[dev] = true;
}

// Streaming multiprocessors of the current device (queried once per device).
inline int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;
    }
    cached[dev] = n;
  }
  return cached[dev];
}

void launch_pack_kv(const void *lat_kv, const void *lat_ix, csa2_dtype dtype, const float *pool_w,
                    const float *gate_kv, const float *gate_ix, int B, int T, const int32_t *first_entry,
                    const csa2_cache &c, int32_t *err, cudaStream_t st);
void launch_pack_swa(const void *x, csa2_dtype dtype, int B, int T, const int32_t *pos, int pos_rows,
                     uint8_t *codes, float *scale, int R, int32_t *err, cudaStream_t st);
// stage_stride: floats from one sequence's staging rows to the next (at least ratio * 640).
void launch_append_kv(const void *lat_kv, const void *lat_ix, csa2_dtype dtype, int B, const int32_t *pos,
                      float *stage, int64_t stage_stride, const csa2_cache &c, int32_t *num_entries, int32_t *err,
                      cudaStream_t st);
void launch_index_score_mma(const uint16_t *q_ix, const uint16_t *w, int B, int Q, const int32_t *q_pos,
                            const int32_t *cand, int P, int n_out, const csa2_cache &c, float *scores, int32_t *err,
                            cudaStream_t st);
// Fused Reindex selection: scores of a candidate list of P <= REINDEX_SELECT_MAX entries and
// their top-k (k <= 512) in one launch, sel [B*Q][k] = the chosen candidates' entries in
// candidate order (ascending for an ascending list), -1 padded -- what launch_index_score_mma
// followed by launch_topk_cluster with the list as map returns.
constexpr int REINDEX_SELECT_MAX = 16384;
void launch_reindex_select(const uint16_t *q_ix, const uint16_t *w, int B, int Q, const int32_t *q_pos,
                           const int32_t *cand, int P, int k, const csa2_cache &c, int32_t *sel, int32_t *err,
                           cudaStream_t st);
// Tensor map of a cache's indexer codes as 128-entry groups (false: the layout does not allow one).
bool make_index_code_map(CUtensorMap *m, const csa2_cache &c);
// Fused prefill indexer + causal top-k (k <= 512): idx [B][Q][k], ascending, -1 padded.
// Entries beyond max_entries are left out and set CSA2_ERR_SHAPE (as the unfused Full path).
void launch_prefill_index(const uint16_t *q_ix, const uint16_t *w, int B, int Q, const int32_t *q_pos, int k,
                          int max_entries, const csa2_cache &c, int32_t *idx, int32_t *err, cudaStream_t st);
void launch_topk_cluster(const float *scores, const int32_t *n_valid, int R, int N, int k0, int32_t *idx0, float *val0,
                         int k1, int32_t *idx1, float *val1, const int32_t *map, cudaStream_t st);
// swa_new [B*Q][512] bf16 (decode): each row's own window token, quantised inside the launch,
// used as the window's last key and stored in the ring (codes / scale must then be writable).
// pdl: launched as a programmatic dependent of the kernel before it in the stream (only when that
// kernel belongs to the same library call, so everything else it reads was written before).
void launch_attn_mma(const uint16_t *q, int B, int Q, const int32_t *q_pos, float tau, const int32_t *idx, int k,
                     bool dense, int e0, int e1, int n_bound, const csa2_cache *c, const uint8_t *codes,
                     const float *scale, int R, int window, float *o, float *lse, int32_t *err, cudaStream_t st,
                     const uint16_t *swa_new = nullptr, bool pdl = false);
// Entries per dense-attention launch (one cluster of at most 16 CTAs x 640 keys per row).
int attn_dense_segment();
void launch_merge(const float *o1, const float *l1, const float *o2, const float *l2, int64_t rows, int D_,
                  float *o, float *lse, cudaStream_t st);

}  // namespace csa2
