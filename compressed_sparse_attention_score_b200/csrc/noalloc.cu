// csa2_sparse_attn_noalloc: csa2_sparse_attn for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain a workspace: an engine whose memory pool
// has reserved the whole device (so cudaMalloc fails), or a serving loop that
// forbids allocation on its hot path because cudaMalloc/cudaFree synchronise
// the device.  This entry point takes the same arguments as csa2_sparse_attn
// minus the workspace and uses a fixed scratch array that lives in the library
// itself (file-scope __device__ storage, so every GPU that loads the library
// holds CSA2_NOALLOC_SCRATCH_BYTES of it until the process exits).
#include <cuda_runtime.h>

#include <cstdio>

#include "../../include/csa2.h"

#define CSA2_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

constexpr size_t kScratchBytes = CSA2_NOALLOC_SCRATCH_BYTES;

// The shared scratch.  In host code this name is only a stand-in for the
// device symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the scratch on the current device.  Looked up on every call (cheap once
// the module is loaded) rather than cached, so that it stays right after the device's primary
// context has been reset and the module reloaded.
cudaError_t scratch_address(void **out) {
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace

namespace csa2 {
void set_last_error(const char *msg);  // api.cu
}

CSA2_EXPORT size_t csa2_noalloc_scratch_bytes(void) { return kScratchBytes; }

CSA2_EXPORT csa2_status csa2_sparse_attn_noalloc(csa2_mode mode, const uint16_t *q, int32_t B, int32_t Q,
                                                 const int32_t *q_pos, float softmax_scale, const uint16_t *q_ix,
                                                 const uint16_t *w, int32_t k, int32_t pool_k, int32_t *pool_io,
                                                 const int32_t *idx_in, int32_t *idx_out, int32_t max_entries,
                                                 const csa2_cache *cache, const uint8_t *swa_codes,
                                                 const float *swa_scale, int32_t R, int32_t window, float *o,
                                                 float *lse, int32_t *err, csa2_stream_t stream) {
  const size_t need = csa2_workspace_size(mode, B, Q, max_entries, k, pool_k);
  if (need > kScratchBytes) {
    char msg[160];
    std::snprintf(msg, sizeof(msg),
                  "csa2_sparse_attn_noalloc: these sizes need %zu bytes of scratch, the static scratch holds %zu",
                  need, kScratchBytes);
    csa2::set_last_error(msg);
    return CSA2_ERR_UNSUPPORTED;
  }
  void *ws = nullptr;
  if (need > 0) {
    const cudaError_t e = scratch_address(&ws);
    if (e != cudaSuccess) {
      char msg[160];
      std::snprintf(msg, sizeof(msg), "csa2_sparse_attn_noalloc: scratch address: %s", cudaGetErrorString(e));
      csa2::set_last_error(msg);
      return CSA2_ERR_CUDA;
    }
  }
  return csa2_sparse_attn(mode, q, B, Q, q_pos, softmax_scale, q_ix, w, k, pool_k, pool_io, idx_in, idx_out,
                          max_entries, cache, swa_codes, swa_scale, R, window, nullptr, o, lse, ws,
                          need > 0 ? kScratchBytes : 0,
                          err, stream);
}
