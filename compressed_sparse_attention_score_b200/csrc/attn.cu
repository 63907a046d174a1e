// K6/K7 (scalar form): attention of 64 query heads over a gathered key set in
// which each 512-d key also serves as the value, on CUDA cores.
//
// One CTA per (query row, group of 8 heads).  Keys are dequantised into shared
// memory 32 at a time; the CTA keeps an online softmax per head and the output
// accumulators in registers (thread = head h, dims d = lane + 32 i).
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

constexpr int AT_HEADS = 8;     // heads per CTA
constexpr int AT_KEYS = 32;     // keys per chunk
constexpr int AT_STRIDE = D + 1;  // padded smem row (conflict-free column reads)

// Key source: the main-KV entries listed in an index row (sparse branch).
struct SparseKeys {
  const int32_t *idx;  // [rows][k]
  int k;
  csa2_cache c;
  int32_t *err;
  int b, nvis;
  const int32_t *list;
  __device__ void setup(int row, int Q, const int32_t *q_pos) {
    b = row / Q;
    nvis = visible_entries(c, b, q_pos[row]);
    list = idx + int64_t(row) * k;
  }
  __device__ int count() const { return k; }
  // Dequantise key j of this row into dst[0..511] (each of the 8 threads of a
  // key writes 64 values); returns false for a pad or a rejected index.
  __device__ bool load(int j, int part, float *dst) {
    const int n = list[j];
    if (n == -1) return false;
    if (n < -1 || n >= nvis) {
      if (part == 0) report(err, CSA2_ERR_INDEX);
      return false;
    }
    const int64_t slot = cache_slot(c, b, n);
    if (slot < 0) {
      if (part == 0) report(err, CSA2_ERR_INDEX);
      return false;
    }
    const uint4 *cp = reinterpret_cast<const uint4 *>(c.kv_codes + slot * CSA2_MAIN_CODE_BYTES) + 2 * part;
    const uint32_t sc = *reinterpret_cast<const uint32_t *>(c.kv_scales + slot * CSA2_MAIN_SCALE_BYTES + 4 * part);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 cw = cp[h];
      const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int e = 32 * h + i;  // element within this part's 64
        const float s = e4m3_value((sc >> (8 * (e >> 4))) & 255);
        dst[64 * part + e] = e2m1_value((w[i >> 3] >> (4 * (i & 7))) & 15) * s;
      }
    }
    return true;
  }
};

// Key source: the sliding window of one query in a per-layer FP8 ring.
struct WindowKeys {
  const uint8_t *codes;  // [B][R][512]
  const float *scale;    // [B][R]
  int R, window;
  int32_t *err;
  int b, lo, n;
  __device__ void setup(int row, int Q, const int32_t *q_pos) {
    b = row / Q;
    const int p = q_pos[row];
    lo = max(0, p - window + 1);
    n = p < 0 ? 0 : p - lo + 1;
  }
  __device__ int count() const { return n; }
  __device__ bool load(int j, int part, float *dst) {
    if (j >= n) return false;
    const int64_t slot = int64_t(b) * R + (lo + j) % R;
    const float s = scale[slot];
    const uint4 *cp = reinterpret_cast<const uint4 *>(codes + slot * CSA2_SWA_DIM + 64 * part);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const uint4 cw = cp[h];
      const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
      for (int i = 0; i < 16; ++i) dst[64 * part + 16 * h + i] = __fmul_rn(e4m3_value((w[i >> 2] >> (8 * (i & 3))) & 255), s);
    }
    return true;
  }
};

template <class Keys>
__global__ void __launch_bounds__(256) attn_scalar_kernel(Keys keys, const uint16_t *__restrict__ q, int Q,
                                                          const int32_t *__restrict__ q_pos, float tau,
                                                          float *__restrict__ o, float *__restrict__ lse) {
  extern __shared__ float sm[];
  float *kv = sm;                                // [AT_KEYS][AT_STRIDE]
  float *qs = kv + AT_KEYS * AT_STRIDE;          // [AT_HEADS][AT_STRIDE]
  float *pl = qs + AT_HEADS * AT_STRIDE;         // [AT_HEADS][AT_KEYS]
  __shared__ int ok_s[AT_KEYS];
  const int row = blockIdx.x, hg = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;  // warp = head within group
  keys.setup(row, Q, q_pos);
  const uint16_t *qrow = q + (int64_t(row) * H + hg * AT_HEADS) * D;
  for (int i = tid; i < AT_HEADS * D; i += 256) qs[(i / D) * AT_STRIDE + i % D] = tau * bf16_to_f32(qrow[i]);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  float m = -INFINITY, l = 0.f;  // this warp's head
  const int nk = keys.count();
  for (int j0 = 0; j0 < nk; j0 += AT_KEYS) {
    __syncthreads();
    {  // dequantise up to 32 keys: thread -> (key tid/8, part tid%8)
      const int j = j0 + tid / 8, part = tid % 8;
      const bool ok = j < nk && keys.load(j, part, kv + (tid / 8) * AT_STRIDE);
      if (part == 0) ok_s[tid / 8] = ok;
    }
    __syncthreads();
    // logits of head `warp` against the 32 keys: lane = key
    float lg = -INFINITY;
    if (ok_s[lane]) {
      const float *kr = kv + lane * AT_STRIDE;
      const float *qr = qs + warp * AT_STRIDE;
      float a = 0.f;
      for (int d = 0; d < D; ++d) a = fmaf(qr[d], kr[d], a);
      lg = a;
    }
    float cm = lg;
#pragma unroll
    for (int off = 16; off; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
    const float mn = fmaxf(m, cm);
    float p = 0.f, alpha = 1.f;
    if (mn != -INFINITY) {
      p = lg == -INFINITY ? 0.f : __expf(lg - mn);
      alpha = m == -INFINITY ? 0.f : __expf(m - mn);
    }
    float ps = p;
#pragma unroll
    for (int off = 16; off; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l = l * alpha + ps;
    m = mn;
    pl[warp * AT_KEYS + lane] = p;
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] *= alpha;
    for (int jj = 0; jj < AT_KEYS; ++jj) {
      const float pj = pl[warp * AT_KEYS + jj];
      if (pj != 0.f) {
        const float *kr = kv + jj * AT_STRIDE + lane;
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = fmaf(pj, kr[32 * i], acc[i]);
      }
    }
  }
  const int h = hg * AT_HEADS + warp;
  float *orow = o + (int64_t(row) * H + h) * D;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) orow[lane + 32 * i] = acc[i] * inv;
  if (lane == 0) lse[int64_t(row) * H + h] = l > 0.f ? m + logf(l) : -INFINITY;
}

static size_t attn_smem() { return sizeof(float) * (AT_KEYS * AT_STRIDE + AT_HEADS * AT_STRIDE + AT_HEADS * AT_KEYS); }

void launch_sparse_attn_scalar(const uint16_t *q, int B, int Q, const int32_t *q_pos, float tau,
                               const int32_t *idx, int k, const csa2_cache &c, float *o, float *lse,
                               int32_t *err, cudaStream_t st) {
  if (B * Q == 0) return;
  SparseKeys keys{idx, k, c, err};
  set_smem_limit(attn_scalar_kernel<SparseKeys>, attn_smem());
  attn_scalar_kernel<SparseKeys><<<dim3(B * Q, H / AT_HEADS), 256, attn_smem(), st>>>(keys, q, Q, q_pos, tau, o, lse);
}

void launch_swa_attn_scalar(const uint16_t *q, int B, int Q, const int32_t *q_pos, const uint8_t *codes,
                            const float *scale, int R, int window, float tau, float *o, float *lse,
                            int32_t *err, cudaStream_t st) {
  if (B * Q == 0) return;
  WindowKeys keys{codes, scale, R, window, err};
  set_smem_limit(attn_scalar_kernel<WindowKeys>, attn_smem());
  attn_scalar_kernel<WindowKeys><<<dim3(B * Q, H / AT_HEADS), 256, attn_smem(), st>>>(keys, q, Q, q_pos, tau, o, lse);
}

}  // namespace csa2
