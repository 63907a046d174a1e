// K3 (scalar form): lightning-indexer scores on CUDA cores.
//
// s_n = sum_h w_h * relu(q^_h . k^_n), q^ the per-32 E8M0/e2m1 quantisation of
// the query heads.  One CTA per (query row, tile of 128 keys); each thread owns
// one key and accumulates the 64 head dot products in registers while the
// quantised query sits in shared memory (broadcast reads).
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

// Quantise the 64 indexer-query heads of one row to MXFP4 values in smem.
// Each warp takes heads; lane l holds values [4l, 4l+4), eight lanes per block.
__device__ void quantise_query_heads(const uint16_t *__restrict__ q, float *qh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int h = warp; h < HI; h += nw) {
    float v[4];
    uint2 a = *reinterpret_cast<const uint2 *>(q + h * DI + 4 * lane);
    v[0] = __uint_as_float(a.x << 16), v[1] = __uint_as_float(a.x & 0xFFFF0000u);
    v[2] = __uint_as_float(a.y << 16), v[3] = __uint_as_float(a.y & 0xFFFF0000u);
    float am = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    float out[4] = {0.f, 0.f, 0.f, 0.f};
    if (am != 0.f) {
      const float s = pow2f(e8m0_ceil_exponent(__fdiv_rn(am, 6.0f)));
#pragma unroll
      for (int i = 0; i < 4; ++i) out[i] = e2m1_value(e2m1_code(__fdiv_rn(v[i], s))) * s;
    }
    *reinterpret_cast<float4 *>(qh + h * DI + 4 * lane) = make_float4(out[0], out[1], out[2], out[3]);
  }
}

__global__ void __launch_bounds__(128) index_score_scalar_kernel(
    const uint16_t *__restrict__ q_ix, const uint16_t *__restrict__ w, int Q,
    const int32_t *__restrict__ q_pos, const int32_t *__restrict__ cand, int P, int n_out,
    csa2_cache c, float *__restrict__ scores, int32_t *err) {
  __shared__ __align__(16) float qh[HI * DI];
  __shared__ float ws[HI];
  const int row = blockIdx.x;
  const int b = row / Q;
  quantise_query_heads(q_ix + int64_t(row) * HI * DI, qh);
  if (threadIdx.x < HI) ws[threadIdx.x] = bf16_to_f32(w[int64_t(row) * HI + threadIdx.x]);
  __syncthreads();

  const int j = blockIdx.y * blockDim.x + threadIdx.x;
  if (j >= n_out) return;
  const int nvis = visible_entries(c, b, q_pos[row]);
  int64_t n = j;
  if (cand) {
    n = cand[int64_t(row) * P + j];
    if (n < -1 || n >= c.num_entries[b]) report(err, CSA2_ERR_INDEX);
  }
  float result = -INFINITY;
  const int64_t slot = (n >= 0 && n < nvis) ? cache_slot(c, b, n) : -1;
  if (n >= 0 && n < nvis && slot < 0) report(err, CSA2_ERR_INDEX);
  if (slot >= 0) {
    const uint4 *kc = reinterpret_cast<const uint4 *>(c.ix_codes + slot * CSA2_IX_CODE_BYTES);
    const uint32_t ksc = *reinterpret_cast<const uint32_t *>(c.ix_scales + slot * CSA2_IX_SCALE_BYTES);
    float acc[HI];
#pragma unroll
    for (int h = 0; h < HI; ++h) acc[h] = 0.f;
#pragma unroll 1
    for (int g = 0; g < 4; ++g) {            // one E8M0 block of 32 values
      const uint4 cw = kc[g];
      const float s = pow2f(int((ksc >> (8 * g)) & 255) - 127);
      float k[32];
      const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
      for (int i = 0; i < 32; ++i) k[i] = e2m1_value((words[i >> 3] >> (4 * (i & 7))) & 15) * s;
#pragma unroll
      for (int h = 0; h < HI; ++h) {
        const float4 *qp = reinterpret_cast<const float4 *>(qh + h * DI + 32 * g);
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 qv = qp[i];
          a = fmaf(qv.x, k[4 * i], a);
          a = fmaf(qv.y, k[4 * i + 1], a);
          a = fmaf(qv.z, k[4 * i + 2], a);
          a = fmaf(qv.w, k[4 * i + 3], a);
        }
        acc[h] += a;
      }
    }
    float sc = 0.f;
#pragma unroll
    for (int h = 0; h < HI; ++h) sc = fmaf(ws[h], fmaxf(acc[h], 0.f), sc);
    result = sc;
  }
  scores[int64_t(row) * n_out + j] = result;
}

void launch_index_score_scalar(const uint16_t *q_ix, const uint16_t *w, int B, int Q,
                               const int32_t *q_pos, const int32_t *cand, int P, int n_out,
                               const csa2_cache &c, float *scores, int32_t *err, cudaStream_t st) {
  if (n_out == 0 || B * Q == 0) return;
  dim3 grid(B * Q, (n_out + 127) / 128);
  index_score_scalar_kernel<<<grid, 128, 0, st>>>(q_ix, w, Q, q_pos, cand, P, n_out, c, scores, err);
}

}  // namespace csa2
