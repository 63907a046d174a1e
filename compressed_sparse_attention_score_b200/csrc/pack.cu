// K1/K2: the compressor + packer of global KV entries and the SWA packer.
//
// Both are HBM streaming kernels: one warp per output entry (or SWA token),
// 16-byte vector loads, quantisation in registers, coalesced row stores.
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

template <typename T>
__device__ __forceinline__ void load16(const T *p, float (&v)[16]);

template <>
__device__ __forceinline__ void load16<float>(const float *p, float (&v)[16]) {
  const float4 *q = reinterpret_cast<const float4 *>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float4 a = q[i];
    v[4 * i] = a.x, v[4 * i + 1] = a.y, v[4 * i + 2] = a.z, v[4 * i + 3] = a.w;
  }
}

template <>
__device__ __forceinline__ void load16<uint16_t>(const uint16_t *p, float (&v)[16]) {
  const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    uint4 a = q[i];
    uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
      v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
}

template <typename T>
__device__ __forceinline__ void load4(const T *p, float (&v)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float *p, float (&v)[4]) {
  float4 a = *reinterpret_cast<const float4 *>(p);
  v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w;
}
template <>
__device__ __forceinline__ void load4<uint16_t>(const uint16_t *p, float (&v)[4]) {
  uint2 a = *reinterpret_cast<const uint2 *>(p);
  v[0] = __uint_as_float(a.x << 16), v[1] = __uint_as_float(a.x & 0xFFFF0000u);
  v[2] = __uint_as_float(a.y << 16), v[3] = __uint_as_float(a.y & 0xFFFF0000u);
}

// One warp per new entry.  Lane l owns main values [16l, 16l+16) (one E4M3 block)
// and indexer values [4l, 4l+4) (eight lanes per E8M0 block).
template <typename T>
__global__ void __launch_bounds__(256) pack_kv_kernel(const T *__restrict__ lat_kv,
                                                      const T *__restrict__ lat_ix,
                                                      const float *__restrict__ pool_w, int B, int T_,
                                                      const int32_t *__restrict__ first_entry,
                                                      csa2_cache c, int32_t *err) {
  const int lane = threadIdx.x & 31;
  const int n_new = T_ / c.ratio;
  const int64_t e = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (e >= int64_t(B) * n_new) return;
  const int b = int(e / n_new), j = int(e % n_new);
  const int64_t slot = cache_slot(c, b, int64_t(first_entry[b]) + j);
  if (slot < 0) {
    if (lane == 0) report(err, CSA2_ERR_INDEX);
    return;
  }
  const float w_default = __fdiv_rn(1.0f, float(c.ratio));

  // ---- pool the tokens of this entry (fp32, left to right, no fused multiply-add)
  float x[16], xi[4];
  for (int t = 0; t < c.ratio; ++t) {
    const int64_t tok = int64_t(b) * T_ + int64_t(j) * c.ratio + t;
    const float wt = pool_w ? pool_w[tok] : w_default;
    float v[16], vi[4];
    load16<T>(lat_kv + tok * D + 16 * lane, v);
    load4<T>(lat_ix + tok * DI + 4 * lane, vi);
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = t == 0 ? __fmul_rn(wt, v[i]) : __fadd_rn(x[i], __fmul_rn(wt, v[i]));
#pragma unroll
    for (int i = 0; i < 4; ++i) xi[i] = t == 0 ? __fmul_rn(wt, vi[i]) : __fadd_rn(xi[i], __fmul_rn(wt, vi[i]));
  }

  // ---- main KV: E4M3 scale per 16 values, e2m1 codes
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  const uint32_t sc = e4m3_code(__fdiv_rn(amax, 6.0f));
  const float s = e4m3_value(sc);
  uint32_t lo = 0, hi = 0;
  if (s != 0.f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) lo |= e2m1_code(__fdiv_rn(x[i], s)) << (4 * i);
#pragma unroll
    for (int i = 0; i < 8; ++i) hi |= e2m1_code(__fdiv_rn(x[8 + i], s)) << (4 * i);
  }
  reinterpret_cast<uint2 *>(c.kv_codes + slot * CSA2_MAIN_CODE_BYTES)[lane] = make_uint2(lo, hi);
  c.kv_scales[slot * CSA2_MAIN_SCALE_BYTES + lane] = uint8_t(sc);

  // ---- indexer key: E8M0 exponent per 32 values (8 lanes), e2m1 codes
  float am = fmaxf(fmaxf(fabsf(xi[0]), fabsf(xi[1])), fmaxf(fabsf(xi[2]), fabsf(xi[3])));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  uint32_t code4 = 0;
  int ex = -127;
  if (am != 0.f) {
    ex = e8m0_ceil_exponent(__fdiv_rn(am, 6.0f));
    const float si = pow2f(ex);
#pragma unroll
    for (int i = 0; i < 4; ++i) code4 |= e2m1_code(__fdiv_rn(xi[i], si)) << (4 * i);
  }
  reinterpret_cast<uint16_t *>(c.ix_codes + slot * CSA2_IX_CODE_BYTES)[lane] = uint16_t(code4);
  if ((lane & 7) == 0) c.ix_scales[slot * CSA2_IX_SCALE_BYTES + (lane >> 3)] = uint8_t(ex + 127);
}

// One warp per SWA token; lane l owns values [16l, 16l+16).  Only the last R
// tokens of a call are stored (earlier ones would be overwritten in the ring).
template <typename T>
__global__ void __launch_bounds__(256) pack_swa_kernel(const T *__restrict__ x, int B, int T_,
                                                       const int32_t *__restrict__ pos,
                                                       uint8_t *__restrict__ codes,
                                                       float *__restrict__ scale, int R,
                                                       int32_t *err) {
  const int lane = threadIdx.x & 31;
  const int64_t e = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (e >= int64_t(B) * T_) return;
  const int b = int(e / T_), t = int(e % T_);
  if (t < T_ - R) return;
  const int p = pos[e];
  if (p < 0) return;  // padding token of a ragged batch
  const int64_t slot = int64_t(b) * R + (p % R);
  float v[16];
  load16<T>(x + e * D + 16 * lane, v);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __fdiv_rn(amax, 448.0f);
  uint32_t w[4] = {0, 0, 0, 0};
  if (s != 0.f) {
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i >> 2] |= e4m3_code(__fdiv_rn(v[i], s)) << (8 * (i & 3));
  }
  reinterpret_cast<uint4 *>(codes + slot * CSA2_SWA_DIM)[lane] = make_uint4(w[0], w[1], w[2], w[3]);
  if (lane == 0) scale[slot] = s;
}

void launch_pack_kv(const void *lat_kv, const void *lat_ix, csa2_dtype dtype, const float *pool_w,
                    int B, int T, const int32_t *first_entry, const csa2_cache &c, int32_t *err,
                    cudaStream_t st) {
  const int64_t n = int64_t(B) * (T / c.ratio);
  if (n == 0) return;
  const int grid = int((n + 7) / 8);
  if (dtype == CSA2_F32)
    pack_kv_kernel<float><<<grid, 256, 0, st>>>((const float *)lat_kv, (const float *)lat_ix, pool_w,
                                                 B, T, first_entry, c, err);
  else
    pack_kv_kernel<uint16_t><<<grid, 256, 0, st>>>((const uint16_t *)lat_kv, (const uint16_t *)lat_ix,
                                                    pool_w, B, T, first_entry, c, err);
}

void launch_pack_swa(const void *x, csa2_dtype dtype, int B, int T, const int32_t *pos,
                     uint8_t *codes, float *scale, int R, int32_t *err, cudaStream_t st) {
  const int64_t n = int64_t(B) * T;
  if (n == 0) return;
  const int grid = int((n + 7) / 8);
  if (dtype == CSA2_F32)
    pack_swa_kernel<float><<<grid, 256, 0, st>>>((const float *)x, B, T, pos, codes, scale, R, err);
  else
    pack_swa_kernel<uint16_t><<<grid, 256, 0, st>>>((const uint16_t *)x, B, T, pos, codes, scale, R, err);
}

}  // namespace csa2
