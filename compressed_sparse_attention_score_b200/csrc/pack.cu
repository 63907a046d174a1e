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

// Quantise the pooled entry a warp holds (lane l: main values [16l, 16l+16), one E4M3 block,
// and indexer values [4l, 4l+4), eight lanes per E8M0 block) and store it at `slot`.
__device__ __forceinline__ void store_entry(const float (&x)[16], const float (&xi)[4], int64_t slot,
                                            const csa2_cache &c, int lane) {
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

// exp(x) from a fixed sequence of fp32 operations (so that the gated compressor's weights,
// and through them the quantised codes, do not depend on a math library): t = x log2(e),
// n = rint(t), f = t - n, 2^f = e^(f ln 2) by its Taylor polynomial of degree 7 (Horner,
// each product and sum rounded), times 2^n; 0 below 2^-126, inf above 2^127.  The
// coefficients are (ln 2)^i / i! rounded to fp32.
__device__ __forceinline__ float exp_fixed(float x) {
  constexpr float c[8] = {0x1.0p+0f,      0x1.62e430p-1f,  0x1.ebfbe0p-3f,  0x1.c6b08ep-5f,
                          0x1.3b2ab6p-7f, 0x1.5d87fep-10f, 0x1.430912p-13f, 0x1.ffcbfcp-17f};
  const float t = __fmul_rn(x, 0x1.715476p+0f);
  const float n = rintf(t);
  const float f = __fsub_rn(t, n);
  float p = c[7];
#pragma unroll
  for (int i = 6; i >= 0; --i) p = __fadd_rn(__fmul_rn(p, f), c[i]);
  if (n < -126.f) return 0.f;
  if (n > 127.f) return INFINITY;
  return __fmul_rn(p, __int_as_float((int(n) + 127) << 23));
}

// One warp per new entry.  Lane l owns main values [16l, 16l+16) (one E4M3 block)
// and indexer values [4l, 4l+4) (eight lanes per E8M0 block).  Pooling: pool_w per token
// (or fp32(1/r)), or with gate_kv / gate_ix the gated sum: per channel the softmax over the
// entry's r tokens of the gate logits (max subtracted, exp_fixed, sum left to right, fp32
// division) weights the tokens, summed left to right.
template <typename T>
__global__ void __launch_bounds__(256) pack_kv_kernel(const T *__restrict__ lat_kv,
                                                      const T *__restrict__ lat_ix,
                                                      const float *__restrict__ pool_w,
                                                      const float *__restrict__ gate_kv,
                                                      const float *__restrict__ gate_ix, int B, int T_,
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
  float x[16], xi[4];
  const int64_t tok0 = int64_t(b) * T_ + int64_t(j) * c.ratio;

  if (gate_kv) {
    // ---- gated sum: three passes over the group (max, normaliser, weighted sum)
    float m[16], mi[4], den[16], deni[4];
    for (int t = 0; t < c.ratio; ++t) {
      float g[16], gi[4];
      load16<float>(gate_kv + (tok0 + t) * D + 16 * lane, g);
      load4<float>(gate_ix + (tok0 + t) * DI + 4 * lane, gi);
#pragma unroll
      for (int i = 0; i < 16; ++i) m[i] = t == 0 ? g[i] : fmaxf(m[i], g[i]);
#pragma unroll
      for (int i = 0; i < 4; ++i) mi[i] = t == 0 ? gi[i] : fmaxf(mi[i], gi[i]);
    }
    for (int t = 0; t < c.ratio; ++t) {
      float g[16], gi[4];
      load16<float>(gate_kv + (tok0 + t) * D + 16 * lane, g);
      load4<float>(gate_ix + (tok0 + t) * DI + 4 * lane, gi);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float ev = exp_fixed(__fsub_rn(g[i], m[i]));
        den[i] = t == 0 ? ev : __fadd_rn(den[i], ev);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float ev = exp_fixed(__fsub_rn(gi[i], mi[i]));
        deni[i] = t == 0 ? ev : __fadd_rn(deni[i], ev);
      }
    }
    for (int t = 0; t < c.ratio; ++t) {
      float g[16], gi[4], v[16], vi[4];
      load16<float>(gate_kv + (tok0 + t) * D + 16 * lane, g);
      load4<float>(gate_ix + (tok0 + t) * DI + 4 * lane, gi);
      load16<T>(lat_kv + (tok0 + t) * D + 16 * lane, v);
      load4<T>(lat_ix + (tok0 + t) * DI + 4 * lane, vi);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float term = __fmul_rn(__fdiv_rn(exp_fixed(__fsub_rn(g[i], m[i])), den[i]), v[i]);
        x[i] = t == 0 ? term : __fadd_rn(x[i], term);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float term = __fmul_rn(__fdiv_rn(exp_fixed(__fsub_rn(gi[i], mi[i])), deni[i]), vi[i]);
        xi[i] = t == 0 ? term : __fadd_rn(xi[i], term);
      }
    }
    store_entry(x, xi, slot, c, lane);
    return;
  }

  // ---- pool the tokens of this entry (fp32, left to right, no fused multiply-add)
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

  store_entry(x, xi, slot, c, lane);
}

// Decode-time append, one warp per sequence (lanes as in pack_kv_kernel).  The token at
// position pos[b] goes to the sequence's staging row pos % r (fp32: exactly the input); when
// it completes a group of r tokens, the group is pooled like pack_kv_kernel does (fp32, left to
// right, weight fp32(1/r)) into entry pos / r, which is quantised and stored, and
// num_entries[b] is raised to pos / r + 1.  Staging row t of sequence b (512 main then 128
// indexer values) starts at stage + b * stage_stride + t * 640; stage may be NULL when r = 1.
template <typename T>
__global__ void __launch_bounds__(256) append_kv_kernel(const T *__restrict__ lat_kv, const T *__restrict__ lat_ix,
                                                        int B, const int32_t *__restrict__ pos, float *stage,
                                                        int64_t stage_stride, csa2_cache c, int32_t *num_entries,
                                                        int32_t *err) {
  const int lane = threadIdx.x & 31;
  const int b = int(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (b >= B) return;
  const int p = pos[b];
  if (p < 0) return;  // padding row
  const int r = c.ratio, cur = p % r;
  float v[16], vi[4];
  load16<T>(lat_kv + int64_t(b) * D + 16 * lane, v);
  load4<T>(lat_ix + int64_t(b) * DI + 4 * lane, vi);
  float *srow = stage ? stage + int64_t(b) * stage_stride : nullptr;
  if (srow && r > 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      reinterpret_cast<float4 *>(srow + cur * (D + DI) + 16 * lane)[i] =
          make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    *reinterpret_cast<float4 *>(srow + cur * (D + DI) + D + 4 * lane) = make_float4(vi[0], vi[1], vi[2], vi[3]);
  }
  if (cur != r - 1) return;  // the group is not complete yet
  const int j = p / r;
  const int64_t slot = cache_slot(c, b, j);
  if (slot < 0) {
    if (lane == 0) report(err, CSA2_ERR_INDEX);
    return;
  }
  if (r > 1 && !srow) {
    if (lane == 0) report(err, CSA2_ERR_SHAPE);
    return;
  }
  const float wt = __fdiv_rn(1.0f, float(r));
  float x[16], xi[4];
  for (int t = 0; t < r; ++t) {
    float u[16], ui[4];
    if (t == cur) {
#pragma unroll
      for (int i = 0; i < 16; ++i) u[i] = v[i];
#pragma unroll
      for (int i = 0; i < 4; ++i) ui[i] = vi[i];
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 f = reinterpret_cast<const float4 *>(srow + t * (D + DI) + 16 * lane)[i];
        u[4 * i] = f.x, u[4 * i + 1] = f.y, u[4 * i + 2] = f.z, u[4 * i + 3] = f.w;
      }
      const float4 f = *reinterpret_cast<const float4 *>(srow + t * (D + DI) + D + 4 * lane);
      ui[0] = f.x, ui[1] = f.y, ui[2] = f.z, ui[3] = f.w;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = t == 0 ? __fmul_rn(wt, u[i]) : __fadd_rn(x[i], __fmul_rn(wt, u[i]));
#pragma unroll
    for (int i = 0; i < 4; ++i) xi[i] = t == 0 ? __fmul_rn(wt, ui[i]) : __fadd_rn(xi[i], __fmul_rn(wt, ui[i]));
  }
  store_entry(x, xi, slot, c, lane);
  if (lane == 0 && num_entries) atomicMax(&num_entries[b], j + 1);
}

// One warp per SWA token; lane l owns values [16l, 16l+16).  Only the last R
// tokens of a call are stored (earlier ones would be overwritten in the ring).  Ring b
// takes its positions from row b % pos_rows of pos (several layers' rings of the same
// sequences in one launch).
template <typename T>
__global__ void __launch_bounds__(256) pack_swa_kernel(const T *__restrict__ x, int B, int T_,
                                                       const int32_t *__restrict__ pos, int pos_rows,
                                                       uint8_t *__restrict__ codes,
                                                       float *__restrict__ scale, int R,
                                                       int32_t *err) {
  const int lane = threadIdx.x & 31;
  const int64_t e = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (e >= int64_t(B) * T_) return;
  const int b = int(e / T_), t = int(e % T_);
  if (t < T_ - R) return;
  const int p = pos[int64_t(b % pos_rows) * T_ + t];
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
                    const float *gate_kv, const float *gate_ix, int B, int T, const int32_t *first_entry,
                    const csa2_cache &c, int32_t *err, cudaStream_t st) {
  const int64_t n = int64_t(B) * (T / c.ratio);
  if (n == 0) return;
  const int grid = int((n + 7) / 8);
  if (dtype == CSA2_F32)
    pack_kv_kernel<float><<<grid, 256, 0, st>>>((const float *)lat_kv, (const float *)lat_ix, pool_w, gate_kv,
                                                 gate_ix, B, T, first_entry, c, err);
  else
    pack_kv_kernel<uint16_t><<<grid, 256, 0, st>>>((const uint16_t *)lat_kv, (const uint16_t *)lat_ix, pool_w,
                                                    gate_kv, gate_ix, B, T, first_entry, c, err);
}

void launch_pack_swa(const void *x, csa2_dtype dtype, int B, int T, const int32_t *pos, int pos_rows,
                     uint8_t *codes, float *scale, int R, int32_t *err, cudaStream_t st) {
  const int64_t n = int64_t(B) * T;
  if (n == 0) return;
  const int grid = int((n + 7) / 8);
  if (dtype == CSA2_F32)
    pack_swa_kernel<float><<<grid, 256, 0, st>>>((const float *)x, B, T, pos, pos_rows, codes, scale, R, err);
  else
    pack_swa_kernel<uint16_t><<<grid, 256, 0, st>>>((const uint16_t *)x, B, T, pos, pos_rows, codes, scale, R,
                                                    err);
}

void launch_append_kv(const void *lat_kv, const void *lat_ix, csa2_dtype dtype, int B, const int32_t *pos,
                      float *stage, int64_t stage_stride, const csa2_cache &c, int32_t *num_entries, int32_t *err,
                      cudaStream_t st) {
  if (B == 0) return;
  const int grid = (B + 7) / 8;
  if (dtype == CSA2_F32)
    append_kv_kernel<float><<<grid, 256, 0, st>>>((const float *)lat_kv, (const float *)lat_ix, B, pos, stage,
                                                   stage_stride, c, num_entries, err);
  else
    append_kv_kernel<uint16_t><<<grid, 256, 0, st>>>((const uint16_t *)lat_kv, (const uint16_t *)lat_ix, B, pos,
                                                      stage, stage_stride, c, num_entries, err);
}

}  // namespace csa2
