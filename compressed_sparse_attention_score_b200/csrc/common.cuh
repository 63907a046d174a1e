// Shared device helpers of the CSA2 kernels: number formats, cache addressing,
// error reporting.  Formats follow the cache entry layout declared in csa2.h.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

constexpr int D = CSA2_MAIN_DIM;
constexpr int DI = CSA2_IX_DIM;
constexpr int H = CSA2_HEADS;
constexpr int HI = CSA2_IX_HEADS;

// ------------------------------------------------------------------ errors
__device__ __forceinline__ void report(int32_t *err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ------------------------------------------------------------------ bf16
__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(uint32_t(b) << 16);
}

// ------------------------------------------------------------------ e2m1
// Round x (already divided by its scale) to the nearest e2m1 value, ties to the
// even code, saturating at +-6.  Magnitude index = decision points passed; a
// value that rounds to zero gets code 0 whatever its sign.
__device__ __forceinline__ uint32_t e2m1_code(float y) {
  float m = fabsf(y);
  uint32_t i = (m > 0.25f) + (m >= 0.75f) + (m > 1.25f) + (m >= 1.75f) + (m > 2.5f) +
               (m >= 3.5f) + (m > 5.0f);
  uint32_t neg = (__float_as_uint(y) >> 31) & (i != 0);
  return i | (neg << 3);
}

__device__ __forceinline__ float e2m1_value(uint32_t c) {
  // magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 as (2 + mantissa) * 2^(exp - 2), subnormal at exp 0
  uint32_t e = (c >> 1) & 3, m = c & 1;
  float mag = e == 0 ? 0.5f * float(m) : float(2 + m) * __int_as_float((127 + int(e) - 2) << 23);
  return (c & 8) ? -mag : mag;
}

// ------------------------------------------------------------------ E4M3
// Round to nearest even, saturating at +-448; a result of zero is code 0 whatever its sign.
__device__ __forceinline__ uint32_t e4m3_code(float v) {
  const uint32_t c = uint32_t(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
  return (c & 0x7F) ? c : 0u;
}

// Exact value of an E4M3 code (bias 7; exponent 0 is subnormal with quantum 2^-9).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  uint32_t e = (c >> 3) & 15, m = c & 7;
  float mag = e == 0 ? float(m) * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (c & 0x80) ? -mag : mag;
}

// ------------------------------------------------------------------ E8M0
// ceil(log2 q) for q = amax / 6 > 0, clamped to [-127, 127].
__device__ __forceinline__ int e8m0_ceil_exponent(float q) {
  uint32_t u = __float_as_uint(q);
  int be = int(u >> 23) & 255;
  uint32_t mant = u & 0x7FFFFF;
  int e;
  if (be == 0) {                       // subnormal: q = mant * 2^-149
    int msb = 31 - __clz(mant);        // floor(log2 mant)
    e = msb - 149 + ((mant & (mant - 1)) != 0);
  } else {
    e = be - 127 + (mant != 0);
  }
  return max(-127, min(127, e));
}

__device__ __forceinline__ float pow2f(int e) {  // exact 2^e for e in [-127, 127]
  return e >= -126 ? __uint_as_float(uint32_t(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// ------------------------------------------------------------------ cache addressing
// Physical slot of entry n of sequence b, or -1 if outside the cache.
__device__ __forceinline__ int64_t cache_slot(const csa2_cache &c, int b, int64_t n) {
  int64_t s;
  if (c.page_table == nullptr) {
    if (n < 0 || n >= c.seq_stride) return -1;
    s = int64_t(b) * c.seq_stride + n;
  } else {
    int64_t p = n / c.page_size;
    if (n < 0 || p >= c.max_pages) return -1;
    int32_t pid = c.page_table[int64_t(b) * c.max_pages + p];
    if (pid < 0) return -1;
    s = int64_t(pid) * c.page_size + (n % c.page_size);
  }
  return s < c.num_slots ? s : -1;
}

// Entries visible to a query at position pos of sequence b.
__device__ __forceinline__ int visible_entries(const csa2_cache &c, int b, int pos) {
  int n = c.num_entries[b];
  int by_pos = pos < 0 ? 0 : (pos + 1) / c.ratio;
  return min(n, by_pos);
}

// Monotone map of fp32 scores to uint32 keys (larger score -> larger key).
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
constexpr uint32_t KEY_NEG_INF = 0x007FFFFFu;  // score_key(-inf)

// Exclusive block-wide prefix sum of v (blockDim a multiple of 32, at most 1024);
// *total receives the block sum.  sm must hold 32 ints.  Contains __syncthreads.
__device__ __forceinline__ int block_exclusive_scan_1024(int v, int *sm, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nw ? sm[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    sm[lane] = t;
  }
  __syncthreads();
  const int off = (warp ? sm[warp - 1] : 0) + x - v;
  *total = sm[nw - 1];
  __syncthreads();
  return off;
}

}  // namespace csa2
