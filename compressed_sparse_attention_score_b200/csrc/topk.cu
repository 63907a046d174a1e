// K5 (row form): deterministic top-k of each score row by radix select.
//
// One CTA of 1024 threads per row.  Four 8-bit radix passes over the row find
// the exact key T of the k-th best candidate and how many candidates equal to T
// are needed; an ordered pass then writes, in ascending position order, every
// candidate above T and the lowest-positioned candidates equal to T.
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

constexpr int TOPK_THREADS = 1024;

// Exclusive block-wide prefix sum of v; *total receives the block sum.
__device__ __forceinline__ int block_exclusive_scan(int v, int *sm, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nw ? sm[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
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

__global__ void __launch_bounds__(TOPK_THREADS) topk_rows_kernel(
    const float *__restrict__ scores, const int32_t *__restrict__ n_valid, int N, int k,
    int32_t *__restrict__ idx, float *__restrict__ val, const int32_t *__restrict__ map) {
  __shared__ int hist[256];
  __shared__ int scan_sm[32];
  __shared__ int sel_bin, sel_rem, take_all;
  const int row = blockIdx.x, tid = threadIdx.x;
  const int n = n_valid ? max(0, min(N, n_valid[row])) : N;
  const float *s = scores + int64_t(row) * N;

  uint32_t prefix = 0, mask = 0;
  if (tid == 0) take_all = 0, sel_rem = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (tid < 256) hist[tid] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += TOPK_THREADS) {
      const uint32_t key = score_key(s[j]);
      if (key != KEY_NEG_INF && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
    }
    __syncthreads();
    if (tid < 32) {
      // lane l covers bins 255-8l down to 248-8l (descending score order)
      int c[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = hist[255 - 8 * tid - i], sum += c[i];
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      const int rem = sel_rem;
      if (pass == 0 && total <= k) {
        if (tid == 0) take_all = 1;
      } else {
        const int excl = incl - sum;
        if (excl < rem && incl >= rem) {
          int cum = excl;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (cum + c[i] >= rem) {
              sel_bin = 255 - 8 * tid - i;
              sel_rem = rem - cum;
              break;
            }
            cum += c[i];
          }
        }
      }
    }
    __syncthreads();
    if (take_all) break;
    prefix |= uint32_t(sel_bin) << shift;
    mask |= 0xFFu << shift;
    __syncthreads();
  }
  const bool all = take_all != 0;
  const uint32_t T = prefix;
  const int need_eq = all ? 0 : sel_rem;

  int out = 0, eq_seen = 0;
  int32_t *orow = idx + int64_t(row) * k;
  float *vrow = val ? val + int64_t(row) * k : nullptr;
  const int32_t *mrow = map ? map + int64_t(row) * N : nullptr;
  for (int base = 0; base < n && out < k; base += 4 * TOPK_THREADS) {
    const int j0 = base + 4 * tid;
    float sv[4];
    bool gt[4], eq[4];
    int ceq = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = j0 + i;
      sv[i] = j < n ? s[j] : -INFINITY;
      const uint32_t key = score_key(sv[i]);
      const bool valid = j < n && key != KEY_NEG_INF;
      gt[i] = valid && (all || key > T);
      eq[i] = valid && !all && key == T;
      ceq += eq[i];
    }
    int tot_eq, tot_sel;
    const int eq_off = block_exclusive_scan(ceq, scan_sm, &tot_eq);
    bool sel[4];
    int csel = 0, eb = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      sel[i] = gt[i] || (eq[i] && eq_seen + eq_off + eb < need_eq);
      eb += eq[i];
      csel += sel[i];
    }
    const int off = block_exclusive_scan(csel, scan_sm, &tot_sel);
    int w = out + off;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (sel[i] && w < k) {
        orow[w] = mrow ? mrow[j0 + i] : j0 + i;
        if (vrow) vrow[w] = sv[i];
        ++w;
      }
    }
    out += tot_sel;
    eq_seen += tot_eq;
  }
  for (int i = min(out, k) + tid; i < k; i += TOPK_THREADS) {
    orow[i] = -1;
    if (vrow) vrow[i] = -INFINITY;
  }
}

void launch_topk_rows(const float *scores, const int32_t *n_valid, int R, int N, int k, int32_t *idx,
                      float *val, const int32_t *map, cudaStream_t st) {
  if (R == 0 || k == 0) return;
  topk_rows_kernel<<<R, TOPK_THREADS, 0, st>>>(scores, n_valid, N, k, idx, val, map);
}

}  // namespace csa2
