// K8: log-sum-exp merge of two attention partials (elementwise, HBM streaming).
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

// One warp per row; lanes stride over the row in float4 units.  o may alias o1 or o2 and
// lse may alias l1 or l2 (each element is read before it is written, by the same thread), so
// none of the pointers is declared __restrict__.
__global__ void __launch_bounds__(256) merge_kernel(const float *o1, const float *l1, const float *o2,
                                                    const float *l2, int64_t rows, int D_, float *o, float *lse) {
  const int lane = threadIdx.x & 31;
  const int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const float a = l1[r], b = l2[r];
  const float m = fmaxf(a, b);
  float w1 = 0.f, w2 = 0.f, out_l = -INFINITY;
  if (m != -INFINITY) {
    w1 = a == -INFINITY ? 0.f : __expf(a - m);
    w2 = b == -INFINITY ? 0.f : __expf(b - m);
    const float den = w1 + w2;
    out_l = m + logf(den);
    w1 /= den;
    w2 /= den;
  }
  const float4 *p1 = reinterpret_cast<const float4 *>(o1 + r * D_);
  const float4 *p2 = reinterpret_cast<const float4 *>(o2 + r * D_);
  float4 *po = reinterpret_cast<float4 *>(o + r * D_);
  for (int i = lane; i < D_ / 4; i += 32) {
    const float4 x = p1[i], y = p2[i];
    po[i] = make_float4(w1 * x.x + w2 * y.x, w1 * x.y + w2 * y.y, w1 * x.z + w2 * y.z, w1 * x.w + w2 * y.w);
  }
  __syncwarp();
  if (lane == 0) lse[r] = out_l;
}

void launch_merge(const float *o1, const float *l1, const float *o2, const float *l2, int64_t rows, int D_,
                  float *o, float *lse, cudaStream_t st) {
  if (rows == 0) return;
  merge_kernel<<<int((rows + 7) / 8), 256, 0, st>>>(o1, l1, o2, l2, rows, D_, o, lse);
}

}  // namespace csa2
