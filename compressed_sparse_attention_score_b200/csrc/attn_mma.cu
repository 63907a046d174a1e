// K6/K7/K8 (tensor-core form): attention of 64 query heads over a row's selected
// global-KV entries and/or its sliding window, on tcgen05 (kind::f16).
//
// Each key's 512-d vector is both key and value.  Keys come from two sources that share
// one softmax (so a CTA given both returns the log-sum-exp merge of the two branches
// exactly):
//   sparse  -- listed main-KV entries (or, dense, every visible entry of a range):
//              e2m1 x E4M3-per-16 dequantised to fp16 (exact: <= 6 significant
//              bits, in fp16 range);
//   window  -- SWA tokens: E4M3 codes to fp16 (exact); the token's fp32 scale is
//              folded into the logit multiplier and into P.
// The bf16 query heads enter the MMA prescaled by a power of two per head (see
// store_query_fp16), so they are exact in fp16 whatever their magnitude.
// Two kernels:
//   attn_tile_kernel  -- one 128-key tile per CTA, 32 heads (a cluster of up to 5 CTAs
//              per row and head group): the producers load their key halves into
//              registers and dequantise them into a 128 KB fp16 tile (8 blocks of 64
//              dims, 128-byte swizzle) that is the K-major A operand of S^T = K Q^T
//              and the MN-major A operand of O^T = V^T P^T, so every key is read and
//              dequantised once;
//   attn_mma_kernel   -- up to 5 tiles per CTA, all 64 heads (many rows, or dense rows
//              in clusters of up to 16): the same tile as a ring with one mbarrier pair
//              per 64-dim block, S^T of every tile kept in TMEM for an exact two-pass
//              softmax, each tile dequantised again for O^T (a CTA with one tile keeps it).
// Softmax: per-head max and sum by warp reduce-scatter, P^T written to shared memory
// in fp16 (MN-major).  Output: O / sum and lse = max + log(sum), coalesced fp32
// stores; when a cluster of CTAs splits the row's keys, each CTA pushes each owner its
// slice of the partial O (with max and sum) into distributed shared memory, and the
// owners combine.  A single thread issues the tensor-core work; every wait is
// time-bounded.
#include <cooperative_groups.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace cg = cooperative_groups;

namespace csa2 {
using namespace sm100;

namespace {
constexpr int AM_PRODUCERS = 256;               // warps 0-7 dequantise keys
constexpr int AM_THREADS = AM_PRODUCERS + 32;   // warp 8 drives the tensor core
constexpr int AM_HG = 32;          // heads per CTA of the one-tile kernel = MMA N
constexpr int RG = 64;             // heads per CTA of the general kernel (every head of a row)
constexpr int AM_TILE = 128;       // keys per S^T tile
constexpr int AM_MAXKEYS = 640;    // 512 listed entries + 128 window tokens
constexpr int AM_BLOCKS = 8;       // 64-dim blocks of a key tile = operand buffers (one tile)
constexpr int AM_STAGE = 16384;    // one block: 128 keys x 64 dims fp16
constexpr uint32_t AM_TMEM_COLS = 256;
constexpr uint64_t AM_WAIT_NS = 2000000000ull;

constexpr int AM_MAXCS = 16;      // largest cluster splitting one row's keys
constexpr int AM_QU = AM_HG * (D / 8) / AM_PRODUCERS;   // 16-byte query chunks per producer thread
template <int HG>
__host__ __device__ constexpr int qu_of() { return HG * (D / 8) / AM_PRODUCERS; }
constexpr uint32_t RG_TMEM_COLS = 512;  // S^T of 5 tiles x 64 heads; O^T (4 x 64) reuses those columns
// General kernel (RG heads): Q during the first phase, P^T (written after every S^T product has
// completed) in the same bytes afterwards.
constexpr int SM_QP_BYTES = (8 * RG * 128 > AM_MAXKEYS * RG * 2) ? 8 * RG * 128 : AM_MAXKEYS * RG * 2;
constexpr int SM_Q = 0;                              // 8 chunks x [RG heads x 128 B]
constexpr int SM_P = 0;                              // P^T [640 keys x RG x 2 B], 128-byte swizzle
constexpr int SM_STG = SM_QP_BYTES;                  // one key tile: 8 x 16 KB blocks
constexpr int SM_SLOT = SM_STG + AM_BLOCKS * AM_STAGE;
constexpr int SM_MU = SM_SLOT + AM_MAXKEYS * 8;      // logit multiplier per key
constexpr int SM_PV = SM_MU + AM_MAXKEYS * 4;        // P multiplier per key
constexpr int SM_RED = SM_PV + AM_MAXKEYS * 4;       // [8 warps][32 heads]; [CS][RG] weights + [RG] sums
constexpr int SM_HM = SM_RED + (AM_MAXCS + 1) * RG * 4;   // head max [RG], head sum [RG]
constexpr int SM_QS = SM_HM + 2 * RG * 4;            // query prescale: [8 warps][QU] max bits, [RG] 2^-s
constexpr int SM_NEW = SM_QS + (8 * qu_of<RG>() + RG) * 4;  // this step's window token: 512 codes, scale, [4] maxima
constexpr int SM_BAR = SM_NEW + 512 + 32;
constexpr int SM_MISC = SM_BAR + 8 * (2 * AM_BLOCKS + 1);
constexpr int SM_TOTAL = SM_MISC + 16;
constexpr size_t AM_SMEM = SM_TOTAL + 1024;
static_assert(AM_SMEM <= 227 * 1024, "general attention kernel exceeds the shared memory of a CTA");
static_assert(SM_STG % 1024 == 0, "operand buffers need 1 KB alignment");
}  // namespace

struct AttnArgs {
  const uint16_t *q;
  int Q;
  const int32_t *q_pos;
  float tau;
  // sparse source: the k listed entries idx (idx == nullptr: none), or with dense != 0
  // every visible entry n in [e0, e1)
  const int32_t *idx;
  int k;
  int dense, e0, e1;
  int n_bound;  // dense: entries a query may see (more sets CSA2_ERR_SHAPE)
  csa2_cache c;
  // window source (codes == nullptr: none); with swa_new [rows][512] bf16, this step's token of
  // each row is quantised in the launch, used as the window's last key and stored in the ring
  const uint8_t *codes;
  const float *scale;
  int R, window;
  const uint16_t *swa_new;
  float *o, *lse;
  int32_t *err;
};

// Offsets inside the swizzled operand layouts (bytes).
// K-major, 128-byte rows, 1 KB atoms of 8 rows: 16-byte unit u of row r.
__device__ __forceinline__ int kmaj128(int r, int u) { return (r >> 3) * 1024 + (r & 7) * 128 + ((u ^ (r & 7)) << 4); }
// MN-major, 128-byte swizzle: element block (m / 64) at LBO 8192, K-row k: unit u of 8 M-elements.
__device__ __forceinline__ int mnmaj128(int k, int mblk, int u) {
  return mblk * 8192 + (k >> 3) * 1024 + (k & 7) * 128 + ((u ^ (k & 7)) << 4);
}
// MN-major, 64-byte swizzle (P^T): K-row k (key), unit u of 8 heads.
__device__ __forceinline__ int mnmaj64(int k, int u) { return (k >> 3) * 512 + (k & 7) * 64 + ((u ^ ((k & 7) >> 1)) << 4); }

// Query prescale.  The query heads enter the fp16 MMA multiplied by a power of two 2^s per
// head that puts the head's largest |q| in [2^14, 2^15): every bf16 value within a factor
// 2^32 of that maximum is then exact in fp16 (no overflow above 65504, no lost bits in the
// subnormals), and the logits are multiplied back by 2^-s, which is exact in fp32.
// Producer thread tid holds query chunks it = tid + 256 u, i.e. head tid / 64 + 4 u, so the
// two warps 2c, 2c + 1 share the heads c + 4 u.  Each warp publishes the largest |bf16| bit
// pattern of each of its AM_QU chunks' heads (|x| orders like its bits).
template <int HG = AM_HG>
__device__ __forceinline__ void publish_query_max(const uint4 (&qraw)[qu_of<HG>()], uint32_t *qmx) {
  constexpr int QU = qu_of<HG>();
  const int warp = threadIdx.x >> 5;
#pragma unroll
  for (int u = 0; u < QU; ++u) {
    const uint32_t w[4] = {qraw[u].x, qraw[u].y, qraw[u].z, qraw[u].w};
    uint32_t mb = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) mb = max(mb, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
    mb = __reduce_max_sync(0xffffffffu, mb);
    if ((threadIdx.x & 31) == 0) qmx[warp * QU + u] = mb;
  }
}
// Exponent s of the prescale of a head whose largest |bf16| bit pattern is mb (0 for an all-zero
// or non-finite head).  floor(log2 max) = E - 127 for the biased exponent E.
__device__ __forceinline__ int query_prescale_exp(uint32_t mb) {
  const int E = int(mb >> 7);
  if (mb == 0 || E >= 255) return 0;
  return min(126, 141 - max(E, 1));
}
template <int HG = AM_HG>
__device__ __forceinline__ uint32_t head_max_bits(const uint32_t *qmx, int h) {
  constexpr int QU = qu_of<HG>();
  const int c = h & 3, u = h >> 2;
  return max(qmx[(2 * c) * QU + u], qmx[(2 * c + 1) * QU + u]);
}
// Write this producer's query chunks, prescaled, as fp16 into the K-major 128-byte-swizzled
// Q operand (8 chunks of 64 dims x HG heads); thread tid < HG also stores 2^-s of head tid.
template <int HG = AM_HG>
__device__ __forceinline__ void store_query_fp16(const uint4 (&qraw)[qu_of<HG>()], const uint32_t *qmx, float *qinv,
                                                 uint8_t *qdst) {
  constexpr int QU = qu_of<HG>();
  const int tid = threadIdx.x;
#pragma unroll
  for (int u = 0; u < QU; ++u) {
    const int it = tid + u * AM_PRODUCERS, h = it / (D / 8), u8 = it % (D / 8);
    const float sc = pow2f(query_prescale_exp(head_max_bits<HG>(qmx, h)));
    const uint32_t w[4] = {qraw[u].x, qraw[u].y, qraw[u].z, qraw[u].w};
    uint32_t o4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 hv = __floats2half2_rn(__uint_as_float(w[i] << 16) * sc, __uint_as_float(w[i] & 0xFFFF0000u) * sc);
      o4[i] = *reinterpret_cast<const uint32_t *>(&hv);
    }
    *reinterpret_cast<uint4 *>(qdst + (u8 / 8) * (HG * 128) + kmaj128(h, u8 % 8)) =
        make_uint4(o4[0], o4[1], o4[2], o4[3]);
  }
  if (tid < HG) qinv[tid] = pow2f(-query_prescale_exp(head_max_bits<HG>(qmx, tid)));
}

// Raw bytes of one half of a key (dims 256 half .. +255) into registers: a listed entry's
// 128 code bytes (rr[0..7]) and 16 scale bytes (rr[8]) from slot s of the cache, a window
// token's 256 code bytes (rr[0..15]) from slot s of the ring, or from own_codes (this step's
// token, quantised in the launch).  Nothing for a masked key (s < 0).
// Pieces [I0, I1) only (of 9 for a listed entry, 16 for a window token), so that a caller can
// load the first 9 of the next key ahead and the rest of a window token later.
template <int I0 = 0, int I1 = 16, int N>
__device__ __forceinline__ void load_key_half(const AttnArgs &p, int64_t s, bool sparse, const uint8_t *own_codes,
                                              int half, uint4 (&rr)[N]) {
  static_assert(I1 <= N, "register set too small");
  if (s < 0) return;
  if (sparse) {
    const uint4 *src = reinterpret_cast<const uint4 *>(p.c.kv_codes + s * CSA2_MAIN_CODE_BYTES + half * 128);
#pragma unroll
    for (int i = I0; i < (I1 < 8 ? I1 : 8); ++i) rr[i] = src[i];
    if (I0 <= 8 && I1 > 8) rr[8] = *reinterpret_cast<const uint4 *>(p.c.kv_scales + s * CSA2_MAIN_SCALE_BYTES + half * 16);
  } else {
    const uint4 *src = reinterpret_cast<const uint4 *>((own_codes ? own_codes : p.codes + s * CSA2_SWA_DIM) + half * 256);
#pragma unroll
    for (int i = I0; i < I1; ++i) rr[i] = src[i];
  }
}

// Block c (dims 256 half + 64 c .. +63) of a key half held in registers, dequantised to fp16
// (exact) into row key_in of a K-major 128-byte-swizzled 128-key block; zeros for a masked key.
__device__ __forceinline__ void dequant_block(const uint4 (&rr)[16], bool sparse, bool valid, int c, int key_in,
                                              uint8_t *dst) {
#pragma unroll
  for (int q2 = 0; q2 < 2; ++q2) {  // 32 dims at a time
    uint32_t h16[16];
    if (!valid) {
#pragma unroll
      for (int i = 0; i < 16; ++i) h16[i] = 0u;
    } else if (sparse) {
      const uint4 a = rr[2 * c + q2];
      const uint32_t sw = (&rr[8].x)[c];  // scale bytes of dims 64c .. 64c+63 of this half
      const uint32_t sc = (sw >> (16 * q2)) & 0xFFFF;
      const uint32_t s0 = cvt_e4m3x2_f16x2((sc & 0xFF) * 0x101u);
      const uint32_t s1 = cvt_e4m3x2_f16x2(((sc >> 8) & 0xFF) * 0x101u);
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int i = 0; i < 16; ++i)
        h16[i] = hmul2_u32(cvt_e2m1x2_f16x2((w[i >> 2] >> (8 * (i & 3))) & 0xFF), i < 8 ? s0 : s1);
    } else {
      const uint4 a = rr[4 * c + 2 * q2], bb = rr[4 * c + 2 * q2 + 1];
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, bb.x, bb.y, bb.z, bb.w};
#pragma unroll
      for (int i = 0; i < 16; ++i) h16[i] = cvt_e4m3x2_f16x2((w[i >> 1] >> (16 * (i & 1))) & 0xFFFF);
    }
#pragma unroll
    for (int v = 0; v < 4; ++v)
      *reinterpret_cast<uint4 *>(dst + kmaj128(key_in, 4 * q2 + v)) =
          make_uint4(h16[4 * v], h16[4 * v + 1], h16[4 * v + 2], h16[4 * v + 3]);
  }
}

// This step's own window token of the CTA's query row, quantised exactly as pack_swa_kernel does
// (fp32 scale = amax / 448, E4M3 codes, a zero result code 0): its 512 codes go to new_codes
// (shared), its scale to *new_scale (shared); the CTA given `store` also writes both to the ring
// slot of position pos, which no CTA of this launch reads (window slots are distinct mod R).
// Called by every thread of the CTA; contains two __syncthreads.
// The token's bf16 values 4 tid .. 4 tid + 3 (threads < 128), loaded at the start of the launch.
__device__ __forceinline__ uint2 load_new_token(const AttnArgs &p, int row) {
  return (p.swa_new && threadIdx.x < 128)
             ? *reinterpret_cast<const uint2 *>(p.swa_new + int64_t(row) * CSA2_SWA_DIM + 4 * threadIdx.x)
             : make_uint2(0u, 0u);
}
__device__ __forceinline__ void quantise_new_token(const AttnArgs &p, uint2 u, int ring, int pos, bool store,
                                                   uint8_t *new_codes, float *new_scale, float *red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  float am = 0.f;
  if (tid < 128) {
    v[0] = __uint_as_float(u.x << 16), v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    v[2] = __uint_as_float(u.y << 16), v[3] = __uint_as_float(u.y & 0xFFFF0000u);
    am = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    if (lane == 0) red[warp] = am;
  }
  __syncthreads();
  const float s = __fdiv_rn(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])), 448.0f);
  if (tid < 128) {
    uint32_t w = 0;
    if (s != 0.f) {
#pragma unroll
      for (int i = 0; i < 4; ++i) w |= e4m3_code(__fdiv_rn(v[i], s)) << (8 * i);
    }
    reinterpret_cast<uint32_t *>(new_codes)[tid] = w;
    const int64_t slot = int64_t(ring) * p.R + pos % p.R;
    // the ring is the caller's writable per-layer SWA cache (given as const for the reading calls)
    if (store) reinterpret_cast<uint32_t *>(const_cast<uint8_t *>(p.codes) + slot * CSA2_SWA_DIM)[tid] = w;
    if (store && tid == 0) const_cast<float *>(p.scale)[slot] = s;
    if (tid == 0) *new_scale = s;
  }
  __syncthreads();
}

// Max or sum over the 32 lanes of each of 32 per-lane values: afterwards lane l
// holds the reduction of value index l.  31 shuffles (reduce-scatter butterfly).
template <bool MAX>
__device__ __forceinline__ float reduce_scatter32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int width = 16; width >= 1; width >>= 1) {
    const bool upper = lane & width;
#pragma unroll
    for (int i = 0; i < width; ++i) {
      // keep the half selected by this lane's bit, send the other half
      const float send = upper ? v[i] : v[i + width];
      const float keep = upper ? v[i + width] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, width);
      v[i] = MAX ? fmaxf(keep, got) : keep + got;
    }
  }
  return v[0];
}

// Cluster epilogue of a key-split row.  Partial of this CTA's keys: O_s (relative to its own
// max m_s) in TMEM, plus m_s and l_s.  CTA q owns dims [q PER, q PER + PER); every CTA pushes
// each owner its slice of O_s and every owner its (m_s, l_s), straight from TMEM into the
// owners' receive buffers (remote stores, nothing waits on them), then one cluster barrier, and
// each owner combines its slice locally: o = sum_s e^(m_s - M) O_s / sum_s e^(m_s - M) l_s,
// M = max_s m_s.  The receive buffer (recv: CS x HG x PER floats, then CS x 2 HG statistics) is
// the CTA's key-tile memory, so a first barrier (split: arrive when this CTA's products are
// complete, wait before the first push) keeps peers from writing into a tile still being read.
template <int CS, int HG = AM_HG>
__device__ __forceinline__ void combine_partials(const AttnArgs &p, uint32_t tmem, bool aborted, bool has_keys,
                                                 float *recv, float *red, float *hmax, float *hsum, int row, int hg,
                                                 int split) {
  constexpr int PER = ((D + CS - 1) / CS + 3) & ~3;  // dims per owner, a multiple of 4
  constexpr int NWARP = 8;                           // warps reading TMEM: 4 lane quarters x 2
  constexpr int DPW = HG / 16;                       // (head group, 128-dim block) pairs per warp
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float *stats = recv + CS * HG * PER;  // [source][max HG | sum HG]
  cg::cluster_group cluster = cg::this_cluster();
  if (tid < HG && aborted) {
    hsum[tid] = 0.f;
    hmax[tid] = -INFINITY;
  }
  cluster_arrive();  // this CTA's tensor-core products are complete
  bool waited = false;
  static_assert(HG % 32 == 0 && 2 * DPW == 4 * (HG / 32), "the 8 warps share the (head group, block) pairs");
  if (warp < NWARP) {
    for (int u = 0; u < DPW; ++u) {
      const int pi = (warp >> 2) * DPW + u, hb = 32 * (pi >> 2), d = pi & 3;  // 32 heads x 128 dims
      uint32_t r0[16], r1[16];
      if (!aborted && has_keys) {
        const uint32_t ta = tmem + (uint32_t(32 * (warp & 3)) << 16) + d * HG + hb;
        tc_ld_32x32b_x16(ta, r0);
        tc_ld_32x32b_x16(ta + 16, r1);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) r0[i] = r1[i] = 0u;
      }
      if (!waited) {
        cluster_wait();  // every peer's tile memory is free
        waited = true;
      }
      const int dim = 128 * d + 32 * (warp & 3) + lane, q = dim / PER;
      float *dst = cluster.map_shared_rank(recv + (split * HG + hb) * PER + (dim - q * PER), q);
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        dst[h * PER] = __uint_as_float(r0[h]);
        dst[(16 + h) * PER] = __uint_as_float(r1[h]);
      }
    }
    if (tid < HG) {
      const float m = hmax[tid], l = hsum[tid];
#pragma unroll
      for (int q = 0; q < CS; ++q) {
        float *st = cluster.map_shared_rank(stats + split * 2 * HG, q);
        st[tid] = m;
        st[HG + tid] = l;
      }
    }
  } else {
    cluster_wait();
  }
  cluster.sync();  // every slice and statistic has arrived; no peer's memory is touched after this
  float *wts = red;  // [CS][HG] combination weights
  float *lsum = red + CS * HG;
  if (tid < HG) {
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < CS; ++q) M = fmaxf(M, stats[q * 2 * HG + tid]);
    float L = 0.f;
#pragma unroll
    for (int q = 0; q < CS; ++q) {
      const float mq = stats[q * 2 * HG + tid];
      const float wq = (M == -INFINITY || mq == -INFINITY) ? 0.f : __expf(mq - M);
      wts[q * HG + tid] = wq;
      L += wq * stats[q * 2 * HG + HG + tid];
    }
    lsum[tid] = L;
    if (split == 0) p.lse[int64_t(row) * H + hg * HG + tid] = L > 0.f ? M + logf(L) : -INFINITY;
  }
  __syncthreads();
  const int d0 = min(D, split * PER), nq = (min(D, d0 + PER) - d0) / 4;
  float *orow = p.o + (int64_t(row) * H + hg * HG) * D;
  for (int it = tid; it < HG * nq; it += AM_THREADS) {
    const int h = it / nq, dl = 4 * (it % nq);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < CS; ++q) {
      const float wq = wts[q * HG + h];
      const float4 x = *reinterpret_cast<const float4 *>(recv + (q * HG + h) * PER + dl);
      acc.x += wq * x.x;
      acc.y += wq * x.y;
      acc.z += wq * x.z;
      acc.w += wq * x.w;
    }
    const float L = lsum[h], inv = L > 0.f ? 1.f / L : 0.f;
    *reinterpret_cast<float4 *>(orow + h * D + d0 + dl) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
}

template <int CS>
__global__ void __launch_bounds__(AM_THREADS, 1) attn_mma_kernel(AttnArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int64_t *slot = reinterpret_cast<int64_t *>(smem + SM_SLOT);
  float *mu = reinterpret_cast<float *>(smem + SM_MU);
  float *pv = reinterpret_cast<float *>(smem + SM_PV);
  float *red = reinterpret_cast<float *>(smem + SM_RED);
  float *hmax = reinterpret_cast<float *>(smem + SM_HM);
  float *hsum = hmax + RG;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM_BAR);  // block written (128 arrivals)
  uint64_t *mma_done = full + AM_BLOCKS;                          // block consumed (tcgen05.commit)
  uint64_t *phase_done = mma_done + AM_BLOCKS;                    // all products of a phase complete
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SM_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + SM_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = tid < AM_PRODUCERS, issuer = tid == AM_PRODUCERS;
  const int row = blockIdx.x, hg = blockIdx.y;   // query row; its sequence b owns SWA ring b
  const int lrow = row, b = row / p.Q, ring = b;
  // The query block (an input of the call) is loaded first; everything else may be written by
  // the kernel launched just before this one, so it is read after grid_dep_wait().
  constexpr int QU = qu_of<RG>();
  uint4 qraw[QU];
  if (producer) {
    const uint16_t *qrow = p.q + (int64_t(row) * H + hg * RG) * D;
#pragma unroll
    for (int u = 0; u < QU; ++u) {
      const int it = tid + u * AM_PRODUCERS;
      qraw[u] = *reinterpret_cast<const uint4 *>(qrow + (it / (D / 8)) * D + (it % (D / 8)) * 8);
    }
  }
  const uint2 tok = load_new_token(p, row);  // this step's window token (an input too)
  grid_dep_launch();
  grid_dep_wait();
  const int pos = p.q_pos[row];

  // ---------------------------------------------------------------- key list
  const int nvis = (p.idx || p.dense) ? visible_entries(p.c, b, pos) : 0;
  const int nks = p.dense ? max(0, min(p.e1, nvis) - p.e0) : (p.idx ? p.k : 0);
  int lo = 0, nkw = 0;
  if (p.codes && pos >= 0) {
    lo = max(0, pos - p.window + 1);
    nkw = pos - lo + 1;
  }
  const int nk = nks + nkw;
  // this CTA's share of the key tiles (a cluster of CS CTAs splits the row's keys)
  const int split = CS > 1 ? int(cg::this_cluster().block_rank()) : 0;
  const int tiles_all = (nk + AM_TILE - 1) / AM_TILE;
  const int tps = (tiles_all + CS - 1) / CS;
  const int tile0 = min(tiles_all, split * tps);
  // a CTA holds at most AM_MAXKEYS keys (the launcher sizes the cluster for that); keys past
  // them, or dense entries past the caller's bound, are left out and reported
  const int ntiles = min(min(tiles_all, tile0 + tps) - tile0, AM_MAXKEYS / AM_TILE);
  if (tid == 0 && (tps > AM_MAXKEYS / AM_TILE || (p.dense && nvis > p.n_bound))) report(p.err, CSA2_ERR_SHAPE);
  const int key0 = tile0 * AM_TILE;  // first key of this CTA; local key j is key key0 + j
  // the query block (loaded above) is converted once the key list is done
  uint32_t *qmx = reinterpret_cast<uint32_t *>(smem + SM_QS);
  float *qinv = reinterpret_cast<float *>(smem + SM_QS + 8 * QU * 4);
  // this step's own window token (the row's last key), quantised here and stored by one CTA
  const bool own_token = p.swa_new && nkw > 0;
  uint8_t *new_codes = own_token ? smem + SM_NEW : nullptr;
  float *new_scale = reinterpret_cast<float *>(smem + SM_NEW + 512);
  if (own_token) quantise_new_token(p, tok, ring, pos, split == 0 && hg == 0, smem + SM_NEW, new_scale, new_scale + 4);
  // The list's index loads go out together (at most three keys per thread), then the slots,
  // then the window tokens' scales.
  constexpr int KPT = (AM_MAXKEYS + AM_THREADS - 1) / AM_THREADS;
  {
    int nidx[KPT];
#pragma unroll
    for (int r = 0; r < KPT; ++r) {
      const int jl = tid + r * AM_THREADS, j = key0 + jl;
      nidx[r] = (jl < ntiles * AM_TILE && j < nks) ? (p.dense ? p.e0 + j : p.idx[int64_t(lrow) * p.k + j]) : -1;
    }
    int64_t sl[KPT];
    float sc[KPT];
#pragma unroll
    for (int r = 0; r < KPT; ++r) {
      const int jl = tid + r * AM_THREADS, j = key0 + jl;
      sl[r] = -1;
      sc[r] = 1.f;
      if (jl >= ntiles * AM_TILE) continue;
      if (j < nks) {
        const int n = nidx[r];
        if (n != -1) {
          if (n < -1 || n >= nvis) {
            report(p.err, CSA2_ERR_INDEX);
          } else {
            sl[r] = cache_slot(p.c, b, n);
            if (sl[r] < 0) report(p.err, CSA2_ERR_INDEX);
          }
        }
      } else if (j < nk) {
        sl[r] = int64_t(ring) * p.R + (lo + (j - nks)) % p.R;
        sc[r] = (own_token && j == nk - 1) ? *new_scale : p.scale[sl[r]];
      }
    }
#pragma unroll
    for (int r = 0; r < KPT; ++r) {
      const int jl = tid + r * AM_THREADS, j = key0 + jl;
      if (jl >= ntiles * AM_TILE) continue;
      const bool win = j >= nks && j < nk;
      slot[jl] = sl[r];
      mu[jl] = j < nks ? p.tau : (win ? p.tau * sc[r] : 0.f);
      pv[jl] = j < nks ? 1.f : (win ? sc[r] : 0.f);
    }
  }
  if (producer) publish_query_max<RG>(qraw, qmx);
  if (warp == AM_PRODUCERS / 32) {
    tmem_alloc(tmem_slot, RG_TMEM_COLS);
    tmem_relinquish();
  }
  if (issuer) {
    for (int i = 0; i < AM_BLOCKS; ++i) {
      mbar_init(&full[i], AM_TILE);
      mbar_init(&mma_done[i], 1);
    }
    mbar_init(phase_done, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();  // key list, query maxima and barriers ready
  // Producer (key_in, half) owns dims 256 half .. +255 of key key_in of every tile: blocks
  // 4 half .. 4 half + 3, dequantised from the key half's raw bytes loaded into registers.
  const int key_in = tid & (AM_TILE - 1), half = (tid >> 7) & 1;
  uint4 cur[16];
  auto load_tile = [&](int t) {
    const int jl = t * AM_TILE + key_in;
    const bool own = own_token && key0 + jl == nk - 1;
    load_key_half(p, slot[jl], key0 + jl < nks, own ? new_codes : nullptr, half, cur);
  };
  if (producer) store_query_fp16<RG>(qraw, qmx, qinv, smem + SM_Q);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t stg = smem_u32(smem + SM_STG);
  bool aborted = false;
  // Write tile t's four blocks of this producer (use u of the block buffers): wait until the
  // tensor core has consumed use u - 1, dequantise, publish.
  auto produce_tile = [&](int t, const uint4 (&rr)[16], int u) -> bool {
    const int jl = t * AM_TILE + key_in;
    const bool sparse = key0 + jl < nks, valid = slot[jl] >= 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int blk = 4 * half + c;
      if (u > 0 && !mbar_wait_bounded(&mma_done[blk], (u - 1) & 1, abort_flag, AM_WAIT_NS)) return false;
      dequant_block(rr, sparse, valid, c, key_in, smem + SM_STG + blk * AM_STAGE);
      fence_proxy_async_smem();
      mbar_arrive(&full[blk]);
    }
    return true;
  };
  // Every tile in turn (uses u0 + t).
  auto produce_all = [&](int u0) -> bool {
    for (int t = 0; t < ntiles; ++t) {
      load_tile(t);
      if (!produce_tile(t, cur, u0 + t)) return false;
    }
    return true;
  };

  // ---------------------------------------------------------------- phase 1: S^T = K Q^T
  // Issuer: per tile, one 4-step MMA group per block as soon as it is published (the two
  // halves' blocks in the order they are written).
  if (producer) {
    aborted = !produce_all(0);
  } else if (issuer) {
    constexpr uint32_t id = idesc_f16(AM_TILE, RG, false, false);
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) {
      for (int i = 0; i < AM_BLOCKS; ++i) {
        const int blk = (i & 1) * 4 + (i >> 1);
        if (!(ok = mbar_wait_bounded(&full[blk], t & 1, abort_flag, AM_WAIT_NS))) break;
        tc_fence_after();
        const uint32_t a0 = stg + blk * AM_STAGE, b0 = smem_u32(smem + SM_Q + blk * (RG * 128));
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)
          tc_mma_f16(tmem + t * RG, smem_desc(a0 + 32 * k4, 16, 1024, LAYOUT_SWIZZLE_128B),
                     smem_desc(b0 + 32 * k4, 16, 1024, LAYOUT_SWIZZLE_128B), id, i > 0 || k4 > 0);
        tc_commit(&mma_done[blk]);
      }
    }
    tc_commit(phase_done);
  }
  {
    const bool ok = mbar_wait_bounded(phase_done, 0, abort_flag, AM_WAIT_NS);
    if (__syncthreads_or(!ok || aborted)) aborted = true;
  }
  tc_fence_after();

  // ---------------------------------------------------------------- phase 2: softmax over all keys
  // The 8 producer warps: warp w reads keys 32 (w % 4) .. + 31 of every tile (its TMEM lanes) for
  // heads 32 (w / 4) .. + 31; the four warps of each head half reduce through shared memory.
  if (!aborted && warp < 8) {
    const int q4 = warp & 3, hb = 32 * (warp >> 2);
    float mx[32];
#pragma unroll
    for (int h = 0; h < 32; ++h) mx[h] = -INFINITY;
    for (int t = 0; t < ntiles; ++t) {
      const int key = t * AM_TILE + 32 * q4 + lane;
      uint32_t r0[16], r1[16];
      const uint32_t ta = tmem + (uint32_t(32 * q4) << 16) + t * RG + hb;
      tc_ld_32x32b_x16(ta, r0);
      tc_ld_32x32b_x16(ta + 16, r1);
      tc_wait_ld();
      if (slot[key] >= 0) {
        const float m = mu[key];
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          mx[h] = fmaxf(mx[h], m * __uint_as_float(r0[h]));
          mx[16 + h] = fmaxf(mx[16 + h], m * __uint_as_float(r1[h]));
        }
      }
    }
    red[warp * 32 + lane] = reduce_scatter32<true>(mx);
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (q4 == 0) {  // the maxima of the prescaled logits, scaled back by 2^-s (exact)
      const float *rg = red + warp * 32;
      hmax[hb + lane] = fmaxf(fmaxf(rg[lane], rg[32 + lane]), fmaxf(rg[64 + lane], rg[96 + lane])) * qinv[hb + lane];
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    float sm[32];  // the head maxima are read from shared memory (a broadcast) as needed
#pragma unroll
    for (int h = 0; h < 32; ++h) sm[h] = 0.f;
    const float *m_h = hmax + hb, *qi = qinv + hb;
    for (int t = 0; t < ntiles; ++t) {
      const int key = t * AM_TILE + 32 * q4 + lane;
      uint32_t r0[16], r1[16];
      const uint32_t ta = tmem + (uint32_t(32 * q4) << 16) + t * RG + hb;
      tc_ld_32x32b_x16(ta, r0);
      tc_ld_32x32b_x16(ta + 16, r1);
      tc_wait_ld();
      const bool valid = slot[key] >= 0;
      const float m = mu[key], pm = pv[key];
      uint32_t ph[16];
#pragma unroll
      for (int h = 0; h < 32; h += 2) {
        const float x0 = (m * __uint_as_float(h < 16 ? r0[h] : r1[h - 16])) * qi[h];
        const float x1 = (m * __uint_as_float(h + 1 < 16 ? r0[h + 1] : r1[h - 15])) * qi[h + 1];
        const float e0 = (valid && m_h[h] != -INFINITY) ? __expf(x0 - m_h[h]) : 0.f;
        const float e1 = (valid && m_h[h + 1] != -INFINITY) ? __expf(x1 - m_h[h + 1]) : 0.f;
        sm[h] += e0;
        sm[h + 1] += e1;
        const __half2 hp = __floats2half2_rn(e0 * pm, e1 * pm);
        ph[h >> 1] = *reinterpret_cast<const uint32_t *>(&hp);
      }
      // P^T row of this key: RG heads x 2 B = 128 B, 128-byte swizzle (MN-major B operand)
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<uint4 *>(smem + SM_P + kmaj128(key, hb / 8 + u)) =
            make_uint4(ph[4 * u], ph[4 * u + 1], ph[4 * u + 2], ph[4 * u + 3]);
    }
    red[warp * 32 + lane] = reduce_scatter32<false>(sm);
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (q4 == 0) {
      const float *rg = red + warp * 32;
      hsum[hb + lane] = (rg[lane] + rg[32 + lane]) + (rg[64 + lane] + rg[96 + lane]);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---------------------------------------------------------------- phase 3: O^T = V^T P^T
  // The same blocks serve as the MN-major V^T operand (two blocks = 128 dims, 16 KB apart).
  // A CTA with one tile still holds it from phase 1; otherwise every tile is dequantised again
  // (uses ntiles + t).  Issuer: O^T accumulates over the tiles' 64-key halves.
  const int nkc = ntiles * 2;  // 64-key chunks (masked keys carry P = 0, V = 0)
  if (!aborted && producer) {
    if (ntiles > 1) aborted = !produce_all(ntiles);
  } else if (!aborted && issuer) {
    constexpr uint32_t id = idesc_f16(AM_TILE, RG, true, true);
    const uint32_t pt = smem_u32(smem + SM_P);
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) {
      const int u = ntiles + t;
      for (int dd = 0; dd < 4; ++dd) {
        const int d = (dd & 1) * 2 + (dd >> 1);  // blocks (0,1), (4,5), (2,3), (6,7): the order they are written
        if (ntiles > 1) {
          if (!(ok = mbar_wait_bounded(&full[2 * d], u & 1, abort_flag, AM_WAIT_NS))) break;
          if (!(ok = mbar_wait_bounded(&full[2 * d + 1], u & 1, abort_flag, AM_WAIT_NS))) break;
        }
        tc_fence_after();
#pragma unroll
        for (int jc = 0; jc < 2; ++jc)
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            tc_mma_f16(tmem + d * RG,
                       smem_desc(stg + (2 * d) * AM_STAGE + jc * 8192 + 2048 * k4, 16384, 1024, LAYOUT_SWIZZLE_128B),
                       smem_desc(pt + (8 * (2 * t + jc) + 2 * k4) * 1024, 16, 1024, LAYOUT_SWIZZLE_128B), id,
                       t > 0 || jc > 0 || k4 > 0);
        tc_commit(&mma_done[2 * d]);
        tc_commit(&mma_done[2 * d + 1]);
      }
    }
  }
  if (issuer) tc_commit(phase_done);
  {
    const bool ok = aborted ? false : mbar_wait_bounded(phase_done, 1, abort_flag, AM_WAIT_NS);
    if (__syncthreads_or(!ok || aborted)) aborted = true;
  }
  tc_fence_after();

  // ---------------------------------------------------------------- phase 4: normalise and store
  if constexpr (CS == 1) {
    if (warp < 8) {  // warp w: dims 32 (w % 4) + .. of each 128-dim block, heads 32 (w / 4) .. + 31
      const int q4 = warp & 3, hb = 32 * (warp >> 2);
      float inv[32];
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        const float s = aborted ? 0.f : hsum[hb + h];
        inv[h] = s > 0.f ? 1.f / s : 0.f;
      }
      float *orow = p.o + (int64_t(row) * H + hg * RG + hb) * D;
      for (int d = 0; d < 4; ++d) {
        uint32_t r0[16], r1[16];
        if (!aborted && nkc > 0) {
          const uint32_t ta = tmem + (uint32_t(32 * q4) << 16) + d * RG + hb;
          tc_ld_32x32b_x16(ta, r0);
          tc_ld_32x32b_x16(ta + 16, r1);
          tc_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) r0[i] = r1[i] = 0u;
        }
        const int dim = 128 * d + 32 * q4 + lane;
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          orow[h * D + dim] = __uint_as_float(r0[h]) * inv[h];
          orow[(16 + h) * D + dim] = __uint_as_float(r1[h]) * inv[16 + h];
        }
      }
      if (q4 == 0) {
        const float s = aborted ? 0.f : hsum[hb + lane];
        p.lse[int64_t(row) * H + hg * RG + hb + lane] = s > 0.f ? hmax[hb + lane] + logf(s) : -INFINITY;
      }
    }
  } else {
    combine_partials<CS, RG>(p, tmem, aborted, nkc > 0, reinterpret_cast<float *>(smem + SM_P), red, hmax, hsum, row,
                             hg, split);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == AM_PRODUCERS / 32) {
    tc_fence_after();
    tmem_dealloc(tmem, RG_TMEM_COLS);
  }
  if (tid == 0 && aborted) report(p.err, CSA2_ERR_TIMEOUT);
}

// ---------------------------------------------------------------------------
// Single-tile form (a cluster of CS CTAs, one 128-key tile each): every key is
// dequantised once, straight from its loads into a 128 KB fp16 tile laid out as
// 8 blocks of 64 dims x 128 keys (128-byte swizzle).  The same bytes are the
// K-major A operand of S^T = K Q^T (one block per 64-dim step) and the MN-major
// A operand of O^T = V^T P^T (two blocks per 128-dim step, 16 KB apart), so the
// second product needs no producer work at all.
namespace {
constexpr int T_Q = 0;                          // Q (32 KB); P^T once S^T is complete
constexpr int T_KT = T_Q + 8 * 4096;            // fp16 key tile (128 KB); the partial O afterwards
constexpr int T_SLOT = T_KT + 8 * 16384;
constexpr int T_MU = T_SLOT + AM_TILE * 8;
constexpr int T_PV = T_MU + AM_TILE * 4;
constexpr int T_RED = T_PV + AM_TILE * 4;
constexpr int T_HM = T_RED + 8 * 32 * 4;
constexpr int T_QS = T_HM + 2 * 32 * 4;         // query prescale (as SM_QS)
constexpr int T_NEW = T_QS + (8 * AM_QU + 32) * 4;   // this step's window token (as SM_NEW)
constexpr int T_BAR = T_NEW + 512 + 32;         // qfull, phase_done
constexpr int T_MISC = T_BAR + 8 * 2;
constexpr size_t T_SMEM = T_MISC + 16 + 1024;
}  // namespace

template <int CS>
__global__ void __launch_bounds__(AM_THREADS, 1) attn_tile_kernel(AttnArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int64_t *slot = reinterpret_cast<int64_t *>(smem + T_SLOT);
  float *mu = reinterpret_cast<float *>(smem + T_MU);
  float *pv = reinterpret_cast<float *>(smem + T_PV);
  float *red = reinterpret_cast<float *>(smem + T_RED);
  float *hmax = reinterpret_cast<float *>(smem + T_HM);
  float *hsum = hmax + 32;
  uint64_t *qfull = reinterpret_cast<uint64_t *>(smem + T_BAR);  // Q and the whole tile written (256)
  uint64_t *phase_done = qfull + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + T_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + T_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = tid < AM_PRODUCERS, issuer = tid == AM_PRODUCERS;
  const int row = blockIdx.x, hg = blockIdx.y;
  const int split = int(cg::this_cluster().block_rank());
  const int lrow = row, b = row / p.Q, ring = b;   // the row's sequence b owns SWA ring b
  // The query block (an input of the call) is loaded first; everything else may be written by
  // the kernel launched just before this one, so it is read after grid_dep_wait().
  uint4 qraw[AM_QU];
  if (producer) {
    const uint16_t *qrow = p.q + (int64_t(row) * H + hg * AM_HG) * D;
#pragma unroll
    for (int u = 0; u < AM_QU; ++u) {
      const int it = tid + u * AM_PRODUCERS;
      qraw[u] = *reinterpret_cast<const uint4 *>(qrow + (it / (D / 8)) * D + (it % (D / 8)) * 8);
    }
  }
  const uint2 tok = load_new_token(p, row);  // this step's window token (an input too)
  grid_dep_launch();
  grid_dep_wait();
  // this thread's listed entry is fetched together with the row's position (not after it)
  const int key_in = tid & (AM_TILE - 1), half = (tid >> 7) & 1;
  const int j = split * AM_TILE + key_in;
  const int n_listed = (producer && p.idx && !p.dense && j < p.k) ? p.idx[int64_t(lrow) * p.k + j] : -1;
  const int pos = p.q_pos[row];
  const int nvis = (p.idx || p.dense) ? visible_entries(p.c, b, pos) : 0;
  const int nks = p.dense ? max(0, min(p.e1, nvis) - p.e0) : (p.idx ? p.k : 0);
  int lo = 0, nkw = 0;
  if (p.codes && pos >= 0) {
    lo = max(0, pos - p.window + 1);
    nkw = pos - lo + 1;
  }
  const int nk = nks + nkw;
  if (tid == 0 && p.dense && nvis > p.n_bound) report(p.err, CSA2_ERR_SHAPE);
  uint32_t *qmx = reinterpret_cast<uint32_t *>(smem + T_QS);
  float *qinv = reinterpret_cast<float *>(smem + T_QS + 8 * AM_QU * 4);
  // this step's own window token (the row's last key), quantised here and stored by one CTA
  const bool own_token = p.swa_new && nkw > 0;
  const uint8_t *new_codes = smem + T_NEW;
  float *new_scale = reinterpret_cast<float *>(smem + T_NEW + 512);

  // ---------------------------------------------------------------- loads
  // Producer t: key t % 128, dims 256 (t / 128) .. +255.  The query block's loads go
  // out first, then the key's index, then its raw bytes, all before any barrier; this step's
  // own window token is quantised while they are in flight, and its key loaded after that.
  uint4 rr[16];  // listed entry: rr[0..7] = 128 code bytes, rr[8] = 16 scale bytes; window: 256 codes
  bool sparse = false;
  int64_t s = -1;
  if (producer) {
    float m = 0.f, pm = 0.f;
    if (j < nks) {
      sparse = true;
      const int n = p.dense ? p.e0 + j : n_listed;
      if (n != -1) {
        if (n < -1 || n >= nvis) {
          if (half == 0) report(p.err, CSA2_ERR_INDEX);
        } else {
          s = cache_slot(p.c, b, n);
          if (s < 0 && half == 0) report(p.err, CSA2_ERR_INDEX);
        }
      }
      m = p.tau, pm = 1.f;
      load_key_half(p, s, true, nullptr, half, rr);
    } else if (j < nk) {
      s = int64_t(ring) * p.R + (lo + (j - nks)) % p.R;
      if (!(own_token && j == nk - 1)) {
        const float sc = p.scale[s];
        m = p.tau * sc, pm = sc;
        load_key_half(p, s, false, nullptr, half, rr);
      }
    }
    if (half == 0) {
      slot[key_in] = s;
      mu[key_in] = m;
      pv[key_in] = pm;
    }
    publish_query_max(qraw, qmx);  // after the key loads are out
  }
  // Only the CTAs holding this step's own token (the row's last key) quantise it; the first
  // head group's stores it in the ring.
  if (own_token && split == (nk - 1) / AM_TILE) {
    quantise_new_token(p, tok, ring, pos, hg == 0, smem + T_NEW, new_scale, new_scale + 4);
    if (producer && j == nk - 1) {
      const float sc = *new_scale;
      load_key_half(p, s, false, new_codes, half, rr);
      if (half == 0) {
        mu[key_in] = p.tau * sc;
        pv[key_in] = sc;
      }
    }
  }
  // Each key half is dequantised into the tile as soon as its bytes are in, before the
  // prologue barrier (the tile is not otherwise used yet); its blocks are published to the
  // issuer after the barrier.
  if (producer)
#pragma unroll
    for (int c = 0; c < 4; ++c) dequant_block(rr, sparse, s >= 0, c, key_in, smem + T_KT + (4 * half + c) * 16384);
  if (warp == AM_PRODUCERS / 32) {
    tmem_alloc(tmem_slot, AM_TMEM_COLS);
    tmem_relinquish();
  }
  if (issuer) {
    mbar_init(qfull, AM_PRODUCERS);
    mbar_init(phase_done, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  tc_fence_before();
  __syncthreads();  // barriers, key list, query maxima and TMEM address ready
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool aborted = false;

  // ---------------------------------------------------------------- phase 1: S^T = K Q^T
  if (producer) {
    store_query_fp16(qraw, qmx, qinv, smem + T_Q);
    fence_proxy_async_smem();  // the query and this thread's key blocks, written before
    mbar_arrive(qfull);        // the whole tile and the query are in place once all have arrived
  } else if (issuer) {
    constexpr uint32_t id = idesc_f16(AM_TILE, AM_HG, false, false);
    if (mbar_wait_bounded(qfull, 0, abort_flag, AM_WAIT_NS)) {
      tc_fence_after();
      for (int blk = 0; blk < 8; ++blk) {
        const uint32_t a0 = smem_u32(smem + T_KT + blk * 16384), b0 = smem_u32(smem + T_Q + blk * 4096);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)
          tc_mma_f16(tmem, smem_desc(a0 + 32 * k4, 16, 1024, LAYOUT_SWIZZLE_128B),
                     smem_desc(b0 + 32 * k4, 16, 1024, LAYOUT_SWIZZLE_128B), id, blk > 0 || k4 > 0);
      }
    }
    tc_commit(phase_done);
  }
  {
    const bool ok = mbar_wait_bounded(phase_done, 0, abort_flag, AM_WAIT_NS);
    if (__syncthreads_or(!ok)) aborted = true;
  }
  tc_fence_after();

  // ---------------------------------------------------------------- phase 2: softmax over the tile
  if (!aborted && warp < 4) {
    const int key = 32 * warp + lane;
    uint32_t r0[16], r1[16];
    const uint32_t ta = tmem + (uint32_t(32 * warp) << 16);
    tc_ld_32x32b_x16(ta, r0);
    tc_ld_32x32b_x16(ta + 16, r1);
    tc_wait_ld();
    const bool valid = slot[key] >= 0;
    const float m = mu[key], pm = pv[key];
    float x[32], mx[32];
#pragma unroll
    for (int h = 0; h < 16; ++h) {  // prescaled logits scaled back by 2^-s (exact)
      x[h] = (m * __uint_as_float(r0[h])) * qinv[h];
      x[16 + h] = (m * __uint_as_float(r1[h])) * qinv[16 + h];
    }
#pragma unroll
    for (int h = 0; h < 32; ++h) mx[h] = valid ? x[h] : -INFINITY;
    red[warp * 32 + lane] = reduce_scatter32<true>(mx);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    // every warp forms the 32 head maxima itself (lane l: head l) and shares them by shuffles
    const float mh = fmaxf(fmaxf(red[lane], red[32 + lane]), fmaxf(red[64 + lane], red[96 + lane]));
    if (warp == 0) hmax[lane] = mh;
    float sm[32];
    uint32_t ph[16];
#pragma unroll
    for (int h = 0; h < 32; h += 2) {
      const float m0 = __shfl_sync(0xffffffffu, mh, h), m1 = __shfl_sync(0xffffffffu, mh, h + 1);
      const float e0 = (valid && m0 != -INFINITY) ? __expf(x[h] - m0) : 0.f;
      const float e1 = (valid && m1 != -INFINITY) ? __expf(x[h + 1] - m1) : 0.f;
      sm[h] = e0;
      sm[h + 1] = e1;
      const __half2 hp = __floats2half2_rn(e0 * pm, e1 * pm);
      ph[h >> 1] = *reinterpret_cast<const uint32_t *>(&hp);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      *reinterpret_cast<uint4 *>(smem + T_Q + mnmaj64(key, u)) =
          make_uint4(ph[4 * u], ph[4 * u + 1], ph[4 * u + 2], ph[4 * u + 3]);
    red[128 + warp * 32 + lane] = reduce_scatter32<false>(sm);  // (the maxima above may still be read)
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (!aborted && warp == 0) hsum[lane] = (red[128 + lane] + red[160 + lane]) + (red[192 + lane] + red[224 + lane]);

  // ---------------------------------------------------------------- phase 3: O^T = V^T P^T
  if (!aborted && issuer) {
    constexpr uint32_t id = idesc_f16(AM_TILE, AM_HG, true, true);
    const uint32_t kt = smem_u32(smem + T_KT), pt = smem_u32(smem + T_Q);
    for (int d = 0; d < 4; ++d)
#pragma unroll
      for (int jc = 0; jc < 2; ++jc)
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)
          tc_mma_f16(tmem + d * AM_HG,
                     smem_desc(kt + (2 * d) * 16384 + jc * 8192 + 2048 * k4, 16384, 1024, LAYOUT_SWIZZLE_128B),
                     smem_desc(pt + (8 * jc + 2 * k4) * 512, 16, 512, LAYOUT_SWIZZLE_64B), id, jc > 0 || k4 > 0);
  }
  if (issuer) tc_commit(phase_done);
  {
    const bool ok = aborted ? false : mbar_wait_bounded(phase_done, 1, abort_flag, AM_WAIT_NS);
    if (__syncthreads_or(!ok)) aborted = true;
  }
  tc_fence_after();

  // ---------------------------------------------------------------- phase 4: combine the cluster's partials
  combine_partials<CS>(p, tmem, aborted, true, reinterpret_cast<float *>(smem + T_KT), red, hmax, hsum, row, hg,
                       split);

  tc_fence_before();
  __syncthreads();
  if (warp == AM_PRODUCERS / 32) {
    tc_fence_after();
    tmem_dealloc(tmem, AM_TMEM_COLS);
  }
  if (tid == 0 && aborted) report(p.err, CSA2_ERR_TIMEOUT);
}

template <int CS>
static void launch_tile(const AttnArgs &a, int rows, cudaStream_t st, bool pdl) {
  static bool attr[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr[dev]) {
    cudaFuncSetAttribute(attn_tile_kernel<CS>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(T_SMEM));
    attr[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows, H / AM_HG, CS);
  cfg.blockDim = dim3(AM_THREADS);
  cfg.dynamicSmemBytes = T_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = CS;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl ? 2 : 1;
  cudaLaunchKernelEx(&cfg, attn_tile_kernel<CS>, a);
}

template <int CS>
static void launch_cs(const AttnArgs &a, int rows, cudaStream_t st, bool pdl) {
  static bool attr[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr[dev]) {
    if (CS > 8) cudaFuncSetAttribute(attn_mma_kernel<CS>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaFuncSetAttribute(attn_mma_kernel<CS>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(AM_SMEM));
    attr[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows, H / RG, CS);
  cfg.blockDim = dim3(AM_THREADS);
  cfg.dynamicSmemBytes = AM_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  int n = 0;
  if (CS > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = 1;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = CS;
    ++n;
  }
  if (pdl) {
    at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  cudaLaunchKernelEx(&cfg, attn_mma_kernel<CS>, a);
}

// Clusters of CS attention CTAs the device can hold at once (0: none), per device.
template <int CS>
static int attn_clusters_fit() {
  static int cached[64] = {};  // 0 unknown, -1 none
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    if (CS > 8) cudaFuncSetAttribute(attn_mma_kernel<CS>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaFuncSetAttribute(attn_mma_kernel<CS>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(AM_SMEM));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, CS);
    cfg.blockDim = dim3(AM_THREADS);
    cfg.dynamicSmemBytes = AM_SMEM;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = CS;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    cached[dev] = (cudaOccupancyMaxActiveClusters(&n, attn_mma_kernel<CS>, &cfg) == cudaSuccess && n > 0) ? n : -1;
    cudaGetLastError();
  }
  return cached[dev] > 0 ? cached[dev] : 0;
}

int attn_dense_segment() { return attn_clusters_fit<16>() > 0 ? 8192 : 4096; }

// Up to 64 query rows: a cluster of CTAs (one per 128-key tile, 32 heads each) splits each row's
// keys and combines the partials through distributed shared memory; when those one-tile CTAs would
// need more than one wave, the 64-head general kernel in clusters of three CTAs of one or two
// tiles (measured on 32 rows of 640 keys: 44 us, against 51 us for two-CTA clusters, 55 us for
// five and 53 us for the one-tile kernel).  A CTA holds at most 5
// tiles (640 keys), so longer key sets (dense segments) always use clusters of up to 16 CTAs.
void launch_attn_mma(const uint16_t *q, int B, int Q, const int32_t *q_pos, float tau, const int32_t *idx, int k,
                     bool dense, int e0, int e1, int n_bound, const csa2_cache *c, const uint8_t *codes,
                     const float *scale, int R, int window, float *o, float *lse, int32_t *err, cudaStream_t st,
                     const uint16_t *swa_new, bool pdl) {
  const int rows = B * Q;
  if (rows == 0) return;
  AttnArgs a{};
  a.q = q, a.Q = Q, a.q_pos = q_pos, a.tau = tau;
  a.idx = dense ? nullptr : idx, a.k = (idx && !dense) ? k : 0;
  a.dense = dense ? 1 : 0, a.e0 = e0, a.e1 = e1, a.n_bound = n_bound;
  if (c) a.c = *c;
  a.codes = codes, a.scale = scale, a.R = R, a.window = window, a.swa_new = codes ? swa_new : nullptr;
  a.o = o, a.lse = lse, a.err = err;
  const int nkeys = (dense ? max(0, e1 - e0) : a.k) + (codes ? window : 0);
  const int tiles = (nkeys + AM_TILE - 1) / AM_TILE;
  int cs = rows * (H / AM_HG) <= 128 ? max(1, min(tiles, 5)) : 1;
  // one-tile CTAs of 32 heads that would need several waves: the 64-head kernel in 3-CTA clusters
  const bool many = cs == 5 && rows * (H / AM_HG) * 5 > sm_count();
  if (many) cs = 3;
  if (!many && cs > 1 && cs == tiles) {  // one tile per CTA: the single-dequant form
    switch (cs) {
      case 2: launch_tile<2>(a, rows, st, pdl); return;
      case 3: launch_tile<3>(a, rows, st, pdl); return;
      case 4: launch_tile<4>(a, rows, st, pdl); return;
      default: launch_tile<5>(a, rows, st, pdl); return;
    }
  }
  cs = max(cs, (tiles + 4) / 5);
  if (cs > 5) cs = cs <= 8 ? 8 : (cs <= 12 ? 12 : 16);
  switch (cs) {
    case 2: launch_cs<2>(a, rows, st, pdl); break;
    case 3: launch_cs<3>(a, rows, st, pdl); break;
    case 4: launch_cs<4>(a, rows, st, pdl); break;
    case 5: launch_cs<5>(a, rows, st, pdl); break;
    case 8: launch_cs<8>(a, rows, st, pdl); break;
    case 12: launch_cs<12>(a, rows, st, pdl); break;
    case 16: launch_cs<16>(a, rows, st, pdl); break;
    default: launch_cs<1>(a, rows, st, pdl); break;
  }
}

}  // namespace csa2
