// K5 (cluster form): deterministic top-k of long score rows with a thread-block
// cluster per row.
//
// The CS CTAs of a cluster split the row into contiguous chunks, each CTA into 32
// contiguous warp ranges read with coalesced loads (index order = (CTA, warp,
// iteration, lane)), so ballots give ordered ranks inside a warp.  A sample of the
// keys bounds the larger selection from below; one full pass then histograms the
// keys above the bound and appends them, in order, to per-warp candidate lists in
// shared memory, and every later pass walks only those lists (falling back to the
// scores themselves if the bound was too high or a list overflowed).  Three radix
// passes (key bits 31..20, 19..8, 7..0) build per-CTA histograms in shared memory
// that are summed across the cluster through distributed shared memory: each CTA
// reduces one slice of bins over all peers, then gathers the full sums.  Up to two
// selections (e.g. top-512 and a 16384-entry pool) are refined in the same passes.
// The exact k-th key T and the number of ties to take follow; a counting pass and
// a cluster-wide exclusive prefix give every thread its output offset, and the
// writing pass emits the chosen positions in ascending order (ties: lower position
// first), padded with -1.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.cuh"

namespace cg = cooperative_groups;

namespace csa2 {

namespace {
constexpr int TK_THREADS = 1024;
constexpr int TK_BINS = 4096;
constexpr int TK_CAPW = 256;  // candidate-list capacity per warp

struct Sel {
  int k;
  int32_t *idx;
  float *val;
};

// Threshold search with the whole CTA: the bin at which the count of keys in bins
// at or above it first reaches rem (scanning from the top), the count strictly
// above that bin, and the total.  Thread t owns bins nb-4t-4 .. nb-4t-1.
__device__ void find_bin_block(const uint32_t *h, int nb, uint32_t rem, int *scan_sm, int *out_bin,
                               uint32_t *out_above, uint32_t *out_total) {
  const int t = threadIdx.x;
  uint32_t c[4] = {0, 0, 0, 0}, sum = 0;
  if (4 * t < nb) {
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = h[nb - 4 * t - 1 - i], sum += c[i];
  }
  int total;
  const uint32_t excl = uint32_t(block_exclusive_scan_1024(int(sum), scan_sm, &total));
  if (t == 0) *out_total = uint32_t(total);
  if (excl < rem && excl + sum >= rem) {
    uint32_t cum = excl;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (cum + c[i] >= rem) {
        *out_bin = nb - 4 * t - 1 - i;
        *out_above = cum;
        break;
      }
      cum += c[i];
    }
  }
  __syncthreads();
}

// Sum the per-CTA histograms [nh][nb] across the cluster (each CTA reduces one
// slice of bins over all peers, then gathers every slice).
template <int CS>
__device__ __forceinline__ void cluster_hist_sum(cg::cluster_group &cluster, uint32_t (*hist)[TK_BINS],
                                                 uint32_t (*red)[TK_BINS / CS], int nh, int nb, int r) {
  if constexpr (CS > 1) {
    cluster.sync();
    const int slice = nb / CS;
    for (int h = 0; h < nh; ++h)
      for (int i = threadIdx.x; i < slice; i += TK_THREADS) {
        uint32_t t = 0;
#pragma unroll
        for (int p = 0; p < CS; ++p) t += cluster.map_shared_rank(&hist[h][0], p)[r * slice + i];
        red[h][i] = t;
      }
    cluster.sync();
    for (int h = 0; h < nh; ++h)
      for (int i = threadIdx.x; i < nb; i += TK_THREADS)
        hist[h][i] = cluster.map_shared_rank(&red[h][0], i / slice)[i % slice];
    cluster.sync();  // peers finished reading my red[] before it is rewritten
  } else {
    __syncthreads();
  }
}
}  // namespace

template <int CS>
__global__ void __launch_bounds__(TK_THREADS, 1) topk_cluster_kernel(const float *__restrict__ scores,
                                                                     const int32_t *__restrict__ n_valid, int N,
                                                                     Sel s0, Sel s1, int nsel,
                                                                     const int32_t *__restrict__ map) {
  constexpr int U = 4;        // loads in flight per lane
  constexpr int SAMPLE = 16;  // one group of 32 keys in SAMPLE is sampled
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ uint32_t tk_smem[];
  uint32_t(*hist)[TK_BINS] = reinterpret_cast<uint32_t(*)[TK_BINS]>(tk_smem);                         // [2][bins]
  uint32_t(*red)[TK_BINS / CS] = reinterpret_cast<uint32_t(*)[TK_BINS / CS]>(tk_smem + 2 * TK_BINS);  // [2][slice]
  uint32_t(*ckey)[TK_CAPW] =
      reinterpret_cast<uint32_t(*)[TK_CAPW]>(tk_smem + 2 * TK_BINS + (CS > 1 ? 2 * TK_BINS / CS : 0));  // [32][cap]
  int32_t(*cidx)[TK_CAPW] = reinterpret_cast<int32_t(*)[TK_CAPW]>(&ckey[32][0]);                        // [32][cap]
  __shared__ int scan_sm[32];
  __shared__ uint32_t prefix_s[2], rem_s[2];
  __shared__ int all_s[2], bin_s[2];
  __shared__ uint32_t above_s[2], total_s[2];
  __shared__ int cta_tot[2][2];  // per selection: count above T, count equal to T
  __shared__ int overflow_s;

  const int r = int(cluster.block_rank());
  const int row = blockIdx.x / CS;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = n_valid ? max(0, min(N, n_valid[row])) : N;
  const float *srow = scores + int64_t(row) * N;
  // CTA chunk, then one contiguous range per warp; lane l reads elements base + 32 u + l
  const int chunk = (n + CS - 1) / CS;
  const int c0 = min(n, r * chunk), c1 = min(n, c0 + chunk);
  const int wsub = (c1 - c0 + 31) / 32;
  const int wb = min(c1, c0 + warp * wsub), we = min(c1, wb + wsub);
  const uint32_t lt_mask = (1u << lane) - 1u;
  const Sel sel[2] = {s0, s1};
  const int kbig = nsel > 1 ? max(s0.k, s1.k) : s0.k;

  auto zero_hist = [&]() {
    for (int i = tid; i < 2 * TK_BINS; i += TK_THREADS) (&hist[0][0])[i] = 0;
    __syncthreads();
  };
  // One pass over the warp's range: warp-aggregated histogram of the top 12 key bits
  // for keys whose bin >= lo_bin; with `keep`, those keys are also appended, in index
  // order, to the warp's candidate list (cnt counts them even past the capacity).
  int cnt = 0;
  auto top_pass = [&](int step, int lo_bin, bool keep) {
    for (int base = wb; base < we; base += 32 * U * step) {
      float v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = base + 32 * u * step + lane;
        v[u] = j < we ? srow[j] : -INFINITY;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t key = score_key(v[u]);
        const int bin = int(key >> 20);
        const bool take = key != KEY_NEG_INF && bin >= lo_bin;
        const uint32_t m = __ballot_sync(0xffffffffu, take);
        if (m) {
          const uint32_t peers = __match_any_sync(0xffffffffu, take ? uint32_t(bin) : 0xFFFFFFFFu);
          if (take && (peers & lt_mask) == 0) atomicAdd(&hist[0][bin], uint32_t(__popc(peers)));
          if (keep) {
            const int at = cnt + __popc(m & lt_mask);
            if (take && at < TK_CAPW) {
              ckey[warp][at] = key;
              cidx[warp][at] = base + 32 * u * step + lane;
            }
            cnt += __popc(m);
          }
        }
      }
    }
  };
  // Visit the warp's keys in index order, 32 per step (lane = position in the step):
  // from its candidate list (fast) or from the scores themselves.  f(key, index, valid).
  auto walk = [&](bool fast, auto &&f) {
    if (fast) {
      const int m = min(cnt, TK_CAPW);
      for (int b0 = 0; b0 < m; b0 += 32) {
        const int i = b0 + lane;
        const bool v = i < m;
        f(v ? ckey[warp][i] : KEY_NEG_INF, v ? cidx[warp][i] : 0, v);
      }
    } else {
      for (int base = wb; base < we; base += 32 * U) {
        float vv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int j = base + 32 * u + lane;
          vv[u] = j < we ? srow[j] : -INFINITY;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const uint32_t key = score_key(vv[u]);
          f(key, base + 32 * u + lane, key != KEY_NEG_INF);
        }
      }
    }
  };

  // ---- sampled lower bound: keys below it cannot reach the larger selection (checked below)
  const uint32_t target = uint32_t(kbig / SAMPLE) + uint32_t(kbig / (2 * SAMPLE)) + 32;
  zero_hist();
  top_pass(SAMPLE, 0, false);
  cluster_hist_sum<CS>(cluster, hist, red, 1, TK_BINS, r);
  if (tid == 0) bin_s[0] = 0;
  find_bin_block(hist[0], TK_BINS, target, scan_sm, &bin_s[0], &above_s[0], &total_s[0]);
  int lo_bin = total_s[0] >= target ? bin_s[0] : 0;

  if (tid < 2) {
    prefix_s[tid] = 0;
    rem_s[tid] = uint32_t(sel[tid].k);
    all_s[tid] = 0;
  }
  // ---- pass 0 (top 12 bits) over keys at or above the bound, keeping them as candidates
  zero_hist();
  if (tid == 0) overflow_s = 0;
  __syncthreads();
  top_pass(1, lo_bin, true);
  if (lane == 0 && cnt > TK_CAPW) atomicOr(&overflow_s, 1);
  cluster_hist_sum<CS>(cluster, hist, red, 1, TK_BINS, r);
  find_bin_block(hist[0], TK_BINS, 1u, scan_sm, &bin_s[1], &above_s[1], &total_s[1]);  // for the total
  int any_overflow = 0;
  for (int q = 0; q < CS; ++q) any_overflow |= *cluster.map_shared_rank(&overflow_s, q);
  bool fast = !any_overflow && (total_s[1] >= uint32_t(kbig) || lo_bin == 0);
  if (!fast) {  // the bound was too high or a list overflowed: count every key from the scores
    lo_bin = 0;
    zero_hist();
    top_pass(1, 0, false);
    cluster_hist_sum<CS>(cluster, hist, red, 1, TK_BINS, r);
    find_bin_block(hist[0], TK_BINS, 1u, scan_sm, &bin_s[1], &above_s[1], &total_s[1]);
  }
  cluster.sync();  // peers have read overflow_s
  const uint32_t counted = total_s[1];
  if (nsel > 1) {
    for (int i = tid; i < TK_BINS; i += TK_THREADS) hist[1][i] = hist[0][i];
  }
  __syncthreads();
  for (int s = 0; s < nsel; ++s) {
    // with the bound in place fewer than all keys are counted, but then at least kbig are
    if (lo_bin == 0 && counted <= uint32_t(sel[s].k)) {
      if (tid == 0) all_s[s] = 1;
      __syncthreads();
      continue;
    }
    find_bin_block(hist[s], TK_BINS, rem_s[s], scan_sm, &bin_s[s], &above_s[s], &total_s[s]);
    if (tid == 0) {
      rem_s[s] -= above_s[s];
      prefix_s[s] = uint32_t(bin_s[s]);
    }
    __syncthreads();
  }

  // ---- passes 1, 2 (bits 19..8, 7..0) over keys matching each selection's prefix
  for (int pass = 1; pass < 3; ++pass) {
    const int width = pass == 2 ? 8 : 12;
    const int sh = pass == 1 ? 8 : 0, nb = 1 << width;
    const uint32_t mask = uint32_t(nb - 1);
    zero_hist();
    const uint32_t pre0 = prefix_s[0], pre1 = prefix_s[1];
    const bool act0 = !all_s[0], act1 = nsel > 1 && !all_s[1];
    if (act0 || act1) {
      walk(fast, [&](uint32_t key, int, bool valid) {
        if (!valid) return;
        const uint32_t hi = key >> (sh + width), bin = (key >> sh) & mask;
        if (act0 && hi == pre0) atomicAdd(&hist[0][bin], 1u);
        if (act1 && hi == pre1) atomicAdd(&hist[1][bin], 1u);
      });
    }
    cluster_hist_sum<CS>(cluster, hist, red, nsel, nb, r);
    for (int s = 0; s < nsel; ++s) {
      if (all_s[s]) continue;
      find_bin_block(hist[s], nb, rem_s[s], scan_sm, &bin_s[s], &above_s[s], &total_s[s]);
      if (tid == 0) {
        rem_s[s] -= above_s[s];
        prefix_s[s] = (prefix_s[s] << width) | uint32_t(bin_s[s]);
      }
      __syncthreads();
    }
  }

  // ---- per-warp counts of keys above / equal to T (warp-uniform via ballots)
  uint32_t T[2];
  int need[2], gt_w[2] = {0, 0}, eq_w[2] = {0, 0};
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    T[s] = all_s[s] ? KEY_NEG_INF : prefix_s[s];
    need[s] = all_s[s] ? 0 : int(rem_s[s]);
  }
  walk(fast, [&](uint32_t key, int, bool valid) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (s >= nsel) break;
      gt_w[s] += __popc(__ballot_sync(0xffffffffu, valid && key > T[s]));
      eq_w[s] += __popc(__ballot_sync(0xffffffffu, valid && key == T[s]));
    }
  });
  // ---- exclusive prefix over (cluster rank, warp)
  int gt_off[2] = {0, 0}, eq_off[2] = {0, 0};
  for (int s = 0; s < nsel; ++s) {
    int tot;
    gt_off[s] = block_exclusive_scan_1024(lane == 0 ? gt_w[s] : 0, scan_sm, &tot);
    gt_off[s] = __shfl_sync(0xffffffffu, gt_off[s], 0);
    if (tid == 0) cta_tot[s][0] = tot;
    eq_off[s] = block_exclusive_scan_1024(lane == 0 ? eq_w[s] : 0, scan_sm, &tot);
    eq_off[s] = __shfl_sync(0xffffffffu, eq_off[s], 0);
    if (tid == 0) cta_tot[s][1] = tot;
  }
  cluster.sync();
  int selected[2] = {0, 0};
  for (int s = 0; s < nsel; ++s) {
    int gb = 0, eb = 0, gall = 0, eall = 0;
    for (int p = 0; p < CS; ++p) {
      const int *pt = cluster.map_shared_rank(&cta_tot[s][0], p);
      if (p < r) gb += pt[0], eb += pt[1];
      gall += pt[0], eall += pt[1];
    }
    gt_off[s] += gb;
    eq_off[s] += eb;
    selected[s] = gall + min(eall, need[s]);
  }
  cluster.sync();  // every peer has read cta_tot before any CTA exits

  // ---- write the chosen positions in ascending order
  for (int s = 0; s < nsel; ++s) {
    const int k = sel[s].k, nd = need[s];
    const uint32_t Ts = T[s];
    int32_t *orow = sel[s].idx + int64_t(row) * k;
    float *vrow = sel[s].val ? sel[s].val + int64_t(row) * k : nullptr;
    const int32_t *mrow = map ? map + int64_t(row) * N : nullptr;
    int g = gt_off[s], e = eq_off[s];
    walk(fast, [&](uint32_t key, int j, bool valid) {
      const bool is_gt = valid && key > Ts, is_eq = valid && key == Ts;
      const uint32_t gm = __ballot_sync(0xffffffffu, is_gt), em = __ballot_sync(0xffffffffu, is_eq);
      const int gbef = g + __popc(gm & lt_mask), ebef = e + __popc(em & lt_mask);
      const int at = is_gt ? gbef + min(ebef, nd) : ((is_eq && ebef < nd) ? gbef + ebef : -1);
      if (at >= 0 && at < k) {
        orow[at] = mrow ? mrow[j] : j;
        if (vrow) vrow[at] = key_score(key);
      }
      g += __popc(gm);
      e += __popc(em);
    });
    if (r == 0)
      for (int i = selected[s] + tid; i < k; i += TK_THREADS) {
        orow[i] = -1;
        if (vrow) vrow[i] = -INFINITY;
      }
  }
}

static size_t tk_smem_bytes(int cs) {
  return sizeof(uint32_t) * (2 * TK_BINS + (cs > 1 ? 2 * TK_BINS / cs : 0) + 2 * 32 * TK_CAPW);
}

template <int CS>
static cudaError_t launch_cs(const float *scores, const int32_t *n_valid, int R, int N, Sel s0, Sel s1, int nsel,
                             const int32_t *map, cudaStream_t st) {
  static bool attr[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr[dev]) {
    if (CS > 8) cudaFuncSetAttribute(topk_cluster_kernel<CS>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaFuncSetAttribute(topk_cluster_kernel<CS>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(tk_smem_bytes(CS)));
    attr[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(R * CS);
  cfg.blockDim = dim3(TK_THREADS);
  cfg.dynamicSmemBytes = tk_smem_bytes(CS);
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CS;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel<CS>, scores, n_valid, N, s0, s1, nsel, map);
}

// Cluster size by row length and count: one CTA per row up to 64K scores or from 148 rows
// on; otherwise 8 CTAs up to 256K scores and 16 above.
void launch_topk_cluster(const float *scores, const int32_t *n_valid, int R, int N, int k0, int32_t *idx0, float *val0,
                         int k1, int32_t *idx1, float *val1, const int32_t *map, cudaStream_t st) {
  if (R == 0) return;
  const Sel s0{k0, idx0, val0}, s1{k1, idx1, val1};
  const int nsel = (k1 > 0 && idx1) ? 2 : 1;
  static int cluster16_ok[64] = {};  // 0 unknown, 1 yes, -1 no
  int dev = 0;
  cudaGetDevice(&dev);
  if (N >= (1 << 18) && R < 148) {
    if (dev >= 0 && dev < 64 && cluster16_ok[dev] == 0) {
      cudaFuncSetAttribute(topk_cluster_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16);
      cfg.blockDim = dim3(TK_THREADS);
      cfg.dynamicSmemBytes = tk_smem_bytes(16);
      cudaFuncSetAttribute(topk_cluster_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(tk_smem_bytes(16)));
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 16;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int nclusters = 0;
      cluster16_ok[dev] =
          (cudaOccupancyMaxActiveClusters(&nclusters, topk_cluster_kernel<16>, &cfg) == cudaSuccess && nclusters > 0)
              ? 1
              : -1;
      cudaGetLastError();
    }
    if (cluster16_ok[dev] > 0) {
      launch_cs<16>(scores, n_valid, R, N, s0, s1, nsel, map, st);
      return;
    }
    launch_cs<8>(scores, n_valid, R, N, s0, s1, nsel, map, st);
  } else if (N > (1 << 16) && R < 148) {
    launch_cs<8>(scores, n_valid, R, N, s0, s1, nsel, map, st);
  } else {
    // rows up to 64K scores, or enough rows to fill the GPU: one CTA per row, no cluster barriers
    launch_cs<1>(scores, n_valid, R, N, s0, s1, nsel, map, st);
  }
}

}  // namespace csa2
