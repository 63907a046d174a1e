// K5 (cluster form): deterministic top-k of long score rows with a thread-block
// cluster per row.
//
// The CS CTAs of a cluster split the row into contiguous chunks, each CTA into 32
// contiguous warp ranges read with coalesced loads (index order = (CTA, warp,
// iteration, lane)), so ballots give ordered ranks inside a warp.  Three radix
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

struct Sel {
  int k;
  int32_t *idx;
  float *val;
};

// Highest bin b (scanning down from the top) at which the running count reaches rem:
// returns b and the count strictly above it.  Uses warp 0; result in *out.
__device__ void find_bin(const uint32_t *h, int nbins, uint32_t rem, int *out_bin, uint32_t *out_above) {
  const int lane = threadIdx.x & 31;
  const int per = nbins / 32;
  // lane l covers bins [nbins - per*(l+1), nbins - per*l), scanned top-down
  uint32_t sum = 0;
  for (int i = 0; i < per; ++i) sum += h[nbins - per * lane - 1 - i];
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t excl = incl - sum;
  if (excl < rem && incl >= rem) {
    uint32_t cum = excl;
    for (int i = 0; i < per; ++i) {
      const int bin = nbins - per * lane - 1 - i;
      if (cum + h[bin] >= rem) {
        *out_bin = bin;
        *out_above = cum;
        break;
      }
      cum += h[bin];
    }
  }
}
}  // namespace

template <int CS>
__global__ void __launch_bounds__(TK_THREADS, 1) topk_cluster_kernel(const float *__restrict__ scores,
                                                                     const int32_t *__restrict__ n_valid, int N,
                                                                     Sel s0, Sel s1, int nsel,
                                                                     const int32_t *__restrict__ map) {
  constexpr int U = 4;  // loads in flight per lane
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ uint32_t tk_smem[];
  uint32_t(*hist)[TK_BINS] = reinterpret_cast<uint32_t(*)[TK_BINS]>(tk_smem);                         // [2][bins]
  uint32_t(*red)[TK_BINS / CS] = reinterpret_cast<uint32_t(*)[TK_BINS / CS]>(tk_smem + 2 * TK_BINS);  // [2][slice]
  __shared__ int scan_sm[32];
  __shared__ uint32_t prefix_s[2], rem_s[2];
  __shared__ int all_s[2], bin_s[2];
  __shared__ uint32_t above_s[2];
  __shared__ int cta_tot[2][2];  // per selection: count above T, count equal to T

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

  if (tid < 2) {
    prefix_s[tid] = 0;
    rem_s[tid] = uint32_t(sel[tid].k);
    all_s[tid] = 0;
  }

  for (int pass = 0; pass < 3; ++pass) {
    const int width = pass == 2 ? 8 : 12;
    const int sh = pass == 0 ? 20 : (pass == 1 ? 8 : 0), nb = 1 << width;
    const uint32_t mask = uint32_t(nb - 1);
    const int nh = pass == 0 ? 1 : nsel;  // the first pass is shared by both selections
    for (int i = tid; i < 2 * TK_BINS; i += TK_THREADS) (&hist[0][0])[i] = 0;
    __syncthreads();
    const uint32_t pre0 = prefix_s[0], pre1 = prefix_s[1];
    const bool act0 = !all_s[0], act1 = nsel > 1 && !all_s[1];
    for (int base = wb; base < we; base += 32 * U) {
      float v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = base + 32 * u + lane;
        v[u] = j < we ? srow[j] : -INFINITY;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t key = score_key(v[u]);
        const bool valid = key != KEY_NEG_INF;
        const uint32_t bin = (key >> sh) & mask;
        if (pass == 0) {
          // one atomic per distinct bin in the warp
          const uint32_t peers = __match_any_sync(0xffffffffu, valid ? bin : 0xFFFFFFFFu);
          if (valid && (peers & lt_mask) == 0) atomicAdd(&hist[0][bin], uint32_t(__popc(peers)));
        } else if (valid) {
          const uint32_t hi = key >> (sh + width);
          if (act0 && hi == pre0) atomicAdd(&hist[0][bin], 1u);
          if (act1 && hi == pre1) atomicAdd(&hist[1][bin], 1u);
        }
      }
    }
    // ---- cluster-wide sums: reduce my slice over all peers, then gather every slice
    if constexpr (CS > 1) {
      cluster.sync();
      const int slice = nb / CS;
      for (int h = 0; h < nh; ++h)
        for (int i = tid; i < slice; i += TK_THREADS) {
          uint32_t t = 0;
#pragma unroll
          for (int p = 0; p < CS; ++p) t += cluster.map_shared_rank(&hist[h][0], p)[r * slice + i];
          red[h][i] = t;
        }
      cluster.sync();
      for (int h = 0; h < nh; ++h)
        for (int i = tid; i < nb; i += TK_THREADS) hist[h][i] = cluster.map_shared_rank(&red[h][0], i / slice)[i % slice];
      cluster.sync();  // peers finished reading my red[] before it is rewritten
    }
    if (pass == 0 && nsel > 1) {
      for (int i = tid; i < nb; i += TK_THREADS) hist[1][i] = hist[0][i];
    }
    __syncthreads();
    // ---- threshold bin per selection
    if (tid < 32) {
      for (int s = 0; s < nsel; ++s) {
        if (all_s[s]) continue;
        if (pass == 0) {
          uint32_t tot = 0;
          for (int i = tid; i < nb; i += 32) tot += hist[s][i];
#pragma unroll
          for (int o = 16; o; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
          if (tot <= uint32_t(sel[s].k)) {
            if (tid == 0) all_s[s] = 1;
            continue;
          }
        }
        find_bin(hist[s], nb, rem_s[s], &bin_s[s], &above_s[s]);
        __syncwarp();
        if (tid == 0) {
          rem_s[s] -= above_s[s];
          prefix_s[s] = (prefix_s[s] << width) | uint32_t(bin_s[s]);
        }
        __syncwarp();
      }
    }
    __syncthreads();
  }

  // ---- per-warp counts of keys above / equal to T (warp-uniform via ballots)
  uint32_t T[2];
  int need[2], gt_w[2] = {0, 0}, eq_w[2] = {0, 0};
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    T[s] = all_s[s] ? KEY_NEG_INF : prefix_s[s];
    need[s] = all_s[s] ? 0 : int(rem_s[s]);
  }
  for (int base = wb; base < we; base += 32 * U) {
    float v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = base + 32 * u + lane;
      v[u] = j < we ? srow[j] : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t key = score_key(v[u]);
      const bool valid = key != KEY_NEG_INF;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        if (s >= nsel) break;
        gt_w[s] += __popc(__ballot_sync(0xffffffffu, valid && key > T[s]));
        eq_w[s] += __popc(__ballot_sync(0xffffffffu, valid && key == T[s]));
      }
    }
  }
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
    for (int base = wb; base < we && g + min(e, nd) < k; base += 32 * U) {
      float v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = base + 32 * u + lane;
        v[u] = j < we ? srow[j] : -INFINITY;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t key = score_key(v[u]);
        const bool valid = key != KEY_NEG_INF;
        const bool is_gt = valid && key > Ts, is_eq = valid && key == Ts;
        const uint32_t gm = __ballot_sync(0xffffffffu, is_gt), em = __ballot_sync(0xffffffffu, is_eq);
        const int gbef = g + __popc(gm & lt_mask), ebef = e + __popc(em & lt_mask);
        const int at = is_gt ? gbef + min(ebef, nd) : ((is_eq && ebef < nd) ? gbef + ebef : -1);
        if (at >= 0 && at < k) {
          const int j = base + 32 * u + lane;
          orow[at] = mrow ? mrow[j] : j;
          if (vrow) vrow[at] = v[u];
        }
        g += __popc(gm);
        e += __popc(em);
      }
    }
    if (r == 0)
      for (int i = selected[s] + tid; i < k; i += TK_THREADS) {
        orow[i] = -1;
        if (vrow) vrow[i] = -INFINITY;
      }
  }
}

static size_t tk_smem_bytes(int cs) { return sizeof(uint32_t) * (2 * TK_BINS + (cs > 1 ? 2 * TK_BINS / cs : 0)); }

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

// Largest usable cluster for a row length: about 64K scores per CTA, at most 16.
void launch_topk_cluster(const float *scores, const int32_t *n_valid, int R, int N, int k0, int32_t *idx0, float *val0,
                         int k1, int32_t *idx1, float *val1, const int32_t *map, cudaStream_t st) {
  if (R == 0) return;
  const Sel s0{k0, idx0, val0}, s1{k1, idx1, val1};
  const int nsel = (k1 > 0 && idx1) ? 2 : 1;
  static int cluster16_ok[64] = {};  // 0 unknown, 1 yes, -1 no
  int dev = 0;
  cudaGetDevice(&dev);
  if (N >= (1 << 18)) {
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
  } else if (N >= (1 << 16)) {
    launch_cs<8>(scores, n_valid, R, N, s0, s1, nsel, map, st);
  } else if (N >= (1 << 14)) {
    launch_cs<4>(scores, n_valid, R, N, s0, s1, nsel, map, st);
  } else if (N >= (1 << 12)) {
    launch_cs<2>(scores, n_valid, R, N, s0, s1, nsel, map, st);
  } else {
    launch_cs<1>(scores, n_valid, R, N, s0, s1, nsel, map, st);
  }
}

}  // namespace csa2
