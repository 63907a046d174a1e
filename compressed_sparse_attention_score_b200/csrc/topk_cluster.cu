// K5 (cluster form): deterministic top-k of long score rows with a thread-block
// cluster per row.
//
// The CS CTAs of a cluster split the row into contiguous chunks, each CTA into 32
// contiguous warp ranges read with coalesced loads (index order = (CTA, warp,
// iteration, lane)), so ballots give ordered ranks inside a warp.  The exact k-th
// key T is found by radix selection on the order-preserving 32-bit keys (bits 31..20,
// 19..8, 7..0).  Every stage builds its histogram in the CTA's own shared memory,
// together with a coarse copy (8 bins summed per entry); after one cluster barrier
// each CTA sums the peers' coarse bins through distributed shared memory, finds the
// coarse bin that holds the threshold and then sums only the 8 fine bins inside it,
// so a stage costs one barrier and no CTA ever writes into a histogram a peer reads.
// A sample of the keys first bounds the larger selection from below; the first full
// pass (each lane 16 consecutive keys, one warp scan to place them) counts only keys
// above the bound and appends them, in index order, to per-warp candidate lists, and
// the later passes walk the lists (or the scores again if the bound was too high or a
// list overflowed).  A CTA whose chunk fits in shared memory instead copies it there
// once as keys and every pass reads it there.  Refinement stops as soon as the
// threshold's prefix bin holds exactly the keys still needed.  Up to two selections
// (e.g. top-512 and a 16384-entry pool) are refined in the same passes.  A counting pass and a
// cluster-wide exclusive prefix (each CTA pushes its totals into every peer) give
// every thread its output offset, and the writing pass emits the chosen positions in
// ascending order (ties: lower position first), padded with -1.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace cg = cooperative_groups;

namespace csa2 {

namespace {
constexpr int TK_THREADS = 1024;
constexpr int TK_BINS = 4096;   // 12-bit radix digit
constexpr int TK_CBINS = 512;   // coarse copy: 8 fine bins per entry
constexpr int TK_CAPW = 256;    // candidate-list capacity per warp
// shared-memory words: candidate lists, then sample / pass-0 / pass-1 (x2) / pass-2 (x2)
// histograms with their coarse copies, then the coarse cluster sums
constexpr int TK_LIST_WORDS = 2 * 32 * TK_CAPW;
constexpr int TK_H12_WORDS = TK_BINS + TK_CBINS;
constexpr int TK_H8_WORDS = 256 + 32;
constexpr int TK_SMEM_WORDS = TK_LIST_WORDS + 4 * TK_H12_WORDS + 2 * TK_H8_WORDS + 2 * TK_CBINS;

struct Sel {
  int k;
  int32_t *idx;
  float *val;
};

}  // namespace

template <int CS>
__global__ void __launch_bounds__(TK_THREADS, 1) topk_cluster_kernel(const float *__restrict__ scores,
                                                                     const int32_t *__restrict__ n_valid, int N,
                                                                     Sel s0, Sel s1, int nsel,
                                                                     const int32_t *__restrict__ map) {
  constexpr int U = 8;        // scalar loads in flight per lane
  constexpr int SAMPLE = 16;  // one group of 32 keys in SAMPLE is sampled
  sm100::grid_dep_launch();  // a dependent attention launch may start its prologue
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ uint32_t tk_smem[];
  uint32_t(*ckey)[TK_CAPW] = reinterpret_cast<uint32_t(*)[TK_CAPW]>(tk_smem);        // [32][cap]
  int32_t(*cidx)[TK_CAPW] = reinterpret_cast<int32_t(*)[TK_CAPW]>(&ckey[32][0]);     // [32][cap]
  uint32_t *hs = tk_smem + TK_LIST_WORDS;    // sample histogram (later: pass 0 over every key)
  uint32_t *h0 = hs + TK_H12_WORDS;          // pass 0 over keys above the sampled bound
  uint32_t *h1 = h0 + TK_H12_WORDS;          // pass 1, one per selection
  uint32_t *h2 = h1 + 2 * TK_H12_WORDS;      // pass 2, one per selection
  uint32_t *sumc = h2 + 2 * TK_H8_WORDS;     // [2][TK_CBINS] coarse bins summed over the cluster
  __shared__ int sel_bin[2];
  __shared__ uint32_t sel_above[2], sel_count[2], sel_total[2];
  __shared__ int overflow_s;
  __shared__ int wc[32][4];          // per warp: keys above / equal to T for both selections
  __shared__ int tot_all[2][CS][2];  // per selection and CTA: count above T, count equal to T

  const int r = int(cluster.block_rank());
  const int row = blockIdx.x / CS;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = n_valid ? max(0, min(N, n_valid[row])) : N;
  const float *srow = scores + int64_t(row) * N;
  const bool vec = (N & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0;
  // CTA chunk, then one contiguous range per warp, both multiples of 4 elements
  const int chunk = ((n + CS - 1) / CS + 3) & ~3;
  const int c0 = min(n, r * chunk), c1 = min(n, c0 + chunk);
  const int wsub = ((c1 - c0 + 31) / 32 + 3) & ~3;
  const int wb = min(c1, c0 + warp * wsub), we = min(c1, wb + wsub);
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int kbig = nsel > 1 ? max(s0.k, s1.k) : s0.k;

  auto csync = [&]() {
    if constexpr (CS > 1)
      cluster.sync();
    else
      __syncthreads();
  };
  auto peer = [&](const uint32_t *p, int q) -> const uint32_t * {
    if constexpr (CS > 1)
      return cluster.map_shared_rank(p, q);
    else
      return p;
  };
  // coarse[i] = fine[8i] + ... + fine[8i + 7] for this CTA's histogram (after its updates)
  auto make_coarse = [&](uint32_t *h, int nfine) {
    __syncthreads();
    for (int i = tid; i < nfine / 8; i += TK_THREADS) {
      uint32_t t = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) t += h[8 * i + j];
      h[nfine + i] = t;
    }
  };
  // After a cluster barrier: sumc[s][b] = the cluster's sum of coarse bin b >= lo of the
  // histogram h + s * stride, for each selection s marked active.
  auto sum_coarse = [&](const uint32_t *h, int stride, int nfine, int lo, bool a0, bool a1) {
    const int nc = nfine / 8;
    for (int b = tid; b < 2 * nc; b += TK_THREADS) {
      const int s = b >= nc, c = b - s * nc;
      uint32_t t = 0;
      if ((s ? a1 : a0) && c >= lo) {
        const uint32_t *hc = h + s * stride + nfine;
#pragma unroll
        for (int q = 0; q < CS; ++q) t += peer(hc, q)[c];
      }
      sumc[s * TK_CBINS + c] = t;
    }
    __syncthreads();
  };
  // One warp: the fine bin at which the cluster-wide count from the top first reaches rem,
  // from the coarse sums sc and the peers' fine bins h (nfine/8 coarse bins, 32 | nfine/8).
  // Results in slot s: bin, count above it, its own count and the total (bin -1 when the
  // total stays below rem).  Cluster-uniform, since every CTA sums the same counts.
  auto warp_select = [&](const uint32_t *sc, const uint32_t *h, int nfine, uint32_t rem, int s) {
    const int nc = nfine / 8, per = nc / 32;  // lane 0 owns the top per bins
    uint32_t sum = 0;
    for (int i = 0; i < per; ++i) sum += sc[nc - 1 - lane * per - i];
    uint32_t x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, x, 31);
    if (total < rem) {
      if (lane == 0) sel_bin[s] = -1, sel_total[s] = total;
      return;
    }
    const uint32_t excl = x - sum;
    const int L = __ffs(__ballot_sync(0xffffffffu, excl < rem && x >= rem)) - 1;
    int cb = 0;
    uint32_t cab = 0;
    if (lane == L) {
      uint32_t cum = excl;
      for (int i = 0; i < per; ++i) {
        const uint32_t v = sc[nc - 1 - L * per - i];
        if (cum + v >= rem) {
          cb = nc - 1 - L * per - i;
          cab = cum;
          break;
        }
        cum += v;
      }
    }
    cb = __shfl_sync(0xffffffffu, cb, L);
    cab = __shfl_sync(0xffffffffu, cab, L);
    uint32_t f = 0;  // lanes 0..7: fine bins 8cb+7 .. 8cb of the cluster, from the top
    if (lane < 8) {
#pragma unroll
      for (int q = 0; q < CS; ++q) f += peer(h, q)[8 * cb + 7 - lane];
    }
    uint32_t fx = f;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, fx, o);
      if (lane >= o) fx += y;
    }
    const int F = __ffs(__ballot_sync(0xffffffffu, lane < 8 && cab + fx - f < rem && cab + fx >= rem)) - 1;
    if (lane == F) {
      sel_bin[s] = 8 * cb + 7 - F;
      sel_above[s] = cab + fx - f;
      sel_count[s] = f;
      sel_total[s] = total;
    }
  };

  // Full pass over the warp's range keeping keys at or above lo_bin: their top-12-bit
  // histogram and, in index order, the warp's candidate list.  Four consecutive keys per
  // lane; stops once the list has overflowed (the caller then counts from the scores).
  int cnt = 0;
  // Each lane takes 16 consecutive keys of a 512-key group, so that one warp scan of the
  // lanes' counts places every kept key, in index order, in the warp's list.
  auto keep_pass = [&](int lo_bin, uint32_t *hdst) {
    for (int base = wb; base < we && cnt <= TK_CAPW; base += 512) {
      const int j0 = base + 16 * lane;
      float f[16];
      if (vec && j0 + 15 < we) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 v = *reinterpret_cast<const float4 *>(srow + j0 + 4 * u);
          f[4 * u] = v.x, f[4 * u + 1] = v.y, f[4 * u + 2] = v.z, f[4 * u + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) f[e] = j0 + e < we ? srow[j0 + e] : -INFINITY;
      }
      uint32_t kk[16], tm = 0;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        kk[e] = score_key(f[e]);
        if (kk[e] != KEY_NEG_INF && int(kk[e] >> 20) >= lo_bin) tm |= 1u << e;
      }
      if (!__any_sync(0xffffffffu, tm != 0)) continue;
      const int c = __popc(tm);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int at = cnt + incl - c;
      while (tm) {  // few keys pass the bound: visit only those
        const int e = __ffs(tm) - 1;
        tm &= tm - 1;
        uint32_t key = kk[0];
#pragma unroll
        for (int i = 1; i < 16; ++i) key = e == i ? kk[i] : key;
        atomicAdd(&hdst[key >> 20], 1u);
        if (at < TK_CAPW) {
          ckey[warp][at] = key;
          cidx[warp][at] = j0 + e;
        }
        ++at;
      }
      cnt += __shfl_sync(0xffffffffu, incl, 31);
    }
  };
  // A CTA chunk of at most TK_LIST_WORDS scores is copied once, as keys, into the
  // candidate-list space; every pass then reads shared memory instead of the scores.
  const bool resident = chunk <= TK_LIST_WORDS;  // the same in every CTA of the cluster
  uint32_t *skeys = tk_smem;                      // key of row position j at skeys[j - c0]
  // Keys u = 0 .. U-1 of the group starting at base (lane-strided), -inf past the range.
  auto load_keys = [&](int base, uint32_t (&kk)[U]) {
    if (resident) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = base + 32 * u + lane;
        kk[u] = j < we ? skeys[j - c0] : KEY_NEG_INF;
      }
    } else {
      float v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = base + 32 * u + lane;
        v[u] = j < we ? srow[j] : -INFINITY;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) kk[u] = score_key(v[u]);
    }
  };
  // Count pass over every key (no lists): warp-aggregated top-12-bit histogram.
  auto count_pass = [&](uint32_t *hdst) {
    for (int base = wb; base < we; base += 32 * U) {
      uint32_t kk[U];
      load_keys(base, kk);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t key = kk[u];
        const bool take = key != KEY_NEG_INF;
        const uint32_t peers = __match_any_sync(0xffffffffu, take ? (key >> 20) : 0xFFFFFFFFu);
        if (take && (peers & lt_mask) == 0) atomicAdd(&hdst[key >> 20], uint32_t(__popc(peers)));
      }
    }
  };
  // Visit the warp's keys in index order, 32 per step (lane = position in the step):
  // from its candidate list (fast) or from all keys (shared memory when the row is
  // resident, else the scores).  f(key, index, valid).
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
        uint32_t kk[U];
        load_keys(base, kk);
#pragma unroll
        for (int u = 0; u < U; ++u) f(kk[u], base + 32 * u + lane, kk[u] != KEY_NEG_INF);
      }
    }
  };

  for (int i = tid; i < 4 * TK_H12_WORDS + 2 * TK_H8_WORDS; i += TK_THREADS) hs[i] = 0;
  if (tid == 0) overflow_s = 0;
  __syncthreads();

  uint32_t prefix[2] = {0, 0}, rem[2] = {0, 0};
  int width[2] = {0, 0};
  bool all[2] = {true, true};
  // Per selection: radix prefix of T and its width in bits (resolved once the prefix's bin
  // holds exactly the keys still needed), keys still needed, or "take every key".
  auto first_digit = [&](const uint32_t *h, int lo) {
    sum_coarse(h, 0, TK_BINS, lo, true, false);
    if (warp < nsel) warp_select(sumc, h, TK_BINS, uint32_t(warp ? s1.k : s0.k), warp);
    __syncthreads();
    for (int s = 0; s < nsel; ++s) {
      all[s] = sel_bin[s] < 0;
      if (!all[s]) {
        prefix[s] = uint32_t(sel_bin[s]);
        rem[s] = uint32_t(s ? s1.k : s0.k) - sel_above[s];
        width[s] = 12;
      }
    }
  };
  bool fast = false;
  if (resident) {
    // ---- this CTA's chunk into shared memory as keys (c0 is a multiple of 4), then pass 0
    if (vec) {
      for (int i = c0 + 4 * tid; i < c1; i += 4 * TK_THREADS) {
        if (i + 3 < c1) {
          const float4 v = *reinterpret_cast<const float4 *>(srow + i);
          *reinterpret_cast<uint4 *>(skeys + (i - c0)) =
              make_uint4(score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w));
        } else {
          for (int e = i; e < c1; ++e) skeys[e - c0] = score_key(srow[e]);
        }
      }
    } else {
      for (int i = c0 + tid; i < c1; i += TK_THREADS) skeys[i - c0] = score_key(srow[i]);
    }
    __syncthreads();
    count_pass(hs);
    make_coarse(hs, TK_BINS);
    csync();
    first_digit(hs, 0);
  } else {
  // ---- sampled lower bound on the larger selection's threshold (top 12 key bits)
  const uint32_t target = uint32_t(kbig / SAMPLE) + uint32_t(kbig / (2 * SAMPLE)) + 32;
  for (int base = wb; base < we; base += 32 * SAMPLE * 8) {  // 8 loads in flight per lane (one round for a
    float v[8];                                                // range of up to 4096 scores)
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = base + 32 * SAMPLE * u + lane;
      v[u] = j < we ? srow[j] : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t key = score_key(v[u]);
      if (key != KEY_NEG_INF) atomicAdd(&hs[key >> 20], 1u);
    }
  }
  make_coarse(hs, TK_BINS);
  csync();  // (1)
  sum_coarse(hs, 0, TK_BINS, 0, true, false);
  if (warp == 0) warp_select(sumc, hs, TK_BINS, target, 0);
  __syncthreads();
  const int lo_bin = sel_bin[0] >= 0 ? sel_bin[0] : 0;

  // ---- pass 0 (bits 31..20) over keys at or above the bound, kept as candidates
  keep_pass(lo_bin, h0);
  if (lane == 0 && cnt > TK_CAPW) atomicOr(&overflow_s, 1);
  make_coarse(h0, TK_BINS);
  csync();  // (2)
  int any_overflow = 0;
#pragma unroll
  for (int q = 0; q < CS; ++q)
    any_overflow |= int(*peer(reinterpret_cast<const uint32_t *>(&overflow_s), q));
  first_digit(h0, lo_bin >> 3);
  // the bound is valid when at least kbig keys lie above it (or there was none)
  fast = !any_overflow && (lo_bin == 0 || sel_total[0] >= uint32_t(kbig));
  if (!fast) {  // count every key from the scores (peers finished reading hs before (2))
    for (int i = tid; i < TK_H12_WORDS; i += TK_THREADS) hs[i] = 0;
    __syncthreads();
    count_pass(hs);
    make_coarse(hs, TK_BINS);
    csync();
    first_digit(hs, 0);
  }
  }

  // ---- pass 1 (bits 19..8) and pass 2 (bits 7..0) over keys matching each prefix, for
  // selections whose prefix bin holds more keys than are still needed
  for (int pass = 1; pass < 3; ++pass) {
    const int w = pass == 1 ? 12 : 8, sh = pass == 1 ? 8 : 0, nfine = 1 << w;
    const int stride = pass == 1 ? TK_H12_WORDS : TK_H8_WORDS;
    uint32_t *hp = pass == 1 ? h1 : h2;
    const uint32_t mask = uint32_t(nfine - 1);
    const bool act0 = !all[0] && sel_count[0] != rem[0];
    const bool act1 = nsel > 1 && !all[1] && sel_count[1] != rem[1];
    if (!act0 && !act1) break;  // cluster-uniform
    walk(fast, [&](uint32_t key, int, bool valid) {
      if (!valid) return;
      const uint32_t hi = key >> (sh + w), bin = (key >> sh) & mask;
      if (act0 && hi == prefix[0]) atomicAdd(&hp[bin], 1u);
      if (act1 && hi == prefix[1]) atomicAdd(&hp[stride + bin], 1u);
    });
    make_coarse(hp, nfine);
    make_coarse(hp + stride, nfine);
    csync();  // (3), (4)
    sum_coarse(hp, stride, nfine, 0, act0, act1);
    if ((warp == 0 && act0) || (warp == 1 && act1))
      warp_select(sumc + warp * TK_CBINS, hp + warp * stride, nfine, rem[warp], warp);
    __syncthreads();
    if (act0) prefix[0] = (prefix[0] << w) | uint32_t(sel_bin[0]), rem[0] -= sel_above[0], width[0] += w;
    if (act1) prefix[1] = (prefix[1] << w) | uint32_t(sel_bin[1]), rem[1] -= sel_above[1], width[1] += w;
  }

  // ---- per-warp counts of keys above / equal to T (compared on the prefix's bits)
  uint32_t T[2];
  int tsh[2], need[2], gt_w[2] = {0, 0}, eq_w[2] = {0, 0};
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    T[s] = all[s] ? KEY_NEG_INF : prefix[s];
    tsh[s] = all[s] ? 0 : 32 - width[s];
    need[s] = all[s] ? 0 : int(rem[s]);
  }
  walk(fast, [&](uint32_t key, int, bool valid) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (s >= nsel) break;
      const uint32_t kh = key >> tsh[s];
      gt_w[s] += __popc(__ballot_sync(0xffffffffu, valid && kh > T[s]));
      eq_w[s] += __popc(__ballot_sync(0xffffffffu, valid && kh == T[s]));
    }
  });
  // ---- exclusive prefix over (cluster rank, warp); each CTA pushes its totals to every peer
  if (lane == 0) wc[warp][0] = gt_w[0], wc[warp][1] = eq_w[0], wc[warp][2] = gt_w[1], wc[warp][3] = eq_w[1];
  __syncthreads();
  if (warp == 0) {
    int v[4], x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = x[i] = wc[lane][i];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int y = __shfl_up_sync(0xffffffffu, x[i], o);
        if (lane >= o) x[i] += y;
      }
    int tot[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      wc[lane][i] = x[i] - v[i];
      tot[i] = __shfl_sync(0xffffffffu, x[i], 31);
    }
    if (lane < CS) {
      for (int s = 0; s < nsel; ++s) {
        int *dst = &tot_all[s][r][0];
        if constexpr (CS > 1) dst = cluster.map_shared_rank(dst, lane);
        dst[0] = tot[2 * s];
        dst[1] = tot[2 * s + 1];
      }
    }
  }
  csync();  // (5): no shared memory of a peer is touched after this barrier
  int gt_off[2], eq_off[2], selected[2] = {0, 0};
  for (int s = 0; s < nsel; ++s) {
    int gb = 0, eb = 0, gall = 0, eall = 0;
#pragma unroll
    for (int p = 0; p < CS; ++p) {
      if (p < r) gb += tot_all[s][p][0], eb += tot_all[s][p][1];
      gall += tot_all[s][p][0], eall += tot_all[s][p][1];
    }
    gt_off[s] = wc[warp][2 * s] + gb;
    eq_off[s] = wc[warp][2 * s + 1] + eb;
    selected[s] = gall + min(eall, need[s]);
  }

  // ---- write the chosen positions in ascending order
  for (int s = 0; s < nsel; ++s) {
    const Sel sl = s ? s1 : s0;
    const int k = sl.k, nd = need[s], ts = tsh[s];
    const uint32_t Ts = T[s];
    int32_t *orow = sl.idx + int64_t(row) * k;
    float *vrow = sl.val ? sl.val + int64_t(row) * k : nullptr;
    const int32_t *mrow = map ? map + int64_t(row) * N : nullptr;
    int g = gt_off[s], e = eq_off[s];
    walk(fast, [&](uint32_t key, int j, bool valid) {
      const uint32_t kh = key >> ts;
      const bool is_gt = valid && kh > Ts, is_eq = valid && kh == Ts;
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

static size_t tk_smem_bytes(int) { return sizeof(uint32_t) * TK_SMEM_WORDS; }

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

// Clusters of CS CTAs (one per SM) that the device can hold at once, per device.
template <int CS>
static int max_active_clusters() {
  static int cached[64] = {};  // 0 unknown, -1 none
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    if (CS > 8) cudaFuncSetAttribute(topk_cluster_kernel<CS>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaFuncSetAttribute(topk_cluster_kernel<CS>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(tk_smem_bytes(CS)));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CS);
    cfg.blockDim = dim3(TK_THREADS);
    cfg.dynamicSmemBytes = tk_smem_bytes(CS);
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = CS;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    cached[dev] = (cudaOccupancyMaxActiveClusters(&n, topk_cluster_kernel<CS>, &cfg) == cudaSuccess && n > 0) ? n : -1;
    cudaGetLastError();
  }
  return cached[dev];
}

// Cluster size by row length and count.  Rows of at least 2^18 scores: the largest of 16,
// 12, 10 and 8 CTAs whose clusters all fit on the device at once (a cluster needs its SMs in
// one GPC, so fewer large clusters fit than SMs / CS).  Shorter rows: about 4096 scores per
// CTA (then every CTA holds its chunk in shared memory), at most 8 CTAs, as long as all
// clusters fit at once.  From one row per SM on, or for rows of at most 4096 scores, one CTA
// per row and no cluster barriers.
void launch_topk_cluster(const float *scores, const int32_t *n_valid, int R, int N, int k0, int32_t *idx0, float *val0,
                         int k1, int32_t *idx1, float *val1, const int32_t *map, cudaStream_t st) {
  if (R == 0) return;
  const Sel s0{k0, idx0, val0}, s1{k1, idx1, val1};
  const int nsel = (k1 > 0 && idx1) ? 2 : 1;
  const int sms = sm_count();
  if (R < sms && N >= (1 << 18)) {
    if (max_active_clusters<16>() >= R) {
      launch_cs<16>(scores, n_valid, R, N, s0, s1, nsel, map, st);
    } else if (max_active_clusters<12>() >= R) {
      launch_cs<12>(scores, n_valid, R, N, s0, s1, nsel, map, st);
    } else if (max_active_clusters<10>() >= R) {
      launch_cs<10>(scores, n_valid, R, N, s0, s1, nsel, map, st);
    } else {
      launch_cs<8>(scores, n_valid, R, N, s0, s1, nsel, map, st);
    }
    return;
  }
  int cs = 1;
  if (R < sms)
    while (cs < 8 && cs * 4096 < N && 2 * cs * R <= sms) cs *= 2;
  if (cs == 8 && max_active_clusters<8>() < R) cs = 4;
  if (cs == 4 && max_active_clusters<4>() < R) cs = 2;
  switch (cs) {
    case 8: launch_cs<8>(scores, n_valid, R, N, s0, s1, nsel, map, st); break;
    case 4: launch_cs<4>(scores, n_valid, R, N, s0, s1, nsel, map, st); break;
    case 2: launch_cs<2>(scores, n_valid, R, N, s0, s1, nsel, map, st); break;
    default: launch_cs<1>(scores, n_valid, R, N, s0, s1, nsel, map, st); break;
  }
}

}  // namespace csa2
