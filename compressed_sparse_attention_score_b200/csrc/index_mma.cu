// K3 (tensor-core form): lightning-indexer scores with block-scaled FP4 tcgen05 MMA.
//
// Scores s_n = sum_h w_h * relu(q^_h . k^_n) are one block-scaled FP4 GEMM per
// 128-key tile: D[128 keys][64 heads] = K^ (e2m1, E8M0 per 32) x Q^^T, then a
// weighted ReLU row reduction.  The e2m1 codes and E8M0 exponents of the cache
// are consumed exactly as stored (kind::mxf4, scale vector 32), so the products
// are exact and only the fp32 accumulation order differs from a plain sum.
//
// CTA = one query row x a contiguous range of key tiles.  Row m of a tile's A
// operand holds tile entry e(m) = (m % 32) * 4 + m / 32, so the entries' scale
// words, copied in their natural order, form the 32 x 4-word scale-factor atom
// that tcgen05.cp expects (word w = (m % 32) * 4 + m / 32 = e).  Warp roles:
//   warp 0     producer: for a run of whole 128-entry groups one TMA box of a
//              4-D tensor map whose outer strides perform the row permutation
//              (64-byte swizzle) plus one 512-byte bulk copy of the scales, the
//              first 8 tiles during the prologue; for long candidate lists,
//              cp.async of each listed entry instead;
//   warp 1     MMA issuer (one lane): tcgen05.cp of the scale atom to TMEM, two
//              K=64 MMAs into one of three TMEM accumulators, tcgen05.commit;
//   warps 2-9  epilogue, two warpgroups taking alternate tiles: tcgen05.ld of
//              the 64 head values of its 32 keys, weighted ReLU sum, fp32 score
//              store.  A candidate list of at most 8 tiles is gathered by these
//              warps, one tile each, in the prologue.
// The query heads are quantised to MXFP4 in the prologue (warps 2-9, one 32-value block per
// thread; the keys' block format, encoded by cvt.rn.satfinite.e2m1x2).
// Every mbarrier wait is time-bounded; on expiry the CTA drains and reports
// CSA2_ERR_TIMEOUT instead of hanging.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace csa2 {
using namespace sm100;
namespace cg = cooperative_groups;

namespace {
constexpr int IM_STAGES = 8;
constexpr int IM_TILE = 128;           // keys per tile = MMA M
constexpr int IM_N = 64;               // indexer heads = MMA N
constexpr int IM_A_BYTES = IM_TILE * 64;
constexpr int IM_STAGE_BYTES = 9216;   // 8192 codes + 512 scale atom, padded to 1024
constexpr int IM_ACC = 3;              // TMEM accumulators (64 columns each)
constexpr int IM_EPI_WG = 2;           // epilogue warpgroups, alternating tiles
constexpr int IM_THREADS = 64 + 128 * IM_EPI_WG;
constexpr uint32_t IM_TMEM_COLS = 256;
constexpr uint32_t COL_SFA = IM_ACC * 64;   // one 4-column scale buffer per accumulator
constexpr uint32_t COL_SFB = COL_SFA + 4 * IM_ACC;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

constexpr int SM_STAGES = 0;
constexpr int SM_B = IM_STAGES * IM_STAGE_BYTES;       // 64 x 64 B query codes
constexpr int SM_SFB = SM_B + IM_N * 64;                // 512 B scale atom
constexpr int SM_W = SM_SFB + 512;                      // 64 fp32 head weights
constexpr int IM_CAND_TILES = 8;                        // candidate lists staged when a CTA has at most this many tiles
constexpr int SM_CAND = SM_W + 256;                     // [IM_CAND_TILES * 128] candidate entry indices
constexpr int SM_BAR = SM_CAND + IM_CAND_TILES * IM_TILE * 4;   // mbarriers
constexpr int N_BARS = 2 * IM_STAGES + 2 * IM_ACC + 1;
constexpr int SM_MISC = SM_BAR + 8 * N_BARS;            // tmem base, abort flag
constexpr int SM_TOTAL = SM_MISC + 16;
constexpr size_t IM_SMEM_BYTES = SM_TOTAL + 1024;       // slack for 1024-byte alignment
// Fused Reindex selection: each CTA keeps its candidates' keys; only digit histograms and
// counts cross the cluster.
constexpr int IM_SEL_MAX = REINDEX_SELECT_MAX;          // candidates per row
constexpr int SM_KEYS = SM_TOTAL;                       // [IM_CAND_TILES * 128] this CTA's keys
constexpr int SM_HL = SM_KEYS + IM_CAND_TILES * IM_TILE * 4;   // [2][256] local histograms (alternate digits)
constexpr int SM_HG = SM_HL + 2 * 256 * 4;              // [2][256] cluster-wide histograms (peers add here)
constexpr int SM_CG = SM_HG + 2 * 256 * 4;              // [16][2] every CTA's counts above / equal
constexpr int SM_WCNT = SM_CG + 16 * 2 * 4;             // per warp: keys above / equal to the threshold
constexpr size_t IM_SEL_SMEM_BYTES = SM_WCNT + 2 * (IM_THREADS / 32) * 4 + 1024;
static_assert(IM_EPI_WG >= 2, "the query is quantised by 8 epilogue warps");
static_assert((IM_SEL_MAX + IM_TILE - 1) / IM_TILE <= 16 * IM_CAND_TILES,
              "a pool of IM_SEL_MAX candidates must fit 16 CTAs of IM_CAND_TILES tiles (the count table holds 16)");
}  // namespace

struct IndexMmaArgs {
  bool use_tma;
  const uint16_t *q_ix;
  const uint16_t *w;
  int Q;
  const int32_t *q_pos;
  const int32_t *cand;
  int P;
  int n_out;
  csa2_cache c;
  float *scores;
  int32_t *err;
  int chunk;  // tiles per CTA
  int k;         // fused selection: top-k of the candidates ...
  int32_t *sel;  // ... written here [rows][k] (entries, ascending; -1 pads)
  int rows;      // query rows (balanced full scan: at most 32)
  int grid;      // > 0: balanced full scan over a one-dimensional grid of this many CTAs
  int spec;      // balanced: CTAs per row of the deal when every row fills the output (0: none)
};

// Balanced full scan.  Rows of very different lengths (a ragged batch) would leave most of a
// fixed (split, row) grid idle while the longest rows' few CTAs stream; instead every CTA deals
// the grid to the rows in proportion to their tiles (the same deal in every warp and CTA: it
// depends only on the rows' visible entries), at least IM_MIN_TILES tiles per CTA, and the score
// positions past each row's visible entries are split evenly over all CTAs.  Lane r of a warp
// holds row r's figures.
constexpr int IM_MIN_TILES = 8;
struct Deal {
  int row, t0, t_end;          // this CTA's row (-1: none) and its tiles [t0, t_end)
  int tiles, fill;             // lane r: row r's tiles and its positions past them
  int64_t fill_pre, fill_all;  // lane r: positions past the tiles of rows < r; of every row
};
__device__ __forceinline__ Deal deal_rows(const IndexMmaArgs &a, int lane) {
  int tl = 0;
  if (lane < a.rows) tl = (min(visible_entries(a.c, lane / a.Q, a.q_pos[lane]), a.n_out) + IM_TILE - 1) / IM_TILE;
  int total = tl;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
  // CTAs of a row with tiles: ceil(g tiles / total), at least 1, at most one per IM_MIN_TILES tiles;
  // with g = grid - rows the sum is at most (grid - rows) + rows (and grid >= rows)
  auto share = [&](int g) {
    if (tl == 0) return 0;
    return max(1, min(int((int64_t(g) * tl + total - 1) / total), (tl + IM_MIN_TILES - 1) / IM_MIN_TILES));
  };
  int sp = share(a.grid), sum = sp;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (sum > a.grid) sp = share(max(0, a.grid - a.rows));
  int incl = sp;
  int64_t fincl = lane < a.rows ? max(0, a.n_out - tl * IM_TILE) : 0;
  const int fill = int(fincl);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    const int64_t fy = __shfl_up_sync(0xffffffffu, fincl, o);
    if (lane >= o) incl += y, fincl += fy;
  }
  const int c = int(blockIdx.x);
  const unsigned own = __ballot_sync(0xffffffffu, sp > 0 && c >= incl - sp && c < incl);
  Deal d;
  d.row = -1, d.t0 = 0, d.t_end = 0;
  if (own) {
    const int r = __ffs(own) - 1;
    const int spr = __shfl_sync(0xffffffffu, sp, r), tlr = __shfl_sync(0xffffffffu, tl, r);
    const int part = c - (__shfl_sync(0xffffffffu, incl, r) - spr), ch = (tlr + spr - 1) / spr;
    d.t0 = min(tlr, part * ch), d.t_end = min(tlr, d.t0 + ch);
    if (d.t0 < d.t_end) d.row = r;
  }
  d.tiles = tl, d.fill = fill;
  d.fill_pre = fincl - fill, d.fill_all = __shfl_sync(0xffffffffu, fincl, 31);
  return d;
}
// The deal's tail figures kept in shared memory (the candidate-list space, which a full scan
// does not use) from the prologue to the end of the epilogue: per row the positions past the
// tiles of the rows before it, its own, its tiles; then the total.
struct Tails {
  int64_t pre[32];
  int n[32], tiles[32];
  int64_t all;
};
__device__ __forceinline__ void keep_tails(Tails *tz, const Deal &d, int lane) {  // one warp
  tz->pre[lane] = d.fill_pre, tz->n[lane] = d.fill, tz->tiles[lane] = d.tiles;
  if (lane == 0) tz->all = d.fill_all;
}
// This CTA's even share of the positions past the rows' visible tiles, written -inf by the
// threads t = 0 .. nt-1.
__device__ __forceinline__ void fill_tails(const IndexMmaArgs &a, const Tails *tz, int t, int nt) {
  const int64_t G = gridDim.x, c = blockIdx.x;
  const int64_t lo = tz->all * c / G, hi = tz->all * (c + 1) / G;
  for (int r = 0; r < a.rows; ++r) {
    const int64_t pre = tz->pre[r];
    float *out = a.scores + int64_t(r) * a.n_out + int64_t(tz->tiles[r]) * IM_TILE;  // first position past its tiles
    for (int64_t i = max(lo, pre) + t; i < min(hi, pre + tz->n[r]); i += nt) out[i - pre] = -INFINITY;
  }
}

// A-operand row of tile entry e and the inverse map.
__device__ __forceinline__ int row_of_entry(int e) { return (e & 3) * 32 + (e >> 2); }
__device__ __forceinline__ int entry_of_row(int m) { return (m & 31) * 4 + (m >> 5); }

// Top-k of one row's candidates spread over the CS CTAs of a cluster (CTA r holds positions
// [pos0, pos0 + nl) of the row: keys kl, entries el), score descending and position ascending
// among equal scores, -inf keys never chosen; written as the chosen candidates' entries in
// position order, -1 padded -- the selection csa2_topk makes of the same scores with the
// candidate list as its map.  The threshold key comes from a radix selection on 8-bit digits
// from the top: per digit every CTA histograms its own keys and adds the histogram into every
// peer's, one cluster barrier, and every CTA finds the same threshold digit; it stops early once
// the threshold bin holds exactly the keys still needed.  A last exchange of per-CTA counts
// places each CTA's chosen entries.  Called by every thread of every CTA of the cluster.
__device__ __forceinline__ void select_cluster(const uint32_t *kl, const int32_t *el, int nl, int k, int32_t *orow,
                                               uint32_t *hl, uint32_t *hg, int *cg_, int *wcnt) {
  constexpr int NW = IM_THREADS / 32;
  cg::cluster_group cluster = cg::this_cluster();
  const int cs = int(cluster.num_blocks()), rank = int(cluster.block_rank());
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  uint32_t prefix = 0;
  int need = k, width = 0;
  bool all = false;
  // Per digit: local histogram, one block barrier, pushes, one cluster barrier; every warp then
  // finds the digit itself.  The local and cluster histograms alternate between two copies, each
  // zeroed a digit ahead, after the last reads of it are ordered by a barrier.
  for (int pass = 0, shift = 24; shift >= 0; ++pass, shift -= 8) {
    uint32_t *hcur = hg + (pass & 1) * 256, *hgn = hg + ((pass + 1) & 1) * 256;
    uint32_t *hlc = hl + (pass & 1) * 256, *hln = hl + ((pass + 1) & 1) * 256;
    const uint32_t himask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int i = t; i - lane < nl; i += IM_THREADS) {  // lanes with the same bin add once
      const uint32_t key = i < nl ? kl[i] : KEY_NEG_INF;
      const bool act = key != KEY_NEG_INF && (key & himask) == prefix;
      const uint32_t am = __ballot_sync(0xffffffffu, act);
      if (act) {
        const uint32_t bin = (key >> shift) & 255u, peers = __match_any_sync(am, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&hlc[bin], uint32_t(__popc(peers)));
      }
    }
    if (t < 256) hln[t] = 0;  // read last by the previous digit's pushes
    __syncthreads();
    if (t < 256) hgn[t] = 0;  // read last by every warp before this digit's block barrier
    for (int j = t; j < 256 * cs; j += IM_THREADS) {  // into every CTA's copy, this one's included
      const uint32_t c = hlc[j & 255];
      if (c) atomicAdd(cluster.map_shared_rank(hcur + (j & 255), j >> 8), c);
    }
    cluster.sync();
    // the digit at which the count from the top reaches `need` (the same in every warp and CTA)
    uint32_t c8[8], sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) sum += (c8[j] = hcur[255 - (8 * lane + j)]);
    uint32_t x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const uint32_t excl = x - sum, total = __shfl_sync(0xffffffffu, x, 31);
    if (total <= uint32_t(need)) {  // first digit only: at most k valid keys, all chosen
      all = true;
      break;
    }
    const int L = __ffs(__ballot_sync(0xffffffffu, excl < uint32_t(need) && x >= uint32_t(need))) - 1;
    uint32_t dg = 0, nd = 0, cnt = 0;
    if (lane == L) {
      uint32_t cum = excl;
#pragma unroll 1
      for (int j = 0; j < 8; ++j) {
        if (cum + c8[j] >= uint32_t(need)) {
          dg = uint32_t(255 - (8 * lane + j));
          nd = uint32_t(need) - cum;
          cnt = c8[j];
          break;
        }
        cum += c8[j];
      }
    }
    dg = __shfl_sync(0xffffffffu, dg, L);
    nd = __shfl_sync(0xffffffffu, nd, L);
    cnt = __shfl_sync(0xffffffffu, cnt, L);
    prefix |= dg << shift;
    need = int(nd);
    width = 32 - shift;
    if (int(cnt) == need) break;  // every key of the threshold bin is chosen
  }
  // keys above / equal to the threshold T, compared on the top `width` bits
  const int sh = 32 - width;
  const uint32_t T = all ? 0u : prefix >> sh;
  const int seg = ((nl + NW * 32 - 1) / (NW * 32)) * 32, j0 = warp * seg, j1 = min(nl, j0 + seg);
  int gt = 0, eq = 0;
  for (int j = j0 + lane; j - lane < j1; j += 32) {
    const uint32_t key = j < j1 ? kl[j] : KEY_NEG_INF;
    const bool valid = key != KEY_NEG_INF;
    gt += __popc(__ballot_sync(0xffffffffu, valid && (all || (key >> sh) > T)));
    eq += __popc(__ballot_sync(0xffffffffu, valid && !all && (key >> sh) == T));
  }
  if (lane == 0) wcnt[2 * warp] = gt, wcnt[2 * warp + 1] = eq;
  __syncthreads();
  if (t < cs) {  // this CTA's totals into every CTA's table
    int g = 0, e = 0;
    for (int w2 = 0; w2 < NW; ++w2) g += wcnt[2 * w2], e += wcnt[2 * w2 + 1];
    int *dst = cluster.map_shared_rank(cg_ + 2 * rank, t);
    dst[0] = g;
    dst[1] = e;
  }
  cluster.sync();  // no shared memory of a peer is touched after this barrier
  int g = 0, e = 0, gall = 0, eall = 0;
  for (int r = 0; r < cs; ++r) {
    if (r < rank) g += cg_[2 * r], e += cg_[2 * r + 1];
    gall += cg_[2 * r];
    eall += cg_[2 * r + 1];
  }
  for (int w2 = 0; w2 < warp; ++w2) g += wcnt[2 * w2], e += wcnt[2 * w2 + 1];
  const int nd = all ? 0 : need;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int j = j0 + lane; j - lane < j1; j += 32) {
    const uint32_t key = j < j1 ? kl[j] : KEY_NEG_INF;
    const bool valid = key != KEY_NEG_INF;
    const bool is_gt = valid && (all || (key >> sh) > T), is_eq = valid && !all && (key >> sh) == T;
    const uint32_t gm = __ballot_sync(0xffffffffu, is_gt), em = __ballot_sync(0xffffffffu, is_eq);
    const int gbef = g + __popc(gm & lt_mask), ebef = e + __popc(em & lt_mask);
    const int at = is_gt ? gbef + min(ebef, nd) : ((is_eq && ebef < nd) ? gbef + ebef : -1);
    if (at >= 0 && at < k) orow[at] = el[j];
    g += __popc(gm);
    e += __popc(em);
  }
  if (rank == 0)
    for (int i = gall + min(eall, nd) + t; i < k; i += IM_THREADS) orow[i] = -1;
}

template <bool SEL>
__global__ void __launch_bounds__(IM_THREADS, 2) index_score_mma_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                                 IndexMmaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM_BAR);
  uint64_t *empty = full + IM_STAGES;
  uint64_t *acc_full = empty + IM_STAGES;
  uint64_t *acc_empty = acc_full + IM_ACC;
  uint64_t *done = acc_empty + IM_ACC;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SM_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + SM_MISC + 4);
  float *ws = reinterpret_cast<float *>(smem + SM_W);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  grid_dep_launch();  // a dependent attention launch may start its prologue
  int row = blockIdx.y, t0 = blockIdx.x * a.chunk, t_end = t0 + a.chunk;
  // The epilogue warps' query block and head weight go out first.  A balanced scan knows its row
  // only from the deal, one round trip later: it loads the row it has when every row fills the
  // output (the deal of equal rows) and loads again only if the deal says otherwise.
  const int qt = int(threadIdx.x) - 64, qhd = qt >> 2, qg = qt & 3;
  uint4 qv[4];
  uint16_t w_raw = 0;
  auto load_query = [&](int r) {
    if (warp >= 2) {
      w_raw = a.w[int64_t(r) * HI + qhd];
      const uint16_t *qh = a.q_ix + (int64_t(r) * HI + qhd) * DI;
#pragma unroll
      for (int i = 0; i < 4; ++i) qv[i] = reinterpret_cast<const uint4 *>(qh + 32 * qg)[i];
    }
  };
  int row_q = row;
  if constexpr (!SEL) {
    if (a.grid > 0) row_q = a.spec > 0 ? min(a.rows - 1, int(blockIdx.x) / a.spec) : 0;
  }
  load_query(row_q);
  Tails *tails = reinterpret_cast<Tails *>(smem + SM_CAND);
  static_assert(sizeof(Tails) <= IM_CAND_TILES * IM_TILE * 4, "the deal's tails fit the candidate-list space");
  if constexpr (!SEL) {
    if (a.grid > 0) {  // balanced full scan: this CTA's row and tiles from the deal
      const Deal d = deal_rows(a, lane);
      if (warp == 0) keep_tails(tails, d, lane);
      if (d.row < 0) {  // no tiles: only its share of the tails
        __syncthreads();
        fill_tails(a, tails, threadIdx.x, IM_THREADS);
        return;
      }
      row = d.row, t0 = d.t0, t_end = d.t_end;
      if (row != row_q) load_query(row);
    }
  }
  const int b = row / a.Q;
  const int nvis = visible_entries(a.c, b, a.q_pos[row]);
  const int n_entries = a.c.num_entries[b];
  const int t_all = (a.n_out + IM_TILE - 1) / IM_TILE;
  const int t_work = a.cand ? (a.P + IM_TILE - 1) / IM_TILE : (nvis + IM_TILE - 1) / IM_TILE;
  const int t1 = min(t_end, t_all);
  const int ntiles = max(0, min(t1, t_work) - t0);
  // a full scan whose output row is shorter than the visible entries would drop the tail
  if (!a.cand && nvis > a.n_out && t0 == 0 && threadIdx.x == 0) report(a.err, CSA2_ERR_SHAPE);

  // Candidate lists of at most IM_CAND_TILES tiles are copied to shared memory by warp 0
  // while the other warps run the prologue, so the producer and the epilogue never wait
  // on a global load of an index.
  int32_t *cand_s = reinterpret_cast<int32_t *>(smem + SM_CAND);
  const bool cand_staged = a.cand && ntiles <= IM_CAND_TILES;
  // Gathered tiles that all fit the ring at once are issued by the epilogue warps, one tile
  // each, right after the prologue (they are idle until the first product anyway); otherwise
  // warp 0 issues every tile in turn.
  static_assert(IM_CAND_TILES <= IM_STAGES && IM_CAND_TILES <= 4 * IM_EPI_WG, "a staged list is one tile per epilogue warp");
  const bool spread = !a.use_tma && cand_staged;
  const uint32_t stages = smem_u32(smem + SM_STAGES);

  // Gather path: lane l resolves the slots of tile entries l, l+32, l+64, l+96, the slots
  // are shuffled to the lanes that copy each 16-byte chunk, and each lane's copies arrive on
  // the stage's barrier by themselves (cp.async.mbarrier.arrive.noinc).
  auto load_cand = [&](int tile, int32_t (&cv)[4]) {  // entry index of each position (-1: none)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int pos = tile * IM_TILE + lane + 32 * j;
      if (tile >= t0 + ntiles) cv[j] = -1;
      else if (!a.cand) cv[j] = pos;
      else if (cand_staged) cv[j] = cand_s[pos - t0 * IM_TILE];
      else cv[j] = pos < a.P ? a.cand[int64_t(row) * a.P + pos] : -1;
    }
  };
  auto resolve = [&](const int32_t (&cv)[4], int64_t (&sl)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = cv[j];
      if (a.cand && (n < -1 || n >= n_entries)) report(a.err, CSA2_ERR_INDEX);
      int64_t sv = -1;
      if (n >= 0 && n < nvis) {
        sv = cache_slot(a.c, b, n);
        if (sv < 0) report(a.err, CSA2_ERR_INDEX);
      }
      sl[j] = sv;
    }
  };
  auto issue_tile = [&](int s, const int64_t (&cur)[4]) {  // the whole warp
    const uint32_t st = stages + s * IM_STAGE_BYTES;
#pragma unroll
    for (int j = 0; j < 16; ++j) {  // 512 chunks of 16 bytes: chunk qd = lane + 32 j
      const int qd = lane + 32 * j, e = qd >> 2, c = qd & 3, m = row_of_entry(e);
      // entry e = 8 j + lane / 4 lives in lane e % 32, register j / 4
      const int64_t slot = __shfl_sync(0xffffffffu, cur[j >> 2], e & 31);
      if (slot >= 0)
        cp_async_16(st + m * 64 + ((c ^ ((m >> 1) & 3)) << 4), a.c.ix_codes + slot * CSA2_IX_CODE_BYTES + c * 16);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)  // scale word of entry e = lane + 32 j at atom word e
      if (cur[j] >= 0) cp_async_4(st + IM_A_BYTES + (lane + 32 * j) * 4, a.c.ix_scales + cur[j] * CSA2_IX_SCALE_BYTES);
    cp_async_arrive_noinc(&full[s]);
  };
  auto issue_tma = [&](int i) {  // one lane: tile i of a whole-group run (its stage is free)
    const int s = i % IM_STAGES;
    const uint32_t st = stages + s * IM_STAGE_BYTES;
    const int64_t slot0 = cache_slot(a.c, b, int64_t(t0 + i) * IM_TILE);
    if (slot0 >= 0 && (slot0 & (IM_TILE - 1)) == 0 && slot0 + IM_TILE <= a.c.num_slots) {
      mbar_arrive_expect_tx(&full[s], IM_A_BYTES + 512);
      tma_load_4d(st, &tmap, 0, 0, 0, int(slot0 / IM_TILE), &full[s]);
      bulk_load(st + IM_A_BYTES, a.c.ix_scales + slot0 * CSA2_IX_SCALE_BYTES, 512, &full[s]);
    } else {
      report(a.err, CSA2_ERR_INDEX);  // a visible tile without a valid page: epilogue masks it
      mbar_arrive(&full[s]);
    }
  };
  // The first tiles go out before the prologue's end: warp 1 initialises the barriers and
  // meets the warps that issue them (warp 0 for whole-group runs, the epilogue warps for
  // staged gathers) on named barrier 1.
  const int pre_tiles = a.use_tma ? min(ntiles, IM_STAGES) : 0;
  const int pre_threads = a.use_tma ? 64 : (spread ? 288 : 0);

  // ---------------------------------------------------------------- prologue
  if (warp == 0) {
    tmem_alloc(tmem_slot, IM_TMEM_COLS);
    tmem_relinquish();
    if (cand_staged) {  // every index copy in flight at once (asynchronous copies), then one wait
      const int32_t *crow = a.cand + int64_t(row) * a.P;
      for (int i = lane; i < ntiles * IM_TILE; i += 32) {
        const int pos = t0 * IM_TILE + i;
        if (pos < a.P)
          cp_async_4(smem_u32(cand_s + i), crow + pos);
        else
          cand_s[i] = -1;
      }
      cp_async_commit();
      cp_async_wait<0>();
    }
    if (a.use_tma) {
      named_bar_sync(1, pre_threads);
      if (lane == 0)
        for (int i = 0; i < pre_tiles; ++i) issue_tma(i);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      for (int s = 0; s < IM_STAGES; ++s) {
        mbar_init(&full[s], a.use_tma ? 1 : 32);  // gather path: one cp.async arrival per producer lane
        mbar_init(&empty[s], 1);
      }
      for (int i = 0; i < IM_ACC; ++i) {
        mbar_init(&acc_full[i], 1);
        mbar_init(&acc_empty[i], 4);
      }
      mbar_init(done, 1);
      *abort_flag = 0;
      mbar_init_fence();
    }
    if (pre_threads) named_bar_sync(1, pre_threads);
  } else if (warp >= 2 && warp < 10) {
    // quantise the query heads: thread 4h + g owns 32-value block g of head h (8 of the epilogue
    // warps, idle until the first tile).  Dividing by the power-of-two scale 2^e is done as the
    // (exactly equal) product with 2^-e.
    const int t = qt, h = qhd, g = qg;  // the query block and w_raw (used at the end) are in flight
    if (spread) {  // this warp's tile of a staged gather (every stage is still free), read from the list
      int32_t cv[4];  // loaded together with the query block
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int pos = (t0 + warp - 2) * IM_TILE + lane + 32 * j;
        cv[j] = (warp - 2 < ntiles && pos < a.P) ? a.cand[int64_t(row) * a.P + pos] : -1;
      }
      named_bar_sync(1, pre_threads);
      if (warp - 2 < ntiles) {
        int64_t sl[4];
        resolve(cv, sl);
        issue_tile(warp - 2, sl);
      }
    }
    uint8_t *brow = smem + SM_B + h * 64;
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 u = qv[i];
      const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * i + 2 * j] = __uint_as_float(ww[j] << 16);
        v[8 * i + 2 * j + 1] = __uint_as_float(ww[j] & 0xFFFF0000u);
      }
    }
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) am = fmaxf(am, fabsf(v[i]));
    int ex = -127;
    uint32_t cw[4] = {0, 0, 0, 0};
    if (am != 0.f) {
      ex = e8m0_ceil_exponent(__fdiv_rn(am, 6.0f));
      const float inv = pow2f(-ex);
#pragma unroll
      for (int i = 0; i < 32; i += 2) {  // a NaN encodes as 0, as the format's encoder does
        const float a0 = __fmul_rn(v[i], inv), a1 = __fmul_rn(v[i + 1], inv);
        cw[i >> 3] |= e2m1x2_code(a0 == a0 ? a0 : 0.f, a1 == a1 ? a1 : 0.f) << (4 * (i & 7));
      }
    }
    // 16 bytes = chunk g of this 64-byte row, at its swizzled position
    *reinterpret_cast<uint4 *>(brow + ((g ^ ((h >> 1) & 3)) << 4)) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    uint32_t sfword = uint32_t(ex + 127) << (8 * g);
    sfword |= __shfl_xor_sync(0xffffffffu, sfword, 1);
    sfword |= __shfl_xor_sync(0xffffffffu, sfword, 2);
    // scale atom word of row r: lane-row r % 32, column r / 32 (rows 64..127 unused, zero)
    if constexpr (SEL)
      for (int j = t; j < 1024; j += 256) reinterpret_cast<uint32_t *>(smem + SM_HL)[j] = 0;  // both pairs
    if (g == 0) {
      *reinterpret_cast<uint32_t *>(smem + SM_SFB + (h & 31) * 16 + (h >> 5) * 4) = sfword;
      ws[h] = bf16_to_f32(w_raw);
    } else if (g == 1) {
      const int rz = 64 + h;
      *reinterpret_cast<uint32_t *>(smem + SM_SFB + (rz & 31) * 16 + (rz >> 5) * 4) = 0u;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if constexpr (SEL) cluster_arrive();  // this CTA has started and zeroed its histograms (waited on before the selection)

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (a.use_tma) {
      if (lane == 0) {
        for (int i = pre_tiles; i < ntiles; ++i) {
          const int s = i % IM_STAGES;
          if (!mbar_wait_bounded(&empty[s], ((i / IM_STAGES) & 1) ^ 1, abort_flag, WAIT_LIMIT_NS)) break;
          issue_tma(i);
        }
      }
    } else if (!spread) {  // gather path, one tile after another (raw candidate indices two tiles ahead)
      int32_t c1[4], c2[4];
      int64_t cur[4], nxt[4];
      load_cand(t0, c1);
      resolve(c1, cur);
      load_cand(t0 + 1, c1);
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % IM_STAGES;
        load_cand(t0 + i + 2, c2);
        resolve(c1, nxt);
        if (!mbar_wait_bounded(&empty[s], ((i / IM_STAGES) & 1) ^ 1, abort_flag, WAIT_LIMIT_NS)) break;
        issue_tile(s, cur);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          cur[j] = nxt[j];
          c1[j] = c2[j];
        }
      }
      cp_async_wait<0>();
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t stages = smem_u32(smem + SM_STAGES);
      const uint32_t bq = smem_u32(smem + SM_B);
      tc_cp_32x128b_warpx4(tmem + COL_SFB, smem_desc(smem_u32(smem + SM_SFB), 16, 128, LAYOUT_SWIZZLE_NONE));
      const uint64_t b0 = smem_desc(bq, 16, 512, LAYOUT_SWIZZLE_64B);
      const uint64_t b1 = smem_desc(bq + 32, 16, 512, LAYOUT_SWIZZLE_64B);
      constexpr uint32_t id0 = idesc_mxf4(IM_TILE, IM_N, 0, 0);
      constexpr uint32_t id1 = idesc_mxf4(IM_TILE, IM_N, 2, 2);
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % IM_STAGES, acc = i % IM_ACC;
        if (!mbar_wait_bounded(&full[s], (i / IM_STAGES) & 1, abort_flag, WAIT_LIMIT_NS)) break;
        if (!mbar_wait_bounded(&acc_empty[acc], ((i / IM_ACC) & 1) ^ 1, abort_flag, WAIT_LIMIT_NS)) break;
        if (!a.use_tma) fence_proxy_async_smem();  // cp.async-filled stages are read by the tensor core
        tc_fence_after();
        const uint32_t st = stages + s * IM_STAGE_BYTES;
        const uint32_t sfa = tmem + COL_SFA + 4 * acc;
        tc_cp_32x128b_warpx4(sfa, smem_desc(st + IM_A_BYTES, 16, 128, LAYOUT_SWIZZLE_NONE));
        const uint32_t d = tmem + acc * IM_N;
        tc_mma_mxf4(d, smem_desc(st, 16, 512, LAYOUT_SWIZZLE_64B), b0, id0, sfa, tmem + COL_SFB, false);
        tc_mma_mxf4(d, smem_desc(st + 32, 16, 512, LAYOUT_SWIZZLE_64B), b1, id1, sfa, tmem + COL_SFB, true);
        tc_commit(&empty[s]);
        tc_commit(&acc_full[acc]);
      }
      tc_commit(done);  // fires once every tcgen05 op of this thread has completed
      // wait for it even after an abort, so TMEM is never freed under a running MMA
      const uint64_t t_start = globaltimer();
      while (!mbar_try_wait(done, 0) && globaltimer() - t_start < WAIT_LIMIT_NS) {
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q4 = warp & 3;              // TMEM sub-partition of this warp
    const int e = entry_of_row(32 * q4 + lane);  // tile entry of this thread's accumulator row
    const float4 *w4 = reinterpret_cast<const float4 *>(ws);
    // warpgroup wg takes tiles wg, wg + IM_EPI_WG, ...; the entry behind this thread's
    // row is fetched one of its tiles ahead (candidate lists are read from global)
    const int wg = (warp - 2) >> 2;
    uint32_t *keys_l = reinterpret_cast<uint32_t *>(smem + SM_KEYS);  // fused selection: this CTA's keys
    auto entry_at = [&](int i) -> int64_t {
      const int pos = (t0 + i) * IM_TILE + e;
      if (!a.cand) return pos;
      if (i >= ntiles || pos >= a.P) return -1;
      return cand_staged ? cand_s[pos - t0 * IM_TILE] : a.cand[int64_t(row) * a.P + pos];
    };
    int64_t n_next = entry_at(wg);
    for (int i = wg; i < ntiles; i += IM_EPI_WG) {
      const int acc = i % IM_ACC;
      const int64_t n_cur = n_next;
      n_next = entry_at(i + IM_EPI_WG);
      // the whole warp takes tcgen05.ld or none of it does
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&acc_full[acc], (i / IM_ACC) & 1, abort_flag, WAIT_LIMIT_NS)))
        break;
      tc_fence_after();
      const uint32_t taddr = tmem + (uint32_t(32 * q4) << 16) + acc * IM_N;
      uint32_t r0[32], r1[32];
      tc_ld_32x32b_x32(taddr, r0);
      tc_ld_32x32b_x32(taddr + 32, r1);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      const float sc = weighted_relu_score(r0, r1, w4);
      const int pos = (t0 + i) * IM_TILE + e;
      if (pos < a.n_out) {
        const bool ok = n_cur >= 0 && n_cur < nvis && cache_slot(a.c, b, n_cur) >= 0;
        if constexpr (SEL)
          keys_l[pos - t0 * IM_TILE] = score_key(ok ? sc : -INFINITY);
        else
          a.scores[int64_t(row) * a.n_out + pos] = ok ? sc : -INFINITY;
      }
    }
    if (spread) cp_async_wait<0>();  // no copy of this thread is left in flight
    // positions past the visible entries (no key tile was loaded for them): in a balanced scan
    // this CTA's share of every row's, else those of its own range
    if constexpr (!SEL) {
      if (a.grid > 0) fill_tails(a, tails, threadIdx.x - 64, 128 * IM_EPI_WG);
    }
    if (!a.cand && a.grid == 0) {
      const int lo = max(t0, t_work) * IM_TILE, hi = min(t1 * IM_TILE, a.n_out);
      for (int pos = lo + threadIdx.x - 64; pos < hi; pos += 128 * IM_EPI_WG)
        a.scores[int64_t(row) * a.n_out + pos] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, IM_TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) report(a.err, CSA2_ERR_TIMEOUT);
  if constexpr (SEL) {
    cluster_wait();
    select_cluster(reinterpret_cast<const uint32_t *>(smem + SM_KEYS), cand_s, max(0, min(a.P - t0 * IM_TILE, ntiles * IM_TILE)),
                   a.k, a.sel + int64_t(row) * a.k, reinterpret_cast<uint32_t *>(smem + SM_HL),
                   reinterpret_cast<uint32_t *>(smem + SM_HG), reinterpret_cast<int *>(smem + SM_CG),
                   reinterpret_cast<int *>(smem + SM_WCNT));
  }
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

// 4-D view of the indexer-code plane: (64 bytes, entry / 4 within a 128-entry
// group [stride 256 B], entry % 4 [stride 64 B], group [stride 8192 B]).  A box
// of (64, 32, 4, 1) lands entry e of the group at shared-memory row (e%4)*32 + e/4.
bool make_index_code_map(CUtensorMap *m, const csa2_cache &c) {
  auto enc = tensor_map_encoder();
  if (!enc || (c.num_slots % IM_TILE) != 0 || c.num_slots / IM_TILE > (int64_t(1) << 31)) return false;
  if ((reinterpret_cast<uintptr_t>(c.ix_scales) & 15) || (reinterpret_cast<uintptr_t>(c.ix_codes) & 15)) return false;
  if (c.page_table ? (c.page_size % IM_TILE) != 0 : (c.seq_stride % IM_TILE) != 0) return false;
  const cuuint64_t dims[4] = {64, 32, 4, cuuint64_t(c.num_slots / IM_TILE)};
  const cuuint64_t strides[3] = {256, 64, uint64_t(IM_TILE) * 64};
  const cuuint32_t box[4] = {64, 32, 4, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, c.ix_codes, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

void launch_index_score_mma(const uint16_t *q_ix, const uint16_t *w, int B, int Q, const int32_t *q_pos,
                            const int32_t *cand, int P, int n_out, const csa2_cache &c, float *scores, int32_t *err,
                            cudaStream_t st) {
  const int rows = B * Q;
  if (n_out == 0 || rows == 0) return;
  const int t_all = (n_out + IM_TILE - 1) / IM_TILE;
  const int want = (2 * sm_count() + rows - 1) / rows;   // about two CTAs per SM in total
  const int min_tiles = cand ? 4 : IM_MIN_TILES;          // short candidate lists: spread them wider
  const int splits = max(1, min(min(want, (t_all + min_tiles - 1) / min_tiles), 65535));
  const int chunk = (t_all + splits - 1) / splits;
  CUtensorMap tmap;
  memset(&tmap, 0, sizeof(tmap));
  const bool use_tma = cand == nullptr && make_index_code_map(&tmap, c);
  IndexMmaArgs a{use_tma, q_ix, w, Q, q_pos, cand, P, n_out, c, scores, err, chunk};
  a.rows = rows;
  set_smem_limit(index_score_mma_kernel<false>, IM_SMEM_BYTES);
  // A full scan of 2 to 32 rows deals the CTAs to the rows by their visible entries (a ragged
  // batch keeps every SM streaming); for rows of equal length the deal is the (split, row) grid.
  // One row keeps that grid, which already spreads it over every CTA, without the deal's round trip.
  if (cand == nullptr && rows >= 2 && rows <= 32) {
    a.grid = min(2 * sm_count(), rows * ((t_all + IM_MIN_TILES - 1) / IM_MIN_TILES));
    a.spec = a.grid % rows == 0 ? a.grid / rows : 0;
    index_score_mma_kernel<false><<<dim3(a.grid), IM_THREADS, IM_SMEM_BYTES, st>>>(tmap, a);
    return;
  }
  index_score_mma_kernel<false><<<dim3((t_all + chunk - 1) / chunk, rows), IM_THREADS, IM_SMEM_BYTES, st>>>(tmap, a);
}

namespace {
// One-time attributes of the fused-selection kernel for a cluster of CS CTAs, and how many
// such clusters the device holds at once (0: none).
template <int CS>
int select_clusters() {
  static int cached[64] = {};  // 0 unknown, -1 none
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    if (CS > 8) cudaFuncSetAttribute(index_score_mma_kernel<true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaFuncSetAttribute(index_score_mma_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         int(IM_SEL_SMEM_BYTES));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CS);
    cfg.blockDim = dim3(IM_THREADS);
    cfg.dynamicSmemBytes = IM_SEL_SMEM_BYTES;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = CS;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    cached[dev] =
        (cudaOccupancyMaxActiveClusters(&n, index_score_mma_kernel<true>, &cfg) == cudaSuccess && n > 0) ? n : -1;
    cudaGetLastError();
  }
  return cached[dev] > 0 ? cached[dev] : 0;
}

int select_clusters(int cs) {
  switch (cs) {
    case 16: return select_clusters<16>();
    case 8: return select_clusters<8>();
    case 4: return select_clusters<4>();
    case 2: return select_clusters<2>();
    default: return select_clusters<1>();
  }
}
}  // namespace

// Cluster size: at most IM_CAND_TILES tiles per CTA (16 CTAs for a pool of 16384), up to 16 CTAs
// of about 8 tiles while the rows' CTAs fit two per SM (every CTA quantises the row's query
// again, so many rows take fewer, longer CTAs), and only as large as lets every row's cluster
// run at once.
void launch_reindex_select(const uint16_t *q_ix, const uint16_t *w, int B, int Q, const int32_t *q_pos,
                           const int32_t *cand, int P, int k, const csa2_cache &c, int32_t *sel, int32_t *err,
                           cudaStream_t st) {
  const int rows = B * Q;
  if (rows == 0 || P == 0) return;
  const int t_all = (P + IM_TILE - 1) / IM_TILE;
  int cs_min = 1;  // every CTA's keys and candidate indices fit its shared memory
  while (cs_min * IM_CAND_TILES < t_all) cs_min *= 2;
  int cs = cs_min;
  while (cs < 16 && cs * 8 < t_all && 2 * cs * rows <= 2 * sm_count()) cs *= 2;
  while (cs > cs_min && select_clusters(cs) < min(rows, sm_count() / cs)) cs /= 2;
  select_clusters(cs);  // sets the kernel's attributes
  const int chunk = (t_all + cs - 1) / cs;
  CUtensorMap tmap;
  memset(&tmap, 0, sizeof(tmap));
  IndexMmaArgs a{false, q_ix, w, Q, q_pos, cand, P, P, c, nullptr, err, chunk, k, sel};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, rows);
  cfg.blockDim = dim3(IM_THREADS);
  cfg.dynamicSmemBytes = IM_SEL_SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = cs;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, index_score_mma_kernel<true>, tmap, a);
}

}  // namespace csa2
