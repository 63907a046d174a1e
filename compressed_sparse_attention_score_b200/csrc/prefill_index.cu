// K4: the prefill indexer with its causal top-k fused in (no score matrix).
//
// CTA = PF_Q consecutive query tokens of one sequence x every key tile any of them sees.
// A 128-entry key tile is loaded once (one TMA box of the codes plus the scale words, or
// cp.async gathers for caches a tensor map cannot describe) and serves all PF_Q queries: their
// 64 heads each are one B operand (N = 64 PF_Q, one scale atom), two K=64 block-scaled FP4
// MMAs (tcgen05 kind::mxf4) per tile, query g's accumulator in columns 64 g ..  Two CTAs
// share an SM (each holds 256 TMEM columns and a 4-stage ring), so one CTA's tensor-core and
// load phases fill the other's epilogue gaps; the epilogue hands the accumulator back as soon
// as it has read it.  Warp roles:
//   warp 0       producer;
//   warp 1       MMA issuer (one lane);
//   warps 2-..   one epilogue warpgroup per query: the weighted-ReLU score of each of its 128
//                keys per tile (the decode kernel's arithmetic, so both give the same fp32
//                score); keys the query cannot see are dropped, keys above the query's running
//                threshold are appended to its candidate list in shared memory.
// A list that could overflow on the next tile is cut back to its best k candidates (radix
// selection on the scores' order-preserving keys), and its threshold becomes the k-th key: a
// later key equal to it has a higher entry index and loses the tie.  At the end each query keeps
// its best k (score descending, entry ascending), written in ascending entry order and padded
// with -1 -- the selection csa2_topk makes from materialised scores.
// Every mbarrier wait is time-bounded; on expiry the CTA drains and reports CSA2_ERR_TIMEOUT.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace csa2 {
using namespace sm100;

namespace {
constexpr int PF_Q = 2;                 // query tokens per CTA = epilogue warpgroups
constexpr int PF_STAGES = 4;
constexpr int PF_TILE = 128;            // keys per tile = MMA M
constexpr int PF_N = 64;                // indexer heads = MMA N
constexpr int PF_A_BYTES = PF_TILE * 64;
constexpr int PF_STAGE_BYTES = 9216;    // 8192 codes + 512 scale atom, padded to 1024
constexpr int PF_WG = 128;              // threads per epilogue warpgroup
constexpr int PF_THREADS = 64 + PF_Q * PF_WG;
constexpr int PF_CAP = 2048;            // candidate list per query
constexpr int PF_KMAX = 512;
constexpr uint32_t PF_TMEM_COLS = 256;   // two CTAs per SM share the 512 columns
constexpr int PF_ACC = 1;               // accumulator sets (the other CTA on the SM fills the gaps)
constexpr uint32_t PF_COL_SFA = PF_ACC * PF_Q * 64;    // after the accumulator sets
constexpr uint32_t PF_COL_SFB = PF_COL_SFA + 4 * PF_ACC;
constexpr uint64_t PF_WAIT_NS = 2000000000ull;
static_assert(PF_COL_SFB + 4 <= PF_TMEM_COLS, "accumulators and scale atoms exceed the TMEM allocation");
static_assert(PF_Q * PF_N <= 256, "the CTA's queries are one MMA's B operand (N <= 256)");

constexpr int PS_STAGES = 0;
constexpr int PS_B = PF_STAGES * PF_STAGE_BYTES;          // PF_Q x [64 heads x 64 B] query codes
constexpr int PS_SFB = PS_B + PF_Q * 4096;                // 512 B scale atom of the PF_Q x 64 B rows
constexpr int PS_W = PS_SFB + 512;                        // PF_Q x 64 fp32 head weights
constexpr int PS_CKEY = PS_W + PF_Q * 256;                // PF_Q x PF_CAP keys
constexpr int PS_CENT = PS_CKEY + PF_Q * PF_CAP * 4;      // PF_Q x PF_CAP entries
constexpr int PS_SCR = PS_CENT + PF_Q * PF_CAP * 4;       // PF_Q x cut scratch: PF_KMAX keys, PF_KMAX entries
constexpr int PS_HIST = PS_SCR + PF_Q * PF_KMAX * 8;      // PF_Q x 256-bin histogram
constexpr int PS_SEL = PS_HIST + PF_Q * 256 * 4;          // PF_Q x selection state (4 words)
constexpr int PS_TCNT = PS_SEL + PF_Q * 16;               // PF_Q x 3 per-tile append counters
constexpr int PS_BAR = PS_TCNT + 64;
constexpr int PF_NBARS = 2 * PF_STAGES + 2 * PF_ACC + 1;
constexpr int PS_MISC = PS_BAR + 8 * PF_NBARS;
constexpr int PS_TOTAL = PS_MISC + 16;
constexpr size_t PF_SMEM = PS_TOTAL + 1024;
}  // namespace

struct PrefillArgs {
  bool use_tma;
  const uint16_t *q_ix;
  const uint16_t *w;
  int Q;
  const int32_t *q_pos;
  int k;
  int max_entries;  // entries a query may see (more: left out, CSA2_ERR_SHAPE)
  csa2_cache c;
  int32_t *idx;  // [B][Q][k]
  int32_t *err;
};

namespace {
__device__ __forceinline__ int pf_row_of_entry(int e) { return (e & 3) * 32 + (e >> 2); }
__device__ __forceinline__ int pf_entry_of_row(int m) { return (m & 31) * 4 + (m >> 5); }

// Named barrier of one epilogue warpgroup (ids 1 .. PF_Q).
__device__ __forceinline__ void wg_sync(int g) { asm volatile("bar.sync %0, %1;" ::"r"(g + 1), "n"(PF_WG) : "memory"); }

// The k-th largest key T of list keys[0..n) (n > k) and how many of the keys equal to T belong
// to the best k (need_eq), by radix selection on 8-bit digits from the top; also whether every
// key equal to T is kept (all_eq).  Called by the PF_WG threads of warpgroup g (t = their index).
__device__ void kth_key(const uint32_t *keys, int n, int k, uint32_t *hist, uint32_t *sel, int t, int g, uint32_t &T,
                        int &need_eq, bool &all_eq) {
  uint32_t prefix = 0;
  int need = k, bin_count = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    hist[t] = 0;
    hist[t + PF_WG] = 0;
    wg_sync(g);
    const uint32_t himask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
    // scores crowd into few bins: lanes with the same bin add once (warp-aggregated)
    const int lane = t & 31;
    for (int i = t; i - lane < n; i += PF_WG) {
      const uint32_t key = i < n ? keys[i] : 0u;
      const bool act = i < n && (key & himask) == prefix;
      const uint32_t am = __ballot_sync(0xffffffffu, act);
      if (act) {
        const uint32_t bin = (key >> shift) & 255u, peers = __match_any_sync(am, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], uint32_t(__popc(peers)));
      }
    }
    wg_sync(g);
    if (t < 32) {  // one warp finds the digit at which the count from the top reaches `need`
      uint32_t c8[8], s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) s += (c8[j] = hist[255 - (8 * t + j)]);
      uint32_t x = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (t >= o) x += y;
      }
      const uint32_t excl = x - s;
      const int L = __ffs(__ballot_sync(0xffffffffu, excl < uint32_t(need) && x >= uint32_t(need))) - 1;
      if (t == L) {
        uint32_t cum = excl;
#pragma unroll 1
        for (int j = 0; j < 8; ++j) {
          if (cum + c8[j] >= uint32_t(need)) {
            sel[0] = uint32_t(255 - (8 * t + j));
            sel[1] = uint32_t(need) - cum;
            sel[2] = c8[j];
            break;
          }
          cum += c8[j];
        }
      }
    }
    wg_sync(g);
    prefix |= sel[0] << shift;
    need = int(sel[1]);
    bin_count = int(sel[2]);
    wg_sync(g);  // sel and hist are rewritten by the next digit
  }
  T = prefix;
  need_eq = need;
  all_eq = bin_count == need;
}

// Cut a query's list (keys, ents; n > k entries) back to its best k (key descending, entry
// ascending) through the scratch and return the k-th key, the list's new threshold.  Ties on
// that key are resolved by counting, for each, the tied keys with smaller entries (only when
// not all of them are kept).  Called by the PF_WG threads of warpgroup g; contains wg_sync.
__device__ uint32_t cut_to_k(uint32_t *keys, int32_t *ents, int n, int k, uint32_t *scr_key, int32_t *scr_ent,
                             uint32_t *hist, uint32_t *sel, int t, int g) {
  uint32_t T;
  int need_eq;
  bool all_eq;
  kth_key(keys, n, k, hist, sel, t, g, T, need_eq, all_eq);
  if (t == 0) sel[3] = 0;
  wg_sync(g);
  const int lane = t & 31;
  for (int i = t; i - lane < n; i += PF_WG) {
    const uint32_t key = i < n ? keys[i] : 0u;
    bool keep = i < n && key > T;
    if (i < n && key == T) {
      if (all_eq) {
        keep = true;
      } else {
        const int e = ents[i];
        int before = 0;
        for (int j = 0; j < n; ++j) before += (keys[j] == T && ents[j] < e);
        keep = before < need_eq;
      }
    }
    const uint32_t km = __ballot_sync(0xffffffffu, keep);
    uint32_t base = 0;
    if (lane == 0 && km) base = atomicAdd(&sel[3], uint32_t(__popc(km)));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (keep) {
      const int s = int(base) + __popc(km & ((1u << lane) - 1u));
      scr_key[s] = key;
      scr_ent[s] = ents[i];
    }
  }
  wg_sync(g);
  for (int i = t; i < k; i += PF_WG) {
    keys[i] = scr_key[i];
    ents[i] = scr_ent[i];
  }
  wg_sync(g);
  return T;
}
}  // namespace

__global__ void __launch_bounds__(PF_THREADS, 2) prefill_index_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                      PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + PS_BAR);
  uint64_t *empty = full + PF_STAGES;
  uint64_t *acc_full = empty + PF_STAGES;
  uint64_t *acc_empty = acc_full + PF_ACC;
  uint64_t *done = acc_empty + PF_ACC;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + PS_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + PS_MISC + 4);
  float *ws = reinterpret_cast<float *>(smem + PS_W);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  grid_dep_launch();  // a dependent attention launch may start its prologue
  const int b = blockIdx.y, q0 = blockIdx.x * PF_Q;
  const int nq = min(PF_Q, a.Q - q0);  // query tokens of this CTA
  int nvis_max = 0;
  int nvis[PF_Q];
#pragma unroll
  for (int qi = 0; qi < PF_Q; ++qi) {
    nvis[qi] = qi < nq ? visible_entries(a.c, b, a.q_pos[int64_t(b) * a.Q + q0 + qi]) : 0;
    if (nvis[qi] > a.max_entries) {
      if (threadIdx.x == 0) report(a.err, CSA2_ERR_SHAPE);
      nvis[qi] = a.max_entries;
    }
    nvis_max = max(nvis_max, nvis[qi]);
  }
  const int ntiles = (nvis_max + PF_TILE - 1) / PF_TILE;

  // ---------------------------------------------------------------- prologue
  if (warp == 0) {
    tmem_alloc(tmem_slot, PF_TMEM_COLS);
    tmem_relinquish();
  } else if (warp == 1 && lane == 0) {
    for (int s = 0; s < PF_STAGES; ++s) {
      mbar_init(&full[s], a.use_tma ? 1 : 32);  // gather path: one cp.async arrival per producer lane
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < PF_ACC; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], PF_Q * 4);  // every epilogue warp
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    mbar_init_fence();
  } else if (warp >= 2) {
    // quantise the query heads (MXFP4, as the decode kernel): item (qi, h, pair of 32-blocks)
    const int t = threadIdx.x - 64;
    for (int item = t; item < PF_Q * 128; item += PF_Q * PF_WG) {
      const int qi = item >> 7, h = (item >> 1) & 63, g0 = 2 * (item & 1);
      uint8_t *brow = smem + PS_B + qi * 4096 + h * 64;
      uint32_t sfpart = 0;
      const uint16_t *qh = a.q_ix + ((int64_t(b) * a.Q + q0 + min(qi, nq - 1)) * HI + h) * DI;
#pragma unroll 1
      for (int g = g0; g < g0 + 2; ++g) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 u = reinterpret_cast<const uint4 *>(qh + 32 * g)[i];
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
        *reinterpret_cast<uint4 *>(brow + ((g ^ ((h >> 1) & 3)) << 4)) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        sfpart |= uint32_t(ex + 127) << (8 * g);
      }
      const uint32_t sfword = sfpart | __shfl_xor_sync(0xffffffffu, sfpart, 1);
      if ((item & 1) == 0) {  // B row 64 qi + h: lane-row r % 32, column r / 32 of the atom
        const int r = 64 * qi + h;
        *reinterpret_cast<uint32_t *>(smem + PS_SFB + (r & 31) * 16 + (r >> 5) * 4) = sfword;
        ws[qi * 64 + h] = bf16_to_f32(a.w[(int64_t(b) * a.Q + q0 + min(qi, nq - 1)) * HI + h]);
      }
    }
    if (t < PF_Q * 3) reinterpret_cast<uint32_t *>(smem + PS_TCNT)[t] = 0;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    const uint32_t stages = smem_u32(smem + PS_STAGES);
    if (a.use_tma) {
      if (lane == 0) {
        for (int i = 0; i < ntiles; ++i) {
          const int s = i % PF_STAGES;
          if (!mbar_wait_bounded(&empty[s], ((i / PF_STAGES) & 1) ^ 1, abort_flag, PF_WAIT_NS)) break;
          const uint32_t st = stages + s * PF_STAGE_BYTES;
          const int64_t slot0 = cache_slot(a.c, b, int64_t(i) * PF_TILE);
          if (slot0 >= 0 && (slot0 & (PF_TILE - 1)) == 0 && slot0 + PF_TILE <= a.c.num_slots) {
            mbar_arrive_expect_tx(&full[s], PF_A_BYTES + 512);
            tma_load_4d(st, &tmap, 0, 0, 0, int(slot0 / PF_TILE), &full[s]);
            bulk_load(st + PF_A_BYTES, a.c.ix_scales + slot0 * CSA2_IX_SCALE_BYTES, 512, &full[s]);
          } else {
            report(a.err, CSA2_ERR_INDEX);  // a visible tile without a valid page: the epilogue drops it
            mbar_arrive(&full[s]);
          }
        }
      }
    } else {
      // gather: lane l copies the 16-byte pieces of entries l, l + 32, l + 64, l + 96
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % PF_STAGES;
        if (!mbar_wait_bounded(&empty[s], ((i / PF_STAGES) & 1) ^ 1, abort_flag, PF_WAIT_NS)) break;
        const uint32_t st = stages + s * PF_STAGE_BYTES;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = lane + 32 * j, n = i * PF_TILE + e, m = pf_row_of_entry(e);
          const int64_t slot = n < nvis_max ? cache_slot(a.c, b, n) : -1;
          if (slot >= 0) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              cp_async_16(st + m * 64 + ((c ^ ((m >> 1) & 3)) << 4), a.c.ix_codes + slot * CSA2_IX_CODE_BYTES + c * 16);
            cp_async_4(st + PF_A_BYTES + e * 4, a.c.ix_scales + slot * CSA2_IX_SCALE_BYTES);
          } else if (n < nvis_max) {
            report(a.err, CSA2_ERR_INDEX);
          }
        }
        cp_async_arrive_noinc(&full[s]);
      }
      cp_async_wait<0>();
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t stages = smem_u32(smem + PS_STAGES);
      // the CTA's queries are one B operand (query qi = rows 64 qi .. 64 qi + 63), one MMA per K half
      const uint32_t bq = smem_u32(smem + PS_B);
      tc_cp_32x128b_warpx4(tmem + PF_COL_SFB, smem_desc(smem_u32(smem + PS_SFB), 16, 128, LAYOUT_SWIZZLE_NONE));
      const uint64_t bd0 = smem_desc(bq, 16, 512, LAYOUT_SWIZZLE_64B);
      const uint64_t bd1 = smem_desc(bq + 32, 16, 512, LAYOUT_SWIZZLE_64B);
      constexpr uint32_t id0 = idesc_mxf4(PF_TILE, PF_Q * PF_N, 0, 0);
      constexpr uint32_t id1 = idesc_mxf4(PF_TILE, PF_Q * PF_N, 2, 2);
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % PF_STAGES, buf = i % PF_ACC;
        if (!mbar_wait_bounded(&full[s], (i / PF_STAGES) & 1, abort_flag, PF_WAIT_NS)) break;
        if (!mbar_wait_bounded(&acc_empty[buf], ((i / PF_ACC) & 1) ^ 1, abort_flag, PF_WAIT_NS)) break;
        if (!a.use_tma) fence_proxy_async_smem();  // cp.async-filled stages are read by the tensor core
        tc_fence_after();
        const uint32_t st = stages + s * PF_STAGE_BYTES;
        const uint32_t sfa = tmem + PF_COL_SFA + 4 * buf;
        tc_cp_32x128b_warpx4(sfa, smem_desc(st + PF_A_BYTES, 16, 128, LAYOUT_SWIZZLE_NONE));
        const uint64_t a0 = smem_desc(st, 16, 512, LAYOUT_SWIZZLE_64B);
        const uint64_t a1 = smem_desc(st + 32, 16, 512, LAYOUT_SWIZZLE_64B);
        const uint32_t d = tmem + buf * PF_Q * PF_N;
        tc_mma_mxf4(d, a0, bd0, id0, sfa, tmem + PF_COL_SFB, false);
        tc_mma_mxf4(d, a1, bd1, id1, sfa, tmem + PF_COL_SFB, true);
        tc_commit(&empty[s]);
        tc_commit(&acc_full[buf]);
      }
      tc_commit(done);
      const uint64_t t_start = globaltimer();
      while (!mbar_try_wait(done, 0) && globaltimer() - t_start < PF_WAIT_NS) {
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    // Warpgroup g scores query g of every tile and keeps its candidate list; the warpgroups
    // never wait for one another.  Per tile the warps append with one shared-memory atomic on
    // the tile's counter (counters rotate over three tiles, so one is zeroed while another is
    // read and a third filled), then meet once; every thread adds the tile's count to its own
    // copy of the list length, so cut decisions are uniform without a second barrier.
    const int g = (warp - 2) >> 2, t = threadIdx.x - 64 - PF_WG * g;
    const int q4 = warp & 3;
    const int e = pf_entry_of_row(32 * q4 + lane);  // tile entry of this thread's accumulator row
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem + PS_CKEY) + g * PF_CAP;
    int32_t *ents = reinterpret_cast<int32_t *>(smem + PS_CENT) + g * PF_CAP;
    uint32_t *scr_key = reinterpret_cast<uint32_t *>(smem + PS_SCR + g * PF_KMAX * 8);
    int32_t *scr_ent = reinterpret_cast<int32_t *>(smem + PS_SCR + g * PF_KMAX * 8 + PF_KMAX * 4);
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem + PS_HIST) + g * 256;
    uint32_t *sel = reinterpret_cast<uint32_t *>(smem + PS_SEL) + g * 4;
    uint32_t *tcnt = reinterpret_cast<uint32_t *>(smem + PS_TCNT) + g * 3;
    const float4 *w4 = reinterpret_cast<const float4 *>(ws + g * 64);
    int qv = 0;  // entries this query sees (0 past the chunk's end)
#pragma unroll
    for (int qi = 0; qi < PF_Q; ++qi)
      if (qi == g) qv = nvis[qi];
    int cnt = 0;                    // list length (the same in every thread of the warpgroup)
    uint32_t thr = KEY_NEG_INF;     // keys must exceed this to enter the list
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int buf = i % PF_ACC;
      if (ok && !mbar_wait_bounded(&acc_full[buf], (i / PF_ACC) & 1, abort_flag, PF_WAIT_NS)) ok = false;
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld is taken by the whole warp or not at all
      float sc = 0.f;
      if (ok) {  // (uniform in the warp)
        tc_fence_after();
        const uint32_t taddr = tmem + (uint32_t(32 * q4) << 16) + (buf * PF_Q + g) * PF_N;
        uint32_t r0[32], r1[32];
        tc_ld_32x32b_x32(taddr, r0);
        tc_ld_32x32b_x32(taddr + 32, r1);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);  // the next tile's products may start now
        sc = weighted_relu_score(r0, r1, w4);         // the decode kernel's arithmetic: the same score
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
      }
      // append the keys above the threshold; an entry without a valid page is never a
      // candidate (its error is already reported)
      const int n = i * PF_TILE + e;
      const uint32_t key = score_key(sc);
      const bool pass = ok && n < qv && key > thr && cache_slot(a.c, b, n) >= 0;
      const uint32_t m = __ballot_sync(0xffffffffu, pass);
      if (m) {
        uint32_t base = 0;
        if (lane == 0) base = atomicAdd(&tcnt[i % 3], uint32_t(__popc(m)));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (pass) {
          const int at = cnt + int(base) + __popc(m & lt_mask);
          keys[at] = key;
          ents[at] = n;
        }
      }
      if (t == 0) tcnt[(i + 1) % 3] = 0;  // last read after tile i - 2's barrier, next filled after this one
      wg_sync(g);
      cnt += int(tcnt[i % 3]);
      if (cnt > PF_CAP - PF_TILE) {  // the next tile could overflow: cut to the best k
        thr = cut_to_k(keys, ents, cnt, a.k, scr_key, scr_ent, hist, sel, t, g);
        cnt = a.k;
      }
    }
    // final: the query's best k, in ascending entry order, -1 padded
    if (g < nq) {
      if (cnt > a.k) {
        cut_to_k(keys, ents, cnt, a.k, scr_key, scr_ent, hist, sel, t, g);
        cnt = a.k;
      }
      int32_t *orow = a.idx + (int64_t(b) * a.Q + q0 + g) * a.k;
      for (int j = t; j < cnt; j += PF_WG) {
        const int ej = ents[j];
        int rank = 0;
        for (int l = 0; l < cnt; ++l) rank += ents[l] < ej;
        orow[rank] = ej;
      }
      for (int j = cnt + t; j < a.k; j += PF_WG) orow[j] = -1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, PF_TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) report(a.err, CSA2_ERR_TIMEOUT);
}

void launch_prefill_index(const uint16_t *q_ix, const uint16_t *w, int B, int Q, const int32_t *q_pos, int k,
                          int max_entries, const csa2_cache &c, int32_t *idx, int32_t *err, cudaStream_t st) {
  if (B == 0 || Q == 0) return;
  CUtensorMap tmap;
  memset(&tmap, 0, sizeof(tmap));
  const bool use_tma = make_index_code_map(&tmap, c);
  PrefillArgs a{use_tma, q_ix, w, Q, q_pos, k, max_entries, c, idx, err};
  set_smem_limit(prefill_index_kernel, PF_SMEM);
  prefill_index_kernel<<<dim3((Q + PF_Q - 1) / PF_Q, B), PF_THREADS, PF_SMEM, st>>>(tmap, a);
}

}  // namespace csa2
