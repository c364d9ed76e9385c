// indexer.cu -- the lightweight indexer on tcgen05 tensor cores.
//
// score(t, s) = sk[s] * sum_h w'[t,h] * ReLU(acc[s, (t,h)]),  w' = w * sq
// acc[s, (t,h)] = e4m3(k[s]) . e4m3(q[t,h])  (or bf16), fp32 in TMEM.
//
// Token sparse attention's indexer (Latent Sparse Attention section 2.1)
// scores every visible key of every query. The contraction over d runs on the
// tensor cores with KEYS on the MMA M dimension (128 TMEM lanes = 128 keys)
// and (query, head) pairs on N, so each epilogue thread owns one key and the
// ReLU + head-weighted reduction is a thread-local loop over TMEM columns
// (no cross-lane reduction). The scales factor out of the ReLU because they
// are positive: ReLU(sq*sk*a) = sq*sk*ReLU(a).
//
// Roles: warp 0 = TMA producer (one lane), warp 1 = MMA issuer (one lane)
// and TMEM owner, warps 2..17 = epilogue teams, warp 18 = metadata stager.
// Prefill and grouped CTAs are persistent (one per SM): each loops over its
// work units with two query buffers and two metadata buffers, so the next
// unit's query tile (TMA) and weights (the stager) load while one runs and
// no unit pays a CTA's setup and drain. The 512 TMEM columns hold
// 512 / N fp32 accumulators (2 at N = 256, 8 at N = 64) used as a ring; team
// b % TEAMS drains buffer b, so the epilogue of one accumulator overlaps the
// MMAs into the others (the pages' bucket scan also overlaps its epilogue
// with its products: appendix F.1, "Flat prefill"). A team has 4 warps per
// accumulator column slice, one per TMEM lane quarter: the wide modes (N =
// 256 = 4 queries x 64 heads) run 2 teams of 8 warps, each warp draining one
// 128-column slice (2 queries); the narrow modes (N = 64, one query) run 4
// teams of 4 warps. On sm_100a one M = 128, K = 32 FP8 MMA costs about the
// same ~97 cycles for any N up to 128 and ~128 cycles at N = 256, so N = 256
// doubles the work per instruction for a third more time.
//
// Key sources (template MODE):
//   IDX_PREFILL  keys [0, lim] of one sequence, NQ consecutive query rows per
//                CTA in G sub-tiles of QS queries (N = QS*H <= 256)
//   IDX_DECODE   one query per sequence, a span of that sequence's key tiles
//   IDX_GATHER   per query, the 64-key blocks it kept (two-stage stage 2);
//                a tile = two kept blocks, N = H
//   IDX_GROUPED  per group of 8 queries, the union of their kept blocks
//                (two-stage stage 2): a tile = two union blocks, scored for
//                QS queries at a time (N = 256); each score goes to the
//                query's own candidate column if it kept the block
// Output: the fp32 score of every (row, key) of the processed tiles, -inf
// where the key is not visible, into a row-major table.
#include <cstdio>

#include "ptx.cuh"
#include "sa_internal.h"

namespace sa {

// Tuning knobs (compile-time): queries per gather CTA and key-tile ring depth.
#ifndef SA_IDX_GATHER_NQ
#define SA_IDX_GATHER_NQ 8
#endif
#ifndef SA_IDX_STAGES
#define SA_IDX_STAGES 6
#endif
// key-tile ring depth of the persistent modes (their two query buffers take
// the shared memory of the other stages)
#ifndef SA_IDX_STAGES_PERSIST
#define SA_IDX_STAGES_PERSIST 5
#endif
// FP8 prefill: sub-tiles of QS queries per CTA (each key tile serves G jobs)
#ifndef SA_IDX_PREFILL_G
#define SA_IDX_PREFILL_G 2
#endif
// the wide modes' MMA N (256 or 128) and their epilogue teams (16 warps in
// 2 or 4 teams; every team owns whole accumulators, so 4 teams need N = 128)
#ifndef SA_IDX_PREFILL_N
#define SA_IDX_PREFILL_N 256
#endif
#ifndef SA_IDX_TEAMS_WIDE
#define SA_IDX_TEAMS_WIDE 2
#endif
constexpr int kIdxEpiWarps = 16;                              // epilogue warps of every mode
constexpr int kIdxThreads = 64 + 32 * kIdxEpiWarps + 32;      // + the staging warp of the persistent modes
// independent partial sums per query in the epilogue when N holds several queries
#ifndef SA_IDX_NP_WIDE
#define SA_IDX_NP_WIDE 2
#endif
// epilogue math: 1 = (w/2) * (a + |a|) accumulated with packed f32x2 FMAs
#ifndef SA_IDX_EPI_PACKED
#define SA_IDX_EPI_PACKED 1
#endif
// FP8 (16x256b) epilogue math per head: 0 = (w/2)(a + |a|) in packed f32x2
// FMAs, 1 = the same in scalar FMAs, 2 = w * max(a, 0) in scalar FMAs
#ifndef SA_IDX_QUAD_MATH
#define SA_IDX_QUAD_MATH 0
#endif

template <int H, int D, bool FP8, int MODE>
struct IdxCfg {
  static constexpr int ESZ = FP8 ? 1 : 2;
  static constexpr int ROWB = D * ESZ;                       // bytes per index row
  static constexpr bool WIDE = MODE == IDX_PREFILL || MODE == IDX_GROUPED;   // N = QS queries x H heads
  static constexpr int QS = WIDE ? (SA_IDX_PREFILL_N / H) : 1;
  static constexpr int N = QS * H;                           // MMA N
  static constexpr int G = (MODE == IDX_PREFILL)   ? (QS * 2 < 8 ? 8 / QS : SA_IDX_PREFILL_G)
                           : (MODE == IDX_GROUPED) ? (kGroupQueries / QS > 0 ? kGroupQueries / QS : 1)
                                                   : 1;      // sub-tiles per CTA
  static constexpr int NQ = (MODE == IDX_PREFILL)   ? QS * G
                            : (MODE == IDX_GATHER)  ? SA_IDX_GATHER_NQ
                            : (MODE == IDX_GROUPED) ? kGroupQueries
                                                    : 1;
  static constexpr int NBUF = 512 / N;                       // TMEM accumulator buffers (fp32 columns)
  static constexpr int TEAMS = WIDE ? SA_IDX_TEAMS_WIDE : 4;
  static constexpr int WPT = kIdxEpiWarps / TEAMS;           // warps per team
  static constexpr int SLICES = WPT / 4;                      // column slices of an accumulator
  static constexpr int SCOLS = N / SLICES;                    // columns one warp drains per job
  static constexpr int QSW = QS / SLICES;                     // queries one warp drains per job
  static constexpr int THREADS = kIdxThreads;
  static_assert(NBUF % TEAMS == 0, "every team owns whole accumulators");
  static_assert(WPT % 4 == 0 && QS % SLICES == 0 && SCOLS == QSW * H, "a warp drains whole queries");
  // prefill and grouped CTAs are persistent: each loops over work units (a
  // block of NQ rows, a query group) with two query buffers and two metadata
  // buffers, so the next unit's queries and weights load while one runs
  static constexpr bool PERSIST = MODE == IDX_PREFILL || MODE == IDX_GROUPED;
  static constexpr int QB = PERSIST ? 2 : 1;                  // query / metadata buffers
  static constexpr int QBYTES = NQ * H * ROWB;
  static constexpr int KBYTES = 128 * ROWB;
  static constexpr int NS = (MODE == IDX_DECODE) ? 8 : PERSIST ? SA_IDX_STAGES_PERSIST : SA_IDX_STAGES;
  static constexpr int KSTEPS = ROWB / 32;                   // 32-byte K slices per MMA
  static constexpr int KEEPMAX = 64;                          // gather: kept blocks per query
  static constexpr int GU = kGroupQueries * KEEPMAX;          // grouped: union blocks per group (at most)
  // gather: kept lists; grouped: union blocks, their slot words and the
  // group's queries; other modes: the rows' thetas (candidate mode); 16-byte multiple
  static constexpr int KEPT_BYTES = (MODE == IDX_GATHER)    ? NQ * KEEPMAX * 4
                                    : (MODE == IDX_GROUPED) ? GU * 8 + GU * 4 + 64
                                                            : (NQ * 4 + 15) / 16 * 16;
  static constexpr int WBYTES = NQ * H * 4;                    // the unit's weights
  static constexpr int META = WBYTES + KEPT_BYTES;              // one metadata buffer
  static constexpr int NBAR = 2 * NS + 4 * QB + 2 * NBUF;
  static constexpr int SMEM_USED = 1024 + QB * QBYTES + NS * KBYTES + QB * META + NBAR * 8 + 16;
  static_assert(SMEM_USED <= 227 * 1024, "shared memory");
  static_assert(WBYTES % 16 == 0 && KEPT_BYTES % 16 == 0, "metadata alignment");
  // at least 120 KB: one CTA per SM, so two CTAs never contend for TMEM
  static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static_assert(N <= 256 && N % 16 == 0, "MMA N");
  static_assert(MODE != IDX_GROUPED || QS * G == kGroupQueries, "one group per CTA");
  static_assert(SCOLS % 32 == 0, "epilogue loads 32 columns at a time");
};

// a compile-time int passed as a value (selects a drain's load range)
template <int V>
struct IntC {
  static constexpr int value = V;
};

__device__ __forceinline__ int vis_limit(int t, const IdxArgs& a) {
  const int p = a.row_pos ? a.row_pos[t] : a.q_pos0 + t;
  return (a.div == 1) ? (p - a.off) : (p / a.div - a.off);
}

// Walks the (query, pair-of-kept-blocks) jobs of a gather CTA in order; every
// role advances its own copy identically. Queries without kept blocks (a
// leading -1) are skipped, so a job never names block -1.
struct GatherCursor {
  const int* kept;
  int keep, q0, nq, ql, pair;
  __device__ void init(const int* k_, int keep_, int q0_, int nq_) {
    kept = k_;
    keep = keep_;
    q0 = q0_;
    nq = nq_;
    ql = 0;
    pair = 0;
    skip_empty();
  }
  __device__ const int* row() const { return kept + (long long)(q0 + ql) * keep; }
  __device__ void skip_empty() {
    while (ql < nq && row()[0] < 0) ++ql;
  }
  __device__ void next() {
    ++pair;
    if (2 * pair >= keep || row()[2 * pair] < 0) {
      pair = 0;
      ++ql;
      skip_empty();
    }
  }
};

template <int H, int D, bool FP8, int MODE>
__global__ void __launch_bounds__(kIdxThreads, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const IdxArgs a) {
  using C = IdxCfg<H, D, FP8, MODE>;
  constexpr bool PERSIST = C::PERSIST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* sQ0 = smem;                                        // [QB] query tiles
  uint8_t* sK = sQ0 + C::QB * C::QBYTES;                       // [NS] key tiles
  uint8_t* sMeta0 = sK + C::NS * C::KBYTES;                    // [QB] per-unit metadata
  uint64_t* bars = reinterpret_cast<uint64_t*>(sMeta0 + C::QB * C::META);
  uint64_t* kfull = bars;
  uint64_t* kempty = kfull + C::NS;
  uint64_t* qfull = kempty + C::NS;    // [QB] the unit's query tile landed
  uint64_t* qempty = qfull + C::QB;    // [QB] the MMAs of the unit that read the buffer are done
  uint64_t* mfull = qempty + C::QB;    // [QB] the unit's metadata is staged
  uint64_t* mempty = mfull + C::QB;    // [QB] the epilogue is done with it
  uint64_t* tfull = mempty + C::QB;
  uint64_t* tempty = tfull + C::NBUF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + C::NBUF);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  // metadata buffer b: the weights (halved: the packed math sums (w / 2) *
  // (a + |a|)), then gather: kept lists [NQ][KEEPMAX], -1 padded; grouped: [GU]
  // slot words, [GU] union blocks, [NQ] the group's queries; prefill: the
  // rows' thetas (candidate mode)
  struct Meta {
    float* w;
    int* kept;
    float* theta;
    unsigned long long* uslot;
    int* ublk;
    int* qt;
  };
  auto meta = [&](int b) {
    uint8_t* m = sMeta0 + b * C::META;
    Meta r;
    r.w = reinterpret_cast<float*>(m);
    r.kept = reinterpret_cast<int*>(m + C::WBYTES);
    r.theta = reinterpret_cast<float*>(m + C::WBYTES);
    r.uslot = reinterpret_cast<unsigned long long*>(m + C::WBYTES);
    r.ublk = reinterpret_cast<int*>(r.uslot + C::GU);
    r.qt = r.ublk + C::GU;
    return r;
  };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kStagerWarp = 2 + kIdxEpiWarps;

  // ---------------- work units (identical in every role) ----------------
  const int n_rows = (a.row_count != nullptr) ? min(a.n_q, *a.row_count - a.row_base) : a.n_q;
  int n_units = 1;
  if constexpr (MODE == IDX_PREFILL) n_units = (a.n_q + C::NQ - 1) / C::NQ;
  if constexpr (MODE == IDX_GROUPED) n_units = a.n_groups;
  // the it-th unit of this CTA (-1: none left). Persistent CTAs take units
  // round-robin, prefill in descending row order (the latest rows see the most
  // keys) and alternating direction per round, which evens out their work
  auto unit_at = [&](int it) -> int {
    if constexpr (PERSIST) {
      const int pos = (MODE == IDX_PREFILL && (it & 1)) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x;
      const long long idx = (long long)it * gridDim.x + pos;
      if (idx >= n_units) return -1;
      return MODE == IDX_PREFILL ? n_units - 1 - (int)idx : (int)idx;
    } else {
      return it == 0 ? (int)blockIdx.x : -1;
    }
  };
  struct UnitP {
    int q0, nq, seq, tile0, ntiles, geff, njobs, n_ub, seq_len;
  };
  int gather_njobs = 0;                // gather: counted from the staged kept lists
  auto unit_params = [&](int unit) {
    UnitP u;
    u.q0 = 0;
    u.nq = 0;
    u.seq = 0;
    u.tile0 = 0;
    u.ntiles = 0;
    u.geff = 1;
    u.njobs = 0;
    u.n_ub = 0;
    u.seq_len = a.n_k;
    if constexpr (MODE == IDX_PREFILL) {
      u.q0 = unit * C::NQ;
      u.nq = min(C::NQ, n_rows - u.q0);
      if (u.nq > 0) {                  // else past the rows flagged on the device
        u.geff = (u.nq + C::QS - 1) / C::QS;
        const int lim = min(vis_limit(u.q0 + u.nq - 1, a), a.n_k - 1);
        u.tile0 = a.tile_lo;           // the key tiles [tile_lo, min(tile_hi, lim / 128 + 1))
        u.ntiles = (lim < 0) ? 0 : max(0, min(lim / 128 + 1, a.tile_hi) - u.tile0);
        u.njobs = u.ntiles * u.geff;
      }
    } else if constexpr (MODE == IDX_DECODE) {
      u.seq = blockIdx.y;
      u.q0 = u.seq;
      u.nq = 1;
      u.seq_len = a.seq_lens ? min(a.seq_lens[u.seq], a.span) : a.span;
      const int total = (u.seq_len + 127) / 128;
      u.tile0 = blockIdx.x * a.tiles_per_cta;
      u.ntiles = max(0, min(a.tiles_per_cta, total - u.tile0));
      u.njobs = u.ntiles;
    } else if constexpr (MODE == IDX_GROUPED) {
      u.q0 = unit * C::NQ;             // the group's slice of perm
      u.nq = C::NQ;
      u.geff = C::G;
      int nv = 0;
      for (int ql = 0; ql < C::NQ; ++ql) {
        const int t = a.perm[u.q0 + ql];
        nv += (t >= 0 && t < a.n_q) ? 1 : 0;
      }
      u.n_ub = a.gb_n[unit];
      u.ntiles = (nv > 0) ? (u.n_ub + 1) / 2 : 0;   // absent queries only: no jobs
      u.njobs = u.ntiles * u.geff;
    } else {
      u.q0 = unit * C::NQ;
      u.nq = min(C::NQ, a.n_q - u.q0);
      u.njobs = u.ntiles = gather_njobs;
    }
    return u;
  };
  // a unit's metadata into buffer m by one warp (the stager): the query rows
  // first (one load per query, shared by shuffles), then every weight and
  // scale load of the lane issued before any is used, so a unit costs about
  // two load latencies however many weights it has
  auto stage_warp = [&](const UnitP& u, const Meta& m) {
    static_assert(C::NQ <= 32 || MODE != IDX_GROUPED, "one query row per lane");
    constexpr int NWI = (C::NQ * H + 31) / 32;
    int myrow = -1;                    // the row of query `lane` (lanes < NQ; NQ <= 32 here)
    if (lane < C::NQ) {
      if constexpr (MODE == IDX_GROUPED) {
        const int t = a.perm[u.q0 + lane];
        myrow = (t >= 0 && t < a.n_q) ? t : -1;
      } else {
        myrow = (lane < u.nq) ? (a.q_rows != nullptr ? a.q_rows[u.q0 + lane] : u.q0 + lane) : -1;
      }
    }
    float wv[NWI], sv[NWI];
#pragma unroll
    for (int k = 0; k < NWI; ++k) {
      const int i = lane + 32 * k, ql = i / H, h = i % H;
      int qrow = (C::NQ <= 32) ? __shfl_sync(0xffffffffu, myrow, ql & 31) : -1;
      if constexpr (C::NQ > 32)        // bf16 prefill with many queries per unit: rows by arithmetic
        qrow = (ql < u.nq) ? (a.q_rows != nullptr ? a.q_rows[u.q0 + ql] : u.q0 + ql) : -1;
      wv[k] = 0.f;
      sv[k] = 1.f;
      if (i < C::NQ * H && qrow >= 0) {
        const long long r = (long long)qrow * H + h;
        wv[k] = a.w[r];
        if (a.q_scale) sv[k] = a.q_scale[r];
      }
    }
#pragma unroll
    for (int k = 0; k < NWI; ++k) {
      const int i = lane + 32 * k;
      const float v = wv[k] * sv[k];
      if (i < C::NQ * H) m.w[i] = SA_IDX_EPI_PACKED ? 0.5f * v : v;
    }
    if constexpr (MODE == IDX_PREFILL) {
      if (a.cand != nullptr)
        for (int i = lane; i < C::NQ; i += 32) m.theta[i] = (i < u.nq) ? a.theta[u.q0 + i] : 0.f;
    }
    if constexpr (MODE == IDX_GROUPED) {
      if (lane < C::NQ) m.qt[lane] = myrow;
      const int gi = u.q0 / C::NQ;
      const int* blk = a.gb_blk + (long long)gi * a.gb_cap;
      const unsigned long long* slot = a.gb_slot + (long long)gi * a.gb_cap;
      for (int i0 = 0; i0 < u.n_ub; i0 += 32 * 8) {   // eight loads of each list in flight per lane
        int bv[8];
        unsigned long long svv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int i = i0 + lane + 32 * k;
          bv[k] = (i < u.n_ub) ? blk[i] : 0;
          svv[k] = (i < u.n_ub) ? slot[i] : 0ull;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int i = i0 + lane + 32 * k;
          if (i < u.n_ub) {
            m.ublk[i] = bv[k];
            m.uslot[i] = svv[k];
          }
        }
      }
    }
  };
  // a unit's metadata into buffer m, by threads tid = 0.. of nthr (the
  // one-unit modes: every thread of the CTA, before the setup barrier)
  auto stage = [&](const UnitP& u, const Meta& m, int tid, int nthr) {
    for (int i = tid; i < C::NQ * H; i += nthr) {
      const int ql = i / H, h = i % H;
      float v = 0.f;
      int qrow = (ql < u.nq) ? (a.q_rows != nullptr ? a.q_rows[u.q0 + ql] : u.q0 + ql) : -1;
      if constexpr (MODE == IDX_GROUPED) {
        qrow = a.perm[u.q0 + ql];
        if (qrow >= a.n_q) qrow = -1;
      }
      if (qrow >= 0) {
        const long long r = (long long)qrow * H + h;
        v = a.w[r] * (a.q_scale ? a.q_scale[r] : 1.f);
      }
      m.w[i] = SA_IDX_EPI_PACKED ? 0.5f * v : v;
    }
    if constexpr (MODE == IDX_PREFILL) {
      if (a.cand != nullptr)
        for (int i = tid; i < C::NQ; i += nthr) m.theta[i] = (i < u.nq) ? a.theta[u.q0 + i] : 0.f;
    }
    if constexpr (MODE == IDX_GATHER) {
      for (int i = tid; i < C::NQ * C::KEEPMAX; i += nthr) {
        const int ql = i / C::KEEPMAX, j = i % C::KEEPMAX;
        m.kept[i] = (ql < u.nq && j < a.keep) ? a.kept[(long long)(u.q0 + ql) * a.keep + j] : -1;
      }
    }
    if constexpr (MODE == IDX_GROUPED) {
      const int gi = u.q0 / C::NQ;
      for (int i = tid; i < C::NQ; i += nthr) {
        const int t = a.perm[u.q0 + i];
        m.qt[i] = (t >= 0 && t < a.n_q) ? t : -1;
      }
      for (int i = tid; i < u.n_ub; i += nthr) {
        m.ublk[i] = a.gb_blk[(long long)gi * a.gb_cap + i];
        m.uslot[i] = a.gb_slot[(long long)gi * a.gb_cap + i];
      }
    }
  };
  // the key tile i of unit u into ring stage st (the TMA lane)
  auto load_tile = [&](const UnitP& u, int i, int st, GatherCursor& gc) {
    uint8_t* dst = sK + st * C::KBYTES;
    if constexpr (MODE == IDX_PREFILL) {
      mbar_arrive_expect_tx(&kfull[st], C::KBYTES);
      tma_load_2d(dst, &kmap, &kfull[st], 0, (u.tile0 + i) * 128);
    } else if constexpr (MODE == IDX_DECODE) {
      mbar_arrive_expect_tx(&kfull[st], C::KBYTES);
      tma_load_2d(dst, &kmap, &kfull[st], 0, (int)((long long)u.seq * a.n_k + (u.tile0 + i) * 128));
    } else if constexpr (MODE == IDX_GROUPED) {
      const int* blk = a.gb_blk + (long long)(u.q0 / C::NQ) * a.gb_cap;   // the union, read from global memory
      const int b0 = blk[2 * i];
      const int b1 = (2 * i + 1 < u.n_ub) ? blk[2 * i + 1] : -1;
      mbar_arrive_expect_tx(&kfull[st], (b1 >= 0 ? 2 : 1) * 64 * C::ROWB);
      tma_load_2d(dst, &kmap, &kfull[st], 0, b0 * 64);
      if (b1 >= 0) tma_load_2d(dst + 64 * C::ROWB, &kmap, &kfull[st], 0, b1 * 64);
    } else {
      const int* kr = gc.row();
      const int b0 = kr[2 * gc.pair];
      const int b1 = kr[2 * gc.pair + 1];
      mbar_arrive_expect_tx(&kfull[st], (b1 >= 0 ? 2 : 1) * 64 * C::ROWB);
      tma_load_2d(dst, &kmap, &kfull[st], 0, b0 * 64);
      if (b1 >= 0) tma_load_2d(dst + 64 * C::ROWB, &kmap, &kfull[st], 0, b1 * 64);
      gc.next();
    }
  };
  // the query tile of unit u into buffer b (the TMA lane)
  auto load_q = [&](const UnitP& u, int b) {
    uint8_t* q = sQ0 + b * C::QBYTES;
    if constexpr (MODE == IDX_PREFILL) {
      if (a.q_rows != nullptr) {       // listed rows: one box of H rows per query
        mbar_arrive_expect_tx(&qfull[b], u.nq * H * C::ROWB);
        for (int ql = 0; ql < u.nq; ++ql) tma_load_2d(q + ql * H * C::ROWB, &qmap, &qfull[b], 0, a.q_rows[u.q0 + ql] * H);
      } else {
        mbar_arrive_expect_tx(&qfull[b], u.geff * C::QS * H * C::ROWB);
        for (int g = 0; g < u.geff; ++g)
          tma_load_2d(q + g * C::QS * H * C::ROWB, &qmap, &qfull[b], 0, (u.q0 + g * C::QS) * H);
      }
    } else if constexpr (MODE == IDX_GROUPED) {
      int qt[C::NQ], nv = 0;
#pragma unroll
      for (int ql = 0; ql < C::NQ; ++ql) {
        const int t = a.perm[u.q0 + ql];
        qt[ql] = (t >= 0 && t < a.n_q) ? t : -1;
        nv += qt[ql] >= 0;
      }
      mbar_arrive_expect_tx(&qfull[b], nv * H * C::ROWB);
#pragma unroll
      for (int ql = 0; ql < C::NQ; ++ql)   // absent queries leave their rows unset: their scores are dropped
        if (qt[ql] >= 0) tma_load_2d(q + ql * H * C::ROWB, &qmap, &qfull[b], 0, qt[ql] * H);
    } else {
      mbar_arrive_expect_tx(&qfull[b], u.nq * H * C::ROWB);
      for (int ql = 0; ql < u.nq; ++ql) tma_load_2d(q + ql * H * C::ROWB, &qmap, &qfull[b], 0, (u.q0 + ql) * H);
    }
  };

  // ---------------- setup ----------------
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
    }
    for (int b = 0; b < C::QB; ++b) {
      mbar_init(&qfull[b], 1);
      mbar_init(&qempty[b], 1);
      mbar_init(&mfull[b], 32);
      mbar_init(&mempty[b], kIdxEpiWarps);
    }
    for (int b = 0; b < C::NBUF; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::WPT);
    }
    *abort_flag = 0u;
    fence_barrier_init();
    if constexpr (MODE == IDX_DECODE) {
      const int seq = blockIdx.y;
      if (a.seq_lens != nullptr && a.seq_lens[seq] > a.span && blockIdx.x == 0 && a.status != nullptr)
        atomicCAS(a.status, 0u, 1u /* SA_ERR_INVALID_ARGUMENT: a sequence longer than the call's max_len */);
    }
  }
  // the TMA lane (thread 0) issues the first unit's query tile and first ring
  // of key tiles right away, so their latency overlaps the rest of the setup
  // (the staging of the weights and lists, the TMEM allocation)
  int early_it = -1, early = 0;        // the unit (its `it`) and key tiles issued during the setup (thread 0)
  if constexpr (MODE != IDX_GATHER) {
    if (threadIdx.x == 0) {
      for (int it = 0;; ++it) {
        const int unit = unit_at(it);
        if (unit < 0) break;
        const UnitP u = unit_params(unit);
        if (u.njobs == 0) continue;
        prefetch_tmap(&qmap);
        prefetch_tmap(&kmap);
        load_q(u, 0);
        early = min(u.ntiles, C::NS);  // the ring starts empty: no wait
        GatherCursor gc = {};
        for (int i = 0; i < early; ++i) load_tile(u, i, i, gc);
        early_it = it;
        break;
      }
    }
  }
  if (warp == 1) tmem_alloc<512>(tmem_slot);
  if constexpr (!PERSIST) {
    // one unit per CTA: every thread stages it
    const int unit = unit_at(0);
    stage(unit_params(unit), meta(0), threadIdx.x, blockDim.x);
  }
  __syncthreads();
  if constexpr (MODE == IDX_GATHER) {
    const UnitP u = unit_params(unit_at(0));
    const int* kept = meta(0).kept;
    for (int ql = 0; ql < u.nq; ++ql) {
      int nb = 0;
      while (nb < C::KEEPMAX && kept[ql * C::KEEPMAX + nb] >= 0) ++nb;
      gather_njobs += (nb + 1) / 2;
    }
  }
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtx wc{abort_flag, a.status, a.budget};

  if (warp == 0) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      int kc = early;                  // key tiles issued (ring position)
      int qn[C::QB];                   // query tiles issued per buffer
#pragma unroll
      for (int b = 0; b < C::QB; ++b) qn[b] = 0;
      int bi = 0;                      // buffer uses
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int unit = unit_at(it);
        if (unit < 0) break;
        const UnitP u = unit_params(unit);
        if (u.njobs == 0) continue;
        const int b = bi % C::QB, use = bi / C::QB;
        ++bi;
        const bool first = it == early_it;
        if (!first) {
          if (use > 0 && !mbar_wait(&qempty[b], (use - 1) & 1, wc, 6)) break;
          if constexpr (MODE == IDX_GATHER) {
            prefetch_tmap(&qmap);
            prefetch_tmap(&kmap);
          }
          load_q(u, b);
        }
        ++qn[b];
        GatherCursor gc = {};
        if constexpr (MODE == IDX_GATHER) gc.init(meta(0).kept, C::KEEPMAX, 0, u.nq);
        for (int i = first ? early : 0; i < u.ntiles; ++i) {
          const int st = kc % C::NS;
          if (kc >= C::NS && !mbar_wait(&kempty[st], ((kc / C::NS) - 1) & 1, wc, 1)) {
            ok = false;
            break;
          }
          load_tile(u, i, st, gc);
          ++kc;
        }
      }
      // never leave with copies in flight (matters only after an abort):
      // wait, bounded and regardless of the abort flag, for the last loads
      const WaitCtx drain{abort_flag, nullptr, a.budget};
      for (int i = max(0, kc - C::NS); i < kc; ++i) mbar_wait_drain(&kfull[i % C::NS], (i / C::NS) & 1, drain);
#pragma unroll
      for (int b = 0; b < C::QB; ++b)
        if (qn[b] > 0) mbar_wait_drain(&qfull[b], (qn[b] - 1) & 1, drain);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc<FP8 ? 0 : 1, 128, C::N>();
      int kt0 = 0;                     // key tiles of the earlier units (ring position of the unit's first)
      int J = 0;                       // jobs of the earlier units (accumulator ring position)
      int bi = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int unit = unit_at(it);
        if (unit < 0) break;
        const UnitP u = unit_params(unit);
        if (u.njobs == 0) continue;
        const int b = bi % C::QB, use = bi / C::QB;
        ++bi;
        if (!mbar_wait(&qfull[b], use & 1, wc, 2)) break;
        tc_fence_after();
        const uint8_t* sQ = sQ0 + b * C::QBYTES;
        GatherCursor gc;
        if constexpr (MODE == IDX_GATHER) gc.init(meta(0).kept, C::KEEPMAX, 0, u.nq);
        int wtile = 0, wg = 0;         // wide modes: job j = tile * geff + g, advanced without division
        for (int j = 0; j < u.njobs; ++j, ++J) {
          int tile, g;
          if constexpr (C::WIDE) {
            tile = wtile;
            g = wg;
            if (++wg == u.geff) {
              wg = 0;
              ++wtile;
            }
          } else {
            tile = j;
            g = (MODE == IDX_GATHER) ? gc.ql : 0;
          }
          const int kt = kt0 + tile;
          const int st = kt % C::NS;
          const int buf = J % C::NBUF, ub = J / C::NBUF;
          if (g == 0 || !C::WIDE) {
            if (!mbar_wait(&kfull[st], (kt / C::NS) & 1, wc, 3)) {
              ok = false;
              break;
            }
          }
          if (!mbar_wait(&tempty[buf], (ub & 1) ^ 1, wc, 4)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (a.hook == SA_HOOK_STALL_WAIT && J == 0) {            // test hook: never signal job 0
            if constexpr (MODE == IDX_GATHER) gc.next();
            continue;
          }
          const uint32_t d_tmem = tmem_base + buf * C::N;
          // descriptors built once per job; a K step advances the start
          // address field (16-byte units, bits 0-13: no carry below 256 KB)
          const uint64_t ad0 = umma_smem_desc<C::ROWB>(smem_u32(sK + st * C::KBYTES));
          const uint64_t bd0 = umma_smem_desc<C::ROWB>(smem_u32(sQ + g * (C::N * C::ROWB)));
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS; ++ks) {
            const uint64_t ad = ad0 + uint64_t(ks * 32 / 16);
            const uint64_t bd = bd0 + uint64_t(ks * 32 / 16);
            if constexpr (FP8)
              mma_f8(d_tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
            else
              mma_bf16(d_tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
          }
          mma_commit(&tfull[buf]);
          if (!C::WIDE || g == u.geff - 1) mma_commit(&kempty[st]);
          if constexpr (MODE == IDX_GATHER) gc.next();
        }
        if (!ok) break;
        mma_commit(&qempty[b]);        // the buffer is free once this unit's MMAs are done
        kt0 += u.ntiles;
      }
    }
  } else if (warp < kStagerWarp) {
    // ======================= epilogue teams =======================
    const int team = (warp - 2) / C::WPT;    // jobs J with J % TEAMS == team
    const int slice = ((warp - 2) % C::WPT) >> 2;   // the accumulator columns [slice * SCOLS, +SCOLS)
    const int lq = warp & 3;                 // TMEM lane quarter this warp may access
    // FP8 modes drain TMEM with the 16x256b shape: thread (quad r = lane / 4,
    // place c = lane % 4) reads lanes r + 8a + 16h of its quarter and the
    // columns 8i + 2c + e of each 32-column chunk, so it needs the weights of
    // a fixed quarter of the columns only (held in registers) and sums its 16
    // heads of a query per lane; a reduce-scatter over the quad then leaves it
    // the full sums of lane 8c + r. The bf16 modes (4 or 8 heads) read one
    // lane per thread (32x32b) with the weights from shared memory.
    constexpr bool QUAD = FP8;
    const int qr = lane >> 2, qc = lane & 3;
    const int row = lq * 32 + (QUAD ? qr + 8 * qc : lane);   // key row of the tile this thread scores
    // job -> (tile, sub-tile / query, this thread's key, its scale); the scale
    // of the team's next job is loaded one job ahead so its global-load
    // latency hides behind the current job
    struct JobKey {
      int tile, g, ql, pair, s, col;
      bool kvalid;
      float sk;
    };
    // the current unit, as the job lambdas below read it
    int q0 = 0, nq = 0, seq = 0, tile0 = 0, geff = 1, njobs = 0, n_ub = 0, seq_len = a.n_k;
    const float* sW = nullptr;
    const int* sKept = nullptr;
    const float* sTheta = nullptr;
    const unsigned long long* sUSlot = nullptr;
    const int* sUBlk = nullptr;
    const int* sQt = nullptr;
    GatherCursor gc = {};                    // gather: cursor at the job being loaded
    int jq = 0;
    // wide modes: (tile, sub-tile) of the job job_key is asked for next; the
    // team's jobs advance by TEAMS, which moves these without a division
    int ktile = 0, kg = 0;
    auto job_key = [&](int jj) {
      JobKey k;
      if constexpr (MODE == IDX_GATHER) {
        while (jq < jj) {
          gc.next();
          ++jq;
        }
      }
      k.ql = gc.ql;
      k.pair = gc.pair;
      if constexpr (C::WIDE) {
        k.tile = ktile;
        k.g = kg;
        kg += C::TEAMS;
        while (kg >= geff) {
          kg -= geff;
          ++ktile;
        }
      } else {
        k.tile = jj;
        k.g = (MODE == IDX_GATHER) ? k.ql : 0;
      }
      if constexpr (MODE == IDX_GROUPED) {
        const int ub = 2 * k.tile + (row >> 6);
        const int blk = (jj < njobs && ub < n_ub) ? sUBlk[ub] : -1;
        k.s = blk * 64 + (row & 63);
        k.kvalid = blk >= 0 && k.s < a.n_k;
        k.col = ub;                          // the union block: each query's slot of it is looked up per query
      } else if constexpr (MODE == IDX_GATHER) {
        const int slot = 2 * k.pair + (row >> 6);
        const int blk = (k.ql < nq) ? sKept[k.ql * C::KEEPMAX + slot] : -1;
        k.s = blk * 64 + (row & 63);
        k.kvalid = blk >= 0;
        k.col = k.pair * 128 + row;
      } else if constexpr (MODE == IDX_DECODE) {
        k.s = (tile0 + k.tile) * 128 + row;
        k.kvalid = k.s < seq_len;
        k.col = k.s;
      } else {
        k.s = (tile0 + k.tile) * 128 + row;
        k.kvalid = k.s < a.n_k;
        k.col = k.s;
      }
      k.sk = 1.f;
      if (jj < njobs && a.k_scale != nullptr && k.kvalid)
        k.sk = a.k_scale[(long long)seq * a.n_k * (MODE == IDX_DECODE) + k.s];
      return k;
    };
    float2 wq[QUAD ? C::SCOLS / 32 : 1][4];   // 16x256b path: this thread's weights (halved), per chunk and group
    int wg = -1;                             // the sub-tile / query they belong to
    // per query of the warp's slice, fixed while the job's queries are: its
    // causal limit (the last visible key) and, grouped, its output row (-1:
    // none). The FP8 modes (one or two queries per warp) keep them in
    // registers; the bf16 modes (up to 32 queries per warp) recompute them per
    // job, as every mode but grouped does the row (a few integer operations)
    constexpr bool HOIST = QUAD;
    constexpr bool HOIST_T = QUAD && MODE == IDX_GROUPED;
    int tq[HOIST_T ? C::QSW : 1], limq[HOIST ? C::QSW : 1];
    auto query_row = [&](int g_, int ql_, int qq) {
      const int qj = slice * C::QSW + qq;    // the query's place among the job's QS
      int t;
      if constexpr (MODE == IDX_PREFILL)
        t = q0 + g_ * C::QS + qj;
      else if constexpr (MODE == IDX_DECODE)
        t = seq;
      else if constexpr (MODE == IDX_GROUPED)
        t = sQt[g_ * C::QS + qj];
      else
        t = q0 + ql_;
      return (t >= n_rows) ? -1 : t;
    };
    int J0 = 0;                              // jobs of the earlier units
    int bi = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int unit = unit_at(it);
      if (unit < 0) break;
      const UnitP u = unit_params(unit);
      if (u.njobs == 0) continue;
      const int bm = bi % C::QB, usem = bi / C::QB;
      ++bi;
      if (PERSIST && !mbar_wait(&mfull[bm], usem & 1, wc, 7)) break;
      const Meta m = meta(bm);
      sW = m.w;
      sKept = m.kept;
      sTheta = m.theta;
      sUSlot = m.uslot;
      sUBlk = m.ublk;
      sQt = m.qt;
      q0 = u.q0;
      nq = u.nq;
      seq = u.seq;
      tile0 = u.tile0;
      geff = u.geff;
      njobs = u.njobs;
      n_ub = u.n_ub;
      seq_len = u.seq_len;
      wg = -1;                               // new weights and limits
      // this team's first job of the unit: the smallest local j with
      // (J0 + j) % TEAMS == team
      const int jfirst = ((team - J0) % C::TEAMS + C::TEAMS) % C::TEAMS;
      if constexpr (C::WIDE) {
        ktile = jfirst / geff;
        kg = jfirst % geff;
      }
      if constexpr (MODE == IDX_GATHER) {
        gc.init(sKept, C::KEEPMAX, 0, nq);
        jq = 0;
      }
      JobKey nxt = job_key(jfirst);
      for (int j = jfirst; j < njobs; j += C::TEAMS) {
        const JobKey cur = nxt;
        nxt = job_key(j + C::TEAMS);
        const int ql = cur.ql, g = cur.g, s = cur.s, col = cur.col;
        const bool kvalid = cur.kvalid;
        const float sk = cur.sk;
        const int Jg = J0 + j;
        const int buf = Jg % C::NBUF, ub = Jg / C::NBUF;   // buffer buf is always drained by team buf % TEAMS
        if (!mbar_wait(&tfull[buf], ub & 1, wc, 5)) {
          ok = false;
          break;
        }
        tc_fence_after();

      float qsum[C::QSW];                      // sum_h w'[h] * ReLU(acc[h]) of this thread's key row, per query
      // grouped, two queries per warp: the jobs skip queries per warp below,
      // and the slot bytes read for that serve the outputs too
      constexpr bool SPLIT = QUAD && MODE == IDX_GROUPED && C::QSW == 2;
      uint32_t slots2 = 0xFFFFu;
      if (HOIST && g != wg) {                  // the job's queries changed
#pragma unroll
        for (int qq = 0; qq < (HOIST ? C::QSW : 0); ++qq) {
          const int t = query_row(g, ql, qq);
          if constexpr (HOIST_T) tq[qq] = t;
          limq[qq] = (MODE == IDX_DECODE || t < 0) ? 0 : vis_limit(t, a);
        }
      }
      auto release = [&]() {   // every column of this accumulator is in registers
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
      };
      if constexpr (QUAD) {
        constexpr int NCC = C::SCOLS / 32;     // 32-column chunks of the warp's slice (each within one query)
        constexpr int NLD = 2 * NCC;           // loads: (lane half h, chunk)
        static_assert(H % 32 == 0, "a chunk holds heads of one query");
        if (g != wg) {                         // the job's queries changed: their weights of this thread's columns
          const float* wrow = sW + g * C::N + slice * C::SCOLS + 2 * qc;
#pragma unroll
          for (int cc = 0; cc < NCC; ++cc)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              wq[cc][i] = *reinterpret_cast<const float2*>(wrow + cc * 32 + 8 * i);
#if SA_IDX_QUAD_MATH == 2
              wq[cc][i] = make_float2(2.f * wq[cc][i].x, 2.f * wq[cc][i].y);
#endif
            }
        }
        // the warp's queries this job scores (bit qq). A grouped job skips a
        // query that did not keep the block of the warp's rows (its 32 rows lie
        // in one 64-key block): the accumulator columns of that query are
        // neither read nor summed, and its scores are not written.
        constexpr uint32_t FULL = (1u << C::QSW) - 1u;
        uint32_t need = FULL;
        if constexpr (SPLIT) {
          if (s < 0) {
            need = 0u;                         // no union block in this half of the tile
          } else {
            // the slot bytes of the warp's two queries (adjacent in the slot word)
            slots2 = (uint32_t)(sUSlot[col] >> (8 * (g * C::QS + slice * C::QSW))) & 0xFFFFu;
#pragma unroll
            for (int qq = 0; qq < C::QSW; ++qq)
              if (tq[qq] < 0 || ((slots2 >> (8 * qq)) & 0xFFu) == 0xFFu) need &= ~(1u << qq);
          }
        }
        // w * ReLU(a) = (w / 2) * (a + |a|): a + |a| is exact (2a or +0) and one
        // FADD; the halved weights sit in sW, pairs of heads accumulate with
        // f32x2 FMAs. acc2[L][qq]: lane 8L + r, query qq (two accumulators per
        // lane and query, alternating over the column groups, measured slower)
        float2 acc2[4][C::QSW];
#pragma unroll
        for (int L = 0; L < 4; ++L)
#pragma unroll
          for (int qq = 0; qq < C::QSW; ++qq) acc2[L][qq] = make_float2(0.f, 0.f);
        // load n covers lane half h and 32-column chunk cc: in query-major
        // order (n = qq * LPQ + h * CPQ + chunk of the query) when a job may
        // skip one of the warp's queries, else lane-half-major (n = h * NCC + cc)
        constexpr int CPQ = NCC / C::QSW;      // 32-column chunks per query
        constexpr int LPQ = 2 * CPQ;           // loads per query
        static_assert(CPQ * C::QSW == NCC && CPQ * 32 == H, "a query's heads fill whole chunks");
        struct LoadAt {
          int qq, h, cc;
        };
        auto load_at = [](int n) {
          if constexpr (SPLIT)
            return LoadAt{n / LPQ, (n % LPQ) / CPQ, (n / LPQ) * CPQ + n % CPQ};
          else
            return LoadAt{(n % NCC) / CPQ, n / NCC, n % NCC};
        };
        const uint32_t t0 = tmem_base + buf * C::N + slice * C::SCOLS;
        auto addr = [&](int n) {
          const LoadAt l = load_at(n);
          return t0 + (uint32_t(lq * 32 + 16 * l.h) << 16) + uint32_t(l.cc * 32);
        };
        auto consume = [&](const uint32_t (&v)[16], int n) {
          const LoadAt l = load_at(n);
          const int qq = l.qq, h = l.h, cc = l.cc;
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int a2 = 0; a2 < 2; ++a2) {
              const float x0 = __uint_as_float(v[4 * i + 2 * a2]), x1 = __uint_as_float(v[4 * i + 2 * a2 + 1]);
              float2& acc = acc2[2 * h + a2][qq];
#if SA_IDX_QUAD_MATH == 0
              acc = __ffma2_rn(wq[cc][i], make_float2(x0 + fabsf(x0), x1 + fabsf(x1)), acc);
#elif SA_IDX_QUAD_MATH == 1
              acc.x = fmaf(wq[cc][i].x, x0 + fabsf(x0), acc.x);
              acc.y = fmaf(wq[cc][i].y, x1 + fabsf(x1), acc.y);
#else
              acc.x = fmaf(wq[cc][i].x, fmaxf(x0, 0.f), acc.x);   // the weights hold w, not w / 2
              acc.y = fmaf(wq[cc][i].y, fmaxf(x1, 0.f), acc.y);
#endif
            }
        };
        // loads [LO, HI), double-buffered: load n + 1 is in flight while load n
        // is consumed; the accumulator is released once its last load is issued
        auto drain = [&](auto lo_c, auto hi_c) {
          constexpr int LO = decltype(lo_c)::value, HI = decltype(hi_c)::value;
          uint32_t va[16], vb[16];
          tmem_ld16x256b_x4(addr(LO), va);
          tmem_ld_wait();
          tmem_regs_ready(va);
#pragma unroll
          for (int n = LO; n < HI; n += 2) {
            if (n + 1 < HI) tmem_ld16x256b_x4(addr(n + 1), vb);
            if (n + 1 >= HI) release();
            consume(va, n);
            if (n + 1 < HI) {
              tmem_ld_wait();
              tmem_regs_ready(vb);
              if (n + 2 < HI) tmem_ld16x256b_x4(addr(n + 2), va);
              if (n + 2 >= HI) release();
              consume(vb, n + 1);
              if (n + 2 < HI) {
                tmem_ld_wait();
                tmem_regs_ready(va);
              }
            }
          }
        };
        if constexpr (SPLIT) {
          if (need == FULL)
            drain(IntC<0>{}, IntC<NLD>{});
          else if (need == 1u)
            drain(IntC<0>{}, IntC<LPQ>{});
          else if (need == 2u)
            drain(IntC<LPQ>{}, IntC<NLD>{});
          else
            release();
        } else {
          drain(IntC<0>{}, IntC<NLD>{});
        }
        // reduce-scatter over the quad: the lane pair {0,1} or {2,3} by bit 1
        // of c, then one lane by bit 0; thread c keeps lane c (row 8c + r)
#pragma unroll
        for (int qq = 0; qq < C::QSW; ++qq) {
          qsum[qq] = 0.f;
          if (SPLIT && !((need >> qq) & 1u)) continue;   // warp-uniform
          float sl[4];
#pragma unroll
          for (int L = 0; L < 4; ++L) sl[L] = acc2[L][qq].x + acc2[L][qq].y;
          const bool hi2 = (qc & 2) != 0, hi1 = (qc & 1) != 0;
          float k0 = hi2 ? sl[2] : sl[0], k1 = hi2 ? sl[3] : sl[1];
          const float o0 = hi2 ? sl[0] : sl[2], o1 = hi2 ? sl[1] : sl[3];
          k0 += __shfl_xor_sync(0xffffffffu, o0, 2);
          k1 += __shfl_xor_sync(0xffffffffu, o1, 2);
          const float kk = hi1 ? k1 : k0, oo = hi1 ? k0 : k1;
          qsum[qq] = kk + __shfl_xor_sync(0xffffffffu, oo, 1);
        }
      } else {
      // sum_h w'[h] * ReLU(acc[h]) in NP independent partial sums per query
      // (a single running sum would be a dependent FMA chain of H links)
      constexpr int NPMAX = (C::QS > 1) ? SA_IDX_NP_WIDE : 8;
      constexpr int NP = (H / 4 < NPMAX) ? H / 4 : NPMAX;
      constexpr int NCH = C::SCOLS / 32;
      float acc[C::QSW][NP];
#pragma unroll
      for (int qq = 0; qq < C::QSW; ++qq)
#pragma unroll
        for (int p = 0; p < NP; ++p) acc[qq][p] = 0.f;
      const uint32_t t_addr = tmem_base + (uint32_t(lq * 32) << 16) + buf * C::N + slice * C::SCOLS;
      const float* wrow = sW + g * C::N + slice * C::SCOLS;
#if SA_IDX_EPI_PACKED
      // w * ReLU(a) = (w / 2) * (a + |a|): a + |a| is exact (2a or +0) and one
      // FADD; the halved weights sit in sW, pairs accumulate with f32x2 FMAs
      float2 acc2[C::QSW][NP];
#pragma unroll
      for (int qq = 0; qq < C::QSW; ++qq)
#pragma unroll
        for (int p = 0; p < NP; ++p) acc2[qq][p] = make_float2(0.f, 0.f);
      auto consume = [&](const float (&v)[32], int c) {
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 w4 = *reinterpret_cast<const float4*>(wrow + c * 32 + e4 * 4);
          const int col0 = c * 32 + e4 * 4;
          const int qq = col0 / H;
          const int p = ((col0 % H) / 4) % NP;
          const float2 r01 = make_float2(v[e4 * 4 + 0] + fabsf(v[e4 * 4 + 0]), v[e4 * 4 + 1] + fabsf(v[e4 * 4 + 1]));
          const float2 r23 = make_float2(v[e4 * 4 + 2] + fabsf(v[e4 * 4 + 2]), v[e4 * 4 + 3] + fabsf(v[e4 * 4 + 3]));
          float2 a2 = acc2[qq][p];
          a2 = __ffma2_rn(make_float2(w4.x, w4.y), r01, a2);
          a2 = __ffma2_rn(make_float2(w4.z, w4.w), r23, a2);
          acc2[qq][p] = a2;
        }
      };
#else
      auto consume = [&](const float (&v)[32], int c) {
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 w4 = *reinterpret_cast<const float4*>(wrow + c * 32 + e4 * 4);
          const int col0 = c * 32 + e4 * 4;
          const int qq = col0 / H;
          const int p = ((col0 % H) / 4) % NP;
          float a4 = acc[qq][p];
          a4 = fmaf(w4.x, fmaxf(v[e4 * 4 + 0], 0.f), a4);
          a4 = fmaf(w4.y, fmaxf(v[e4 * 4 + 1], 0.f), a4);
          a4 = fmaf(w4.z, fmaxf(v[e4 * 4 + 2], 0.f), a4);
          a4 = fmaf(w4.w, fmaxf(v[e4 * 4 + 3], 0.f), a4);
          acc[qq][p] = a4;
        }
      };
#endif
      // double-buffered TMEM loads: chunk c + 1 is in flight while chunk c is
      // consumed (one wait::ld covers it)
      float va[32], vb[32];
      tmem_ld32(t_addr, va);
      tmem_ld_wait();
      tmem_regs_ready(va);
#pragma unroll
      for (int c = 0; c < NCH; c += 2) {
        if (c + 1 < NCH) tmem_ld32(t_addr + (c + 1) * 32, vb);
        if (c + 1 >= NCH) release();
        consume(va, c);
        if (c + 1 < NCH) {
          tmem_ld_wait();
          tmem_regs_ready(vb);
          if (c + 2 < NCH) tmem_ld32(t_addr + (c + 2) * 32, va);
          if (c + 2 >= NCH) release();
          consume(vb, c + 1);
          if (c + 2 < NCH) {
            tmem_ld_wait();
            tmem_regs_ready(va);
          }
        }
      }
#pragma unroll
      for (int qq = 0; qq < C::QSW; ++qq) {
        float sum = 0.f;
#if SA_IDX_EPI_PACKED
#pragma unroll
        for (int p = 0; p < NP; ++p) sum += acc2[qq][p].x + acc2[qq][p].y;
#else
#pragma unroll
        for (int p = 0; p < NP; ++p) sum += acc[qq][p];
#endif
        qsum[qq] = sum;
      }
      }
      wg = g;
      // outputs
#pragma unroll
      for (int qq = 0; qq < C::QSW; ++qq) {
        const int t = HOIST_T ? tq[HOIST_T ? qq : 0] : query_row(g, ql, qq);
        if (t < 0) continue;                   // absent query, or a row past the last
        int gcol = 0;                          // grouped: the query's candidate column of this key
        if constexpr (MODE == IDX_GROUPED) {
          if (cur.s < 0) continue;             // no union block in this half
          const int ql = g * C::QS + slice * C::QSW + qq;
          const int slot = SPLIT ? (int)((slots2 >> (8 * qq)) & 0xFFu) : (int)((sUSlot[col] >> (8 * ql)) & 0xFFu);
          if (slot == 0xFF) continue;          // the query did not keep this block
          gcol = slot * 64 + (row & 63);
        }
        bool vis;
        if constexpr (MODE == IDX_DECODE)
          vis = kvalid;
        else
          vis = kvalid && s <= (HOIST ? limq[HOIST ? qq : 0] : vis_limit(t, a));
        const float score = vis ? qsum[qq] * sk : -__int_as_float(0x7f800000);
        if constexpr (MODE == IDX_PREFILL) {
          if (a.cand != nullptr) {
            // candidate mode: warp-aggregated append of keys at or above theta
            const bool take = vis && score >= sTheta[t - q0];
            const unsigned bal = __ballot_sync(0xffffffffu, take);
            if (bal != 0u) {
              int base = 0;
              if (lane == 0) base = atomicAdd(&a.cand_cnt[t], __popc(bal));
              base = __shfl_sync(0xffffffffu, base, 0);
              const int pos = base + __popc(bal & ((1u << lane) - 1u));
              if (take && pos < a.cap) {
                uint32_t b = __float_as_uint(score);
                if (b == 0x80000000u) b = 0u;
                const uint32_t key = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
                a.cand[(long long)t * a.cap + pos] = ((unsigned long long)key << 32) | (uint32_t)(~(uint32_t)s);
              }
            }
            continue;
          }
        }
        if constexpr (MODE == IDX_GATHER) {
          a.out[(long long)t * a.ld + col] = score;
        } else if constexpr (MODE == IDX_GROUPED) {
          a.out[(long long)t * a.ld + gcol] = score;
        } else {
          if (col < a.n_k) a.out[(long long)t * a.ld + col] = score;
        }
      }
      }
      J0 += njobs;
      if constexpr (PERSIST) {                 // this warp is done with the unit's metadata
        __syncwarp();
        if (lane == 0) mbar_arrive(&mempty[bm]);
      }
    }
  } else {
    // ======================= metadata stager =======================
    // persistent modes: stages each unit's weights and lists into the
    // metadata buffer its epilogue reads, up to two units ahead
    if constexpr (PERSIST) {
      int bi = 0;
      for (int it = 0;; ++it) {
        const int unit = unit_at(it);
        if (unit < 0) break;
        const UnitP u = unit_params(unit);
        if (u.njobs == 0) continue;
        const int b = bi % C::QB, use = bi / C::QB;
        ++bi;
        if (use > 0 && !mbar_wait(&mempty[b], (use - 1) & 1, wc, 8)) break;
        stage_warp(u, meta(b));
        mbar_arrive(&mfull[b]);                // each lane after its own stores
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<512>(tmem_base);
  }
}

// ----------------------------------------------------------------- host side
template <int H, int D, bool FP8, int MODE>
static cudaError_t launch_t(const void* q, const void* k, int q_rows, long long k_rows, const IdxArgs& a,
                            cudaStream_t st) {
  using C = IdxCfg<H, D, FP8, MODE>;
  CUtensorMap qm, km;
  const CUtensorMapDataType dt = FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle sw = (C::ROWB == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const uint32_t qbox = (MODE == IDX_PREFILL && a.q_rows == nullptr) ? C::QS * H : H;
  const uint32_t kbox = (MODE == IDX_GATHER || MODE == IDX_GROUPED) ? 64 : 128;
  if (!make_tmap_2d(&qm, q, dt, D, (uint64_t)q_rows * H, C::ROWB, D, qbox, sw)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&km, k, dt, D, (uint64_t)k_rows, C::ROWB, D, kbox, sw)) return cudaErrorInvalidValue;
  auto kern = indexer_kernel<H, D, FP8, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid;
  if constexpr (C::PERSIST) {
    // one persistent CTA per SM (at most one per unit)
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int units = (MODE == IDX_PREFILL) ? (a.n_q + C::NQ - 1) / C::NQ : a.n_groups;
    grid = dim3(units < sms ? units : sms);
  } else if constexpr (MODE == IDX_DECODE) {
    grid = dim3(((a.span + 127) / 128 + a.tiles_per_cta - 1) / a.tiles_per_cta, a.n_q);
  } else {
    grid = dim3((a.n_q + C::NQ - 1) / C::NQ);
  }
  if (grid.x == 0 || grid.y == 0) return cudaSuccess;
  kern<<<grid, C::THREADS, C::SMEM, st>>>(qm, km, a);
  return cudaGetLastError();
}

cudaError_t launch_indexer(int mode, int heads, int d, sa_dtype dt, const void* q, const void* k, int q_rows,
                           long long k_rows, const IdxArgs& a, cudaStream_t st) {
#define SA_IDX_CASE(H_, D_, F_)                                                                   \
  if (heads == H_ && d == D_ && (dt == SA_FP8_E4M3) == F_) {                                       \
    if (mode == IDX_PREFILL) return launch_t<H_, D_, F_, IDX_PREFILL>(q, k, q_rows, k_rows, a, st); \
    if (mode == IDX_DECODE) return launch_t<H_, D_, F_, IDX_DECODE>(q, k, q_rows, k_rows, a, st);   \
    if (mode == IDX_GATHER) return launch_t<H_, D_, F_, IDX_GATHER>(q, k, q_rows, k_rows, a, st);   \
    if (mode == IDX_GROUPED) return launch_t<H_, D_, F_, IDX_GROUPED>(q, k, q_rows, k_rows, a, st); \
  }
#define SA_IDX_CASE_PREFILL(H_, D_, F_)                                                            \
  if (heads == H_ && d == D_ && (dt == SA_FP8_E4M3) == F_ && mode == IDX_PREFILL)                  \
    return launch_t<H_, D_, F_, IDX_PREFILL>(q, k, q_rows, k_rows, a, st);
  SA_IDX_CASE(64, 128, true)
  SA_IDX_CASE(32, 128, true)
  SA_IDX_CASE_PREFILL(4, 32, false)
  SA_IDX_CASE_PREFILL(8, 32, false)
#undef SA_IDX_CASE_PREFILL
#undef SA_IDX_CASE
  return cudaErrorNotSupported;
}

}  // namespace sa
