// lsa.cu -- the LSA flat semantic search: bucket cache and per-query index
// rows ("Latent Sparse Attention", paperpeel 2610.42147, section 3.1
// "Semantic Clustering", section 3.2 "Semantic Search", appendix F.1
// "Kernels").
//
// Clustering (one CTA per cluster block): the block's index keys are L2
// normalised and summed n_pool at a time into pool keys, which stay in shared
// memory for every round of Ward's method: each bucket finds its cheapest
// partner among those it may merge with (the merged bucket holds at most
// n_b^max keys), every mutually cheapest pair merges, and rounds repeat until
// m buckets remain (a round that would overshoot merges its cheapest pairs).
// The host neither launches nor reads anything between rounds. The kernel
// writes each bucket's bf16 unit centroid and the ascending positions of its
// keys. Costs decide integer outcomes, so they are computed with explicitly
// rounded fp32 operations (no fused multiply-add) summing the dimensions from
// 0 upward: n_a n_b / (n_a + n_b) * |mu_a - mu_b|^2 with mu = sum / n, counts in
// pool keys. Ties go to the lower index.
//
// Search: queries are normalised to bf16; a tcgen05 kernel scores 128 buckets
// (MMA M dimension) against 128 queries (N), both operands bf16, K = d_idx =
// 64, fp32 accumulation in tensor memory. Two regimes (appendix F.1 "Flat
// prefill"): below 32,768 buckets the kernel writes each query's row of
// scores S and the library's radix top-k keeps the p best of the query's
// visible buckets (the cluster blocks before its own); beyond, S is never
// written -- a threshold per query from sampled centroids, the same kernel
// appending the buckets at or above it to the query's list in its epilogue,
// a radix select over the list, and a whole-row rescoring for the rows whose
// list missed ("Selection by threshold"). Either way one CTA per query sorts
// its p buckets by packed key (score, then lower id), takes their keys best
// first into k long-range keys, skipping keys of the sinks and the window, and
// writes the index row [sinks | window | long-range keys | -1 ...].
//
// Decode ("Flat decode"): each sequence's new query scores the centroids of
// its own bucket cache on the CUDA cores (one flop per byte: bound by HBM),
// then the same top-p and expansion; fixed shapes, no host synchronisation.
#include <cuda_bf16.h>

#include "debug.cuh"
#include "ptx.cuh"
#include "radix.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int LSA_D = 64;              // d_idx of the index space
constexpr int LSA_PMAX = 256;          // pool keys per cluster block
constexpr int LSA_CT = 256;            // clustering threads
constexpr int LSA_MU_LD = LSA_D + 1;   // padded row of the means (conflict-free per-row reads)
constexpr int LSA_TILE = 128;          // buckets x queries per score tile
constexpr int LSA_ST = 128;            // score kernel threads
constexpr int LSA_SCORE_SMEM = 48 * 1024;   // 33 KB used; 48 KB caps residency at 4 CTAs (4 x 128 TMEM columns)
constexpr int LSA_PSORT_MAX = 2048;    // largest p
constexpr int LSA_MAX_BUCKETS = 32768; // short-context regime of the search
constexpr long long LSA_WAIT_BUDGET = 4000000000ll;

// ------------------------------------------------------------ fp32 steps
// One correctly rounded fp32 operation each; never contracted into an FMA.
__device__ __forceinline__ void load_bf16_row(const __nv_bfloat16* src, float (&x)[LSA_D]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int c = 0; c < LSA_D / 8; ++c) {
    const uint4 u = __ldg(s4 + c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[8 * c + 2 * e] = __uint_as_float(w[e] << 16);
      x[8 * c + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
}

// x / |x| in place (|x|^2 summed from dimension 0; an all-zero row stays 0).
__device__ __forceinline__ void normalize_in_place(float (&x)[LSA_D]) {
  float ss = __fmul_rn(x[0], x[0]);
#pragma unroll
  for (int j = 1; j < LSA_D; ++j) ss = __fadd_rn(ss, __fmul_rn(x[j], x[j]));
  const float nrm = __fsqrt_rn(ss);
#pragma unroll
  for (int j = 0; j < LSA_D; ++j) x[j] = nrm > 0.f ? __fdiv_rn(x[j], nrm) : 0.f;
}

// ---------------------------------------------------------- clustering
struct ClusterArgs {
  const __nv_bfloat16* k;     // [n_k, 64]
  int block0;
  int n_pool, n_cluster, P, m, cap;   // cap in pool keys
  __nv_bfloat16* cent;        // [n_blocks_total * m, 64]
  int32_t* bucket_off;        // [n_blocks_total * m]
  int32_t* bucket_keys;       // [n_blocks_total * n_cluster]
  uint32_t* status;           // sa_device_status words, nullable
};

struct ClusterSmem {
  int cnt[LSA_PMAX];
  int alive[LSA_PMAX];
  int parent[LSA_PMAX];
  int best[LSA_PMAX];
  float bcost[LSA_PMAX];
  int hbest[2][LSA_PMAX];      // per half of the partner search (H <= 2 halves stored)
  float hcost[2][LSA_PMAX];
  int pa[LSA_PMAX / 2];        // mutual pairs of the round: lower index, its cost
  float pc[LSA_PMAX / 2];
  int psel[LSA_PMAX / 2];
  int root[LSA_PMAX];
  int number[LSA_PMAX];
  int koff[LSA_PMAX];          // key offset of a surviving bucket within the block's lists
  int n_pairs;
  int n_alive;
  int failed;
};

__global__ void __launch_bounds__(LSA_CT) lsa_cluster_kernel(ClusterArgs a) {
  extern __shared__ __align__(16) float lsa_dyn[];
  __shared__ ClusterSmem sh;
  const int P = a.P, tid = threadIdx.x;
  const int c = a.block0 + blockIdx.x;
  float* S = lsa_dyn;                              // [P][64] bucket sums
  float* Mu = lsa_dyn + P * LSA_D;                 // [P][65] bucket means

  // ---- unit keys pooled n_pool at a time (section 3.1 "Pooling") ----
  for (int g = tid; g < P; g += LSA_CT) {
    float acc[LSA_D];
    for (int r = 0; r < a.n_pool; ++r) {
      float x[LSA_D];
      load_bf16_row(a.k + ((long long)c * a.n_cluster + (long long)g * a.n_pool + r) * LSA_D, x);
      normalize_in_place(x);
      if (r == 0) {
#pragma unroll
        for (int j = 0; j < LSA_D; ++j) acc[j] = x[j];
      } else {
#pragma unroll
        for (int j = 0; j < LSA_D; ++j) acc[j] = __fadd_rn(acc[j], x[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < LSA_D; ++j) S[g * LSA_D + j] = acc[j];
    sh.cnt[g] = 1;
    sh.alive[g] = 1;
    sh.parent[g] = g;
  }
  if (tid == 0) {
    sh.n_alive = P;
    sh.failed = 0;
  }
  __syncthreads();

  // ---- Ward rounds (section 3.1 "Clustering") ----
  const int H = P <= LSA_CT / 2 ? 2 : 1;          // threads per bucket in the partner search
  for (int round = 0; round < P && sh.n_alive > a.m; ++round) {
    for (int e = tid; e < P * LSA_D; e += LSA_CT) {
      const int b = e / LSA_D, j = e - b * LSA_D;
      if (sh.alive[b]) Mu[b * LSA_MU_LD + j] = __fdiv_rn(S[b * LSA_D + j], (float)sh.cnt[b]);
    }
    if (tid == 0) sh.n_pairs = 0;
    __syncthreads();
    // cheapest fitting partner of bucket x over the candidates y = h, h + H, ...
    if (tid < P * H) {
      const int x = tid % P, h = tid / P;
      int bx = -1;
      float cx = 0.f;
      if (sh.alive[x]) {
        float mx[LSA_D];
#pragma unroll
        for (int j = 0; j < LSA_D; ++j) mx[j] = Mu[x * LSA_MU_LD + j];
        const int nx = sh.cnt[x];
        for (int y = h; y < P; y += H) {
          if (y == x || !sh.alive[y]) continue;
          const int ny = sh.cnt[y];
          if (nx + ny > a.cap) continue;
          const float* my = Mu + y * LSA_MU_LD;
          float dist = 0.f;
#pragma unroll
          for (int j = 0; j < LSA_D; ++j) {
            const float df = __fsub_rn(mx[j], my[j]);
            dist = __fadd_rn(dist, __fmul_rn(df, df));
          }
          const float w = __fdiv_rn((float)(nx * ny), (float)(nx + ny));
          const float cost = __fmul_rn(w, dist);
          if (bx < 0 || cost < cx) {
            bx = y;
            cx = cost;
          }
        }
      }
      sh.hbest[h][x] = bx;
      sh.hcost[h][x] = cx;
    }
    __syncthreads();
    for (int x = tid; x < P; x += LSA_CT) {
      int bx = sh.hbest[0][x];
      float cx = sh.hcost[0][x];
      if (H == 2) {
        const int b1 = sh.hbest[1][x];
        const float c1 = sh.hcost[1][x];
        if (b1 >= 0 && (bx < 0 || c1 < cx || (c1 == cx && b1 < bx))) {
          bx = b1;
          cx = c1;
        }
      }
      sh.best[x] = sh.alive[x] ? bx : -1;
      sh.bcost[x] = cx;
    }
    __syncthreads();
    for (int x = tid; x < P; x += LSA_CT) {
      const int y = sh.best[x];
      if (y > x && sh.best[y] == x) {
        const int i = atomicAdd(&sh.n_pairs, 1);
        sh.pa[i] = x;
        sh.pc[i] = sh.bcost[x];
      }
    }
    __syncthreads();
    const int M = sh.n_pairs, need = sh.n_alive - a.m;
    if (M == 0) {                                  // no pair fits (possible only when n_b^max < 2 n_cluster / m)
      if (tid == 0 && a.status != nullptr) atomicCAS(a.status, 0u, (uint32_t)SA_ERR_INTERNAL);
      sh.failed = 1;
      break;
    }
    // merge the `need` cheapest pairs when there are more (cost, then lower index)
    for (int i = tid; i < M; i += LSA_CT) {
      int rank = 0;
      for (int j = 0; j < M; ++j)
        rank += (sh.pc[j] < sh.pc[i] || (sh.pc[j] == sh.pc[i] && sh.pa[j] < sh.pa[i])) ? 1 : 0;
      sh.psel[i] = rank < need ? 1 : 0;
    }
    __syncthreads();
    for (int e = tid; e < M * LSA_D; e += LSA_CT) {
      const int i = e / LSA_D, j = e - i * LSA_D;
      if (sh.psel[i]) {
        const int x = sh.pa[i], y = sh.best[x];
        S[x * LSA_D + j] = __fadd_rn(S[x * LSA_D + j], S[y * LSA_D + j]);
      }
    }
    __syncthreads();
    for (int i = tid; i < M; i += LSA_CT) {
      if (sh.psel[i]) {
        const int x = sh.pa[i], y = sh.best[x];
        sh.cnt[x] += sh.cnt[y];
        sh.alive[y] = 0;
        sh.parent[y] = x;
      }
    }
    __syncthreads();
    if (tid == 0) sh.n_alive -= min(M, need);
    __syncthreads();
  }
  if (sh.failed || sh.n_alive != a.m) {
    if (tid == 0 && !sh.failed && a.status != nullptr) atomicCAS(a.status, 0u, (uint32_t)SA_ERR_INTERNAL);
    return;
  }

  // ---- bucket cache (section 3.1 "Bucket cache") ----
  for (int g = tid; g < P; g += LSA_CT) {
    int r = g;
    for (int s = 0; s < P && sh.parent[r] != r; ++s) r = sh.parent[r];
    sh.root[g] = r;
    if (sh.alive[g]) {
      int num = 0, off = 0;
      for (int x = 0; x < g; ++x)
        if (sh.alive[x]) {
          ++num;
          off += sh.cnt[x];
        }
      sh.number[g] = num;
      sh.koff[g] = off * a.n_pool;
    }
  }
  __syncthreads();
  const long long kbase = (long long)c * a.n_cluster;
  for (int g = tid; g < P; g += LSA_CT) {
    const int r = sh.root[g];
    int before = 0;
    for (int x = 0; x < g; ++x) before += sh.root[x] == r ? 1 : 0;
    SA_DBG_CHECK(sh.koff[r] + (before + 1) * a.n_pool <= a.n_cluster, SA_DBG_LSA_CLUSTER, g);
    int32_t* dst = a.bucket_keys + kbase + sh.koff[r] + before * a.n_pool;
    for (int e = 0; e < a.n_pool; ++e) dst[e] = (int32_t)(kbase + (long long)g * a.n_pool + e);
    if (sh.alive[g]) {
      const long long b = (long long)c * a.m + sh.number[g];
      a.bucket_off[b] = (int32_t)(kbase + sh.koff[g]);
      float v[LSA_D];
#pragma unroll
      for (int j = 0; j < LSA_D; ++j) v[j] = S[g * LSA_D + j];
      normalize_in_place(v);
      uint32_t* out = reinterpret_cast<uint32_t*>(a.cent + b * LSA_D);
#pragma unroll
      for (int j = 0; j < LSA_D; j += 2) {
        const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
        const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(v[j + 1]));
        out[j / 2] = lo | (hi << 16);
      }
    }
  }
}

// ------------------------------------------------ query normalisation
__global__ void __launch_bounds__(256) lsa_qnorm_kernel(const __nv_bfloat16* __restrict__ q, int n,
                                                        __nv_bfloat16* __restrict__ out) {
  const int i = blockIdx.x * 256 + threadIdx.x;
  if (i >= n) return;
  float x[LSA_D];
  load_bf16_row(q + (long long)i * LSA_D, x);
  normalize_in_place(x);
  uint4* o4 = reinterpret_cast<uint4*>(out + (long long)i * LSA_D);
#pragma unroll
  for (int c8 = 0; c8 < LSA_D / 8; ++c8) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(x[8 * c8 + 2 * e]));
      const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(x[8 * c8 + 2 * e + 1]));
      w[e] = lo | (hi << 16);
    }
    o4[c8] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ------------------------------------------------------- bucket scores
// Buckets visible to the query at position pos: those of the cluster blocks
// before its own (section 3.2 "Scoring").
__device__ __forceinline__ int visible_buckets(int pos, int n_cluster, int m, int n_blocks) {
  return min(n_blocks, pos / n_cluster) * m;
}

struct ScoreArgs {
  const __nv_bfloat16* cent;   // [n_buckets, 64]
  const __nv_bfloat16* qn;     // [rows, 64] unit queries of the chunk
  int n_buckets;               // rows of cent
  int rows, pos0;              // chunk rows; position of row 0
  const int* row_pos;          // position of every row (ascending), overriding pos0 + row when non-null
  int col_stride;              // column b holds bucket b * col_stride (the sampled buckets of the estimate)
  int n_cluster, m, n_blocks;
  float* S;                    // table mode: [rows, ld]
  long long ld;
  // candidate mode: every visible bucket b with score >= theta[row] is appended
  // to the row's list as (score key << 32 | ~b); cnt[row] counts past cap
  const float* theta;
  unsigned long long* cand;    // [rows, cap]
  int* cnt;                    // [rows]
  int cap;
  uint32_t* status;
  long long budget;
};

__device__ __forceinline__ int row_position(const ScoreArgs& a, int i) {
  return a.row_pos != nullptr ? a.row_pos[i] : a.pos0 + i;
}

// 128 rows x 64 bf16 (128 B each) into the 128-byte-swizzled K-major layout
// of the MMA: row r's 16-byte chunk c at r * 128 + ((c ^ (r & 7)) << 4).
// Rows at or beyond n_rows are zero.
__device__ __forceinline__ void stage_rows_sw128(uint8_t* dst, const __nv_bfloat16* src, int row0, int n_rows) {
  for (int e = threadIdx.x; e < LSA_TILE * 8; e += LSA_ST) {
    const int r = e >> 3, c = e & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row0 + r < n_rows) v = __ldg(reinterpret_cast<const uint4*>(src + (long long)(row0 + r) * LSA_D) + c);
    *reinterpret_cast<uint4*>(dst + r * 128 + ((c ^ (r & 7)) << 4)) = v;
  }
}

template <bool CAND>
__global__ void __launch_bounds__(LSA_ST) lsa_score_kernel(ScoreArgs a) {
  extern __shared__ uint8_t lsa_score_raw[];
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;
  const int b0 = blockIdx.x * LSA_TILE, i0 = blockIdx.y * LSA_TILE;
  const int i_last = min(a.rows, i0 + LSA_TILE) - 1;
  if ((long long)b0 * a.col_stride >= visible_buckets(row_position(a, i_last), a.n_cluster, a.m, a.n_blocks))
    return;                                 // no query of the tile sees a bucket of it
  uint8_t* sm = smem_align1024(lsa_score_raw);
  uint8_t* sA = sm;                         // 128 buckets x 64 (16 KB)
  uint8_t* sB = sm + LSA_TILE * 128;        // 128 queries x 64 (16 KB)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  stage_rows_sw128(sA, a.cent, b0, a.n_buckets);
  stage_rows_sw128(sB, a.qn, i0, a.rows);
  fence_proxy_async_smem();                 // generic-proxy stores -> visible to the tensor core
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc<LSA_TILE>(&tmem_slot);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (threadIdx.x == 0) {
    constexpr uint32_t idesc = umma_idesc<1, 128, LSA_TILE>();
    const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
#pragma unroll
    for (int kk = 0; kk < LSA_D / 16; ++kk)
      mma_bf16(tmem, umma_smem_desc<128>(a_base + kk * 32), umma_smem_desc<128>(b_base + kk * 32), idesc,
               kk > 0 ? 1u : 0u);
    mma_commit(&bar);
  }
  const WaitCtx wc{&abort_flag, a.status, a.budget};
  const bool ok = mbar_wait(&bar, 0, wc, 60);
  tc_fence_after();
  if (ok) {
    // warp w reads TMEM lanes 32w.. (buckets b0 + 32w + lane), 32 query columns at a time
    const int b = b0 + warp * 32 + lane;
    const uint32_t t_row = tmem + (uint32_t(warp * 32) << 16);
    for (int c0 = 0; c0 < LSA_TILE; c0 += 32) {
      float v[32];
      tmem_ld32(t_row + c0, v);
      tmem_ld_wait();
      tmem_regs_ready(v);
      if constexpr (!CAND) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int i = i0 + c0 + j;
          if (i < a.rows) a.S[(long long)i * a.ld + b] = v[j];
        }
      } else {
        // threshold scan: one ballot per (warp, query), one atomic when a lane hits
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int i = i0 + c0 + j;
          if (i < a.rows) {
            const int vis = visible_buckets(row_position(a, i), a.n_cluster, a.m, a.n_blocks);
            const bool hit = b < vis && v[j] >= a.theta[i];
            const unsigned bal = __ballot_sync(0xffffffffu, hit);
            if (bal != 0u) {
              int base = 0;
              if (lane == 0) base = atomicAdd(a.cnt + i, __popc(bal));
              base = __shfl_sync(0xffffffffu, base, 0);
              const int slot = base + __popc(bal & ((1u << lane) - 1u));
              if (hit && slot < a.cap)
                a.cand[(long long)i * a.cap + slot] =
                    ((unsigned long long)score_key(v[j]) << 32) | (uint32_t)~(uint32_t)b;
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc<LSA_TILE>(tmem);
}

__global__ void lsa_rowlen_kernel(int rows, int pos0, const int* row_pos, int n_cluster, int m, int n_blocks,
                                  int* len) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < rows) len[i] = visible_buckets(row_pos != nullptr ? row_pos[i] : pos0 + i, n_cluster, m, n_blocks);
}

// ------------------------------------------------ threshold regime pieces
// Appendix F.1 "Selection by threshold": theta_i is set before the scan from
// a sample of the row; the scan lists every bucket at or above it; only the
// list is ranked; a row whose list holds fewer than p buckets, or more than
// its room, falls back to its whole row. Here the sample is every stride-th
// bucket (about 8192 of them); the query sees the n_vs samples below its
// visible bucket count vis and takes the round(gamma p n_vs / vis)-th largest
// sampled score, so that its list holds about gamma p buckets. Rows whose
// visible buckets all fit in the list take theta = -inf.
constexpr float LSA_GAMMA = 1.5f;   // list target gamma p, room 3p (twice the target, as the pages size it)
constexpr int LSA_SAMPLES = 8192;

__device__ __forceinline__ float lsa_key_to_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

__global__ void __launch_bounds__(TK_THREADS, 1)
    lsa_theta_kernel(const float* __restrict__ stab, long long ld, int pos0, int n_cluster, int m, int n_blocks,
                     int stride, int p, int cap, int hook, float* __restrict__ theta) {
  extern __shared__ uint8_t lsa_th_raw[];
  TkShared& sh = *reinterpret_cast<TkShared*>(lsa_th_raw);
  const int t = blockIdx.x, tid = threadIdx.x;
  const int vis = visible_buckets(pos0 + t, n_cluster, m, n_blocks);
  float th;
  if (hook == SA_HOOK_THETA_POS_INF) {
    th = INFINITY;
  } else if (hook == SA_HOOK_THETA_NEG_INF || vis <= cap) {
    th = -INFINITY;
  } else {
    const int n_vs = (vis + stride - 1) / stride;
    const long long want = llrintf(LSA_GAMMA * (float)p * (float)n_vs / (float)vis);
    int need = (int)max(1ll, min((long long)n_vs, want));
    const float* row = stab + (long long)t * ld;
    uint32_t prefix = 0;
    int pbits = 0;
    while (pbits < 32) {                    // 12 + 12 + 8 bits: the exact need-th largest sample
      const int db = (pbits == 24) ? 8 : TK_HBITS;
      const int nbins = 1 << db;
      for (int b = tid; b < nbins; b += TK_THREADS) sh.hist[b] = 0;
      __syncthreads();
      const int sdig = 32 - pbits - db;
      for (int j = tid; j < n_vs; j += TK_THREADS) {
        const uint32_t key = score_key(row[j]);
        if (pbits == 0 || (key >> (32 - pbits)) == prefix) atomicAdd(&sh.hist[(key >> sdig) & (nbins - 1)], 1u);
      }
      __syncthreads();
      find_bucket(sh, nbins, need);
      need -= sh.above;
      prefix = (prefix << db) | (uint32_t)sh.bucket;
      pbits += db;
      __syncthreads();
    }
    th = lsa_key_to_float(prefix);
  }
  if (tid == 0) theta[t] = th;
}

// The top-p of each row's list, written as packed keys (0 past the row's
// min(p, vis) entries); rows whose list missed are flagged for the fallback.
__global__ void __launch_bounds__(TK_THREADS, 1)
    lsa_select_kernel(const unsigned long long* __restrict__ cand, const int* __restrict__ cnt, int cap, int pos0,
                      int n_cluster, int m, int n_blocks, int p, unsigned long long* __restrict__ sig,
                      int* __restrict__ miss, uint32_t* status) {
  extern __shared__ uint8_t lsa_sel_raw[];
  TkShared& sh = *reinterpret_cast<TkShared*>(lsa_sel_raw);
  const int t = blockIdx.x, tid = threadIdx.x;
  const int vis = visible_buckets(pos0 + t, n_cluster, m, n_blocks);
  const int need = min(p, vis);
  const int c = cnt[t];
  const bool ok = c <= cap && c >= need;
  if (tid == 0) {
    miss[t] = ok ? 0 : 1;
    if (status != nullptr) {
      if (!ok) atomicAdd(status + 2, 1u);
      if (c > cap) atomicAdd(status + 3, 1u);
    }
    sh.n_out = 0;
  }
  if (!ok) return;
  const unsigned long long* row = cand + (long long)t * cap;
  for (int j = tid; j < c; j += TK_THREADS) sh.cand[j] = row[j];
  __syncthreads();
  unsigned long long* out = sig + (long long)t * p;
  smem_select64(sh, c, need, [&](uint64_t key) { out[atomicAdd(&sh.n_out, 1)] = key; });
  for (int j = need + tid; j < p; j += TK_THREADS) out[j] = 0ull;
}

// Packed keys of the fallback rows from their rescored rows: fallback row f
// (of n_f) is chunk row rows[f]; its top-p bucket ids sel[f] index S row f.
__global__ void __launch_bounds__(256)
    lsa_sig_from_table_kernel(const float* __restrict__ S, long long ld, const int32_t* __restrict__ sel, int p,
                              const int* __restrict__ rows, int n_f, unsigned long long* __restrict__ sig) {
  const int f = blockIdx.x;
  if (f >= n_f) return;
  unsigned long long* out = sig + (long long)rows[f] * p;
  for (int j = threadIdx.x; j < p; j += 256) {
    const int b = sel[(long long)f * p + j];
    out[j] = b >= 0 ? ((unsigned long long)score_key(S[(long long)f * ld + b]) << 32) | (uint32_t)~(uint32_t)b
                    : 0ull;
  }
}

// ------------------------------------------------------- decode scores
// One new query per sequence scores the centroids of its own cache on the
// CUDA cores: a thread per bucket reads its 128-byte centroid once (the scan
// is bound by HBM at one flop per byte, appendix F.1 "Flat decode").
struct DecodeScoreArgs {
  const __nv_bfloat16* cent;   // [batch, max_blocks * m, 64]
  const __nv_bfloat16* qn;     // [batch, 64] unit queries
  const int* n_blocks;         // [batch] cluster blocks in each cache
  const int* seq_lens;         // [batch] the query sits at seq_lens[b] - 1
  int n_cluster, m, max_blocks;
  float* S;                    // [batch, ld]
  long long ld;
  int* len;                    // [batch] visible buckets
};

__global__ void __launch_bounds__(256) lsa_decode_score_kernel(DecodeScoreArgs a) {
  const int sq = blockIdx.y;
  const int pos = a.seq_lens[sq] - 1;
  const int nb = max(0, min(min(a.n_blocks[sq], a.max_blocks), pos >= 0 ? pos / a.n_cluster : 0));
  const int vis = nb * a.m;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.len[sq] = vis;
  const int b = blockIdx.x * 256 + threadIdx.x;
  if (b >= vis) return;
  float q[LSA_D], x[LSA_D];
  load_bf16_row(a.qn + (long long)sq * LSA_D, q);
  load_bf16_row(a.cent + ((long long)sq * a.max_blocks * a.m + b) * LSA_D, x);
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < LSA_D; ++j) acc = fmaf(q[j], x[j], acc);
  a.S[(long long)sq * a.ld + b] = acc;
}

// ------------------------------------------------------------ expansion
struct ExpandArgs {
  const unsigned long long* sig_in;   // [rows, p] packed keys of the top-p (0 = none), or null: from S and sel
  const float* S;              // [rows, ld]
  long long ld;
  const int32_t* sel;          // [rows, p] top-p bucket ids (any order, -1 padded)
  int p, psort;                // psort: power of two >= p
  const int32_t* bucket_off;
  const int32_t* bucket_keys;
  long long off_stride, keys_stride;   // per row (decode: every sequence has its own cache), else 0
  int n_cluster, m;
  int rows, pos0;
  const int* seq_lens;         // decode: row i sits at seq_lens[i] - 1 (else at pos0 + i)
  int k, n_sink, n_window;
  int32_t* J;                  // [rows, n_sink + n_window + k]
};

__global__ void __launch_bounds__(TK_THREADS) lsa_expand_kernel(ExpandArgs a) {
  __shared__ unsigned long long sig[LSA_PSORT_MAX];
  __shared__ int red[TK_THREADS / 32];
  const int i = blockIdx.x, tid = threadIdx.x;
  const int pos = a.seq_lens != nullptr ? a.seq_lens[i] - 1 : a.pos0 + i;
  const float* srow = a.S + (long long)i * a.ld;
  const int32_t* srl = a.sel + (long long)i * a.p;
  const int32_t* boff = a.bucket_off + (long long)i * a.off_stride;
  const int32_t* bkeys = a.bucket_keys + (long long)i * a.keys_stride;
  for (int j = tid; j < a.psort; j += TK_THREADS) {
    if (a.sig_in != nullptr) {
      sig[j] = j < a.p ? a.sig_in[(long long)i * a.p + j] : 0ull;
    } else {
      const int b = j < a.p ? srl[j] : -1;
      sig[j] = b >= 0 ? ((unsigned long long)score_key(srow[b]) << 32) | (uint32_t)~(uint32_t)b : 0ull;
    }
  }
  __syncthreads();
  // bitonic sort, descending: best bucket first (higher score, then lower id)
  for (int k2 = 2; k2 <= a.psort; k2 <<= 1) {
    for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1) {
      for (int t = tid; t < a.psort; t += TK_THREADS) {
        const int u = t ^ j2;
        if (u > t) {
          const unsigned long long x = sig[t], y = sig[u];
          const bool desc = (t & k2) == 0;
          if (desc ? x < y : x > y) {
            sig[t] = y;
            sig[u] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  const long long width = (long long)a.n_sink + a.n_window + a.k;
  int32_t* out = a.J + (long long)i * width;
  const int n_s = max(0, min(a.n_sink, pos + 1));             // sinks 0 .. n_s - 1
  const int w_lo = max(a.n_sink, pos - a.n_window + 1);        // window w_lo .. pos
  const int n_w = max(0, pos - w_lo + 1);
  for (int t = tid; t < n_s; t += TK_THREADS) out[t] = t;
  for (int t = tid; t < n_w; t += TK_THREADS) out[n_s + t] = w_lo + t;
  int32_t* far = out + n_s + n_w;
  int run = 0;                                                 // long-range keys taken so far
  for (int base = 0; base < a.psort && run < a.k; base += TK_THREADS) {
    const int j = base + tid;
    int lo = 0, hi = 0, u = 0;
    if (j < a.psort && sig[j] != 0ull) {
      const int b = (int)~(uint32_t)(sig[j] & 0xFFFFFFFFull);
      const int c = b / a.m;
      SA_DBG_CHECK(b >= 0 && c < max(0, pos) / a.n_cluster, SA_DBG_LSA_BUCKET, b);
      lo = boff[b];
      hi = (b - c * a.m == a.m - 1) ? (c + 1) * a.n_cluster : boff[b + 1];
      for (int e = lo; e < hi; ++e) {
        const int s = bkeys[e];
        u += (s < a.n_sink || s >= w_lo) ? 0 : 1;
      }
    }
    int tot;
    const int at = run + block_excl_scan(u, red, &tot);
    for (int e = lo, w = at; e < hi && w < a.k; ++e) {
      const int s = bkeys[e];
      if (s < a.n_sink || s >= w_lo) continue;
      SA_DBG_CHECK(s >= 0 && s <= pos, SA_DBG_LSA_KEY, s);
      far[w++] = s;
    }
    run += tot;
  }
  for (long long t = (long long)n_s + n_w + min(run, a.k) + tid; t < width; t += TK_THREADS) out[t] = -1;
}

// --------------------------------------------------------- validation
static bool params_ok(const sa_lsa_params* prm) {
  if (prm == nullptr) return false;
  const int np = prm->n_pool, nc = prm->n_cluster, m = prm->n_buckets, cap = prm->max_bucket_keys;
  if (np < 1 || nc < 1 || m < 1 || cap < 1) return false;
  if (nc % np != 0 || cap % np != 0) return false;
  const int P = nc / np;
  return m <= P;
}

static bool params_supported(const sa_lsa_params* prm) {
  return prm->d_idx == LSA_D && prm->n_cluster / prm->n_pool <= LSA_PMAX;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int LSA_MAX_BUCKETS_STREAM = 1 << 21;   // the threshold regime: up to 16M tokens at 8 keys a bucket

struct SearchPlan {
  bool stream;      // threshold regime (no score matrix)
  int R;            // query rows per chunk
  long long ld;     // score row stride (multiple of the tile)
  int psort;
  // table regime
  size_t off_qn, off_S, off_len, off_sel;
  // threshold regime
  int stride, n_s, cap, F;
  long long ld_s;
  size_t off_cs, off_stab, off_theta, off_cand, off_cnt, off_miss, off_frows, off_fpos, off_count, off_qnf, off_Sf,
      off_lenf, off_self, off_sig;
  size_t total;
};

static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

static bool use_stream(const sa_lsa_search_opts* o, long long nb) {
  return o->regime == SA_LSA_STREAM || (o->regime == SA_LSA_AUTO && nb > LSA_MAX_BUCKETS);
}

static SearchPlan plan_search(const sa_lsa_params* prm, const sa_lsa_search_opts* o, int n_q, int n_blocks) {
  SearchPlan pl{};
  const long long nb = (long long)n_blocks * prm->n_buckets;
  pl.stream = use_stream(o, nb);
  pl.ld = ((nb > 0 ? nb : 1) + LSA_TILE - 1) / LSA_TILE * LSA_TILE;
  pl.R = max(1, min(n_q, 8192));
  pl.psort = 1;
  while (pl.psort < o->p) pl.psort <<= 1;
  size_t off = 0;
  pl.off_qn = off;
  off = up256(off + (size_t)pl.R * LSA_D * 2);
  if (!pl.stream) {
    pl.off_S = off;
    off = up256(off + (size_t)pl.R * pl.ld * 4);
    pl.off_len = off;
    off = up256(off + (size_t)pl.R * 4);
    pl.off_sel = off;
    off = up256(off + (size_t)pl.R * o->p * 4);
    pl.total = off;
    return pl;
  }
  pl.stride = (int)max(1ll, (nb + LSA_SAMPLES - 1) / LSA_SAMPLES);
  pl.n_s = (int)max(1ll, (nb + pl.stride - 1) / pl.stride);
  pl.ld_s = ((long long)pl.n_s + LSA_TILE - 1) / LSA_TILE * LSA_TILE;
  pl.cap = 3 * o->p;
  pl.F = (int)max(16ll, min(1024ll, (512ll << 20) / (pl.ld * 4)));
  pl.off_cs = off;
  off = up256(off + (size_t)pl.n_s * LSA_D * 2);
  pl.off_stab = off;
  off = up256(off + (size_t)pl.R * pl.ld_s * 4);
  pl.off_theta = off;
  off = up256(off + (size_t)pl.R * 4);
  pl.off_cand = off;
  off = up256(off + (size_t)pl.R * pl.cap * 8);
  pl.off_cnt = off;
  off = up256(off + (size_t)pl.R * 4);
  pl.off_miss = off;
  off = up256(off + (size_t)pl.R * 4);
  pl.off_frows = off;
  off = up256(off + (size_t)pl.R * 4);
  pl.off_fpos = off;
  off = up256(off + (size_t)pl.R * 4);
  pl.off_count = off;
  off = up256(off + 4);
  pl.off_qnf = off;
  off = up256(off + (size_t)pl.F * LSA_D * 2);
  pl.off_Sf = off;
  off = up256(off + (size_t)pl.F * pl.ld * 4);
  pl.off_lenf = off;
  off = up256(off + (size_t)pl.F * 4);
  pl.off_self = off;
  off = up256(off + (size_t)pl.F * o->p * 4);
  pl.off_sig = off;
  off = up256(off + (size_t)pl.R * o->p * 8);
  pl.total = off;
  return pl;
}

static sa_status check_search(const sa_lsa_params* prm, const sa_lsa_search_opts* o, int n_q, int q_pos0,
                              int n_blocks) {
  if (!params_ok(prm) || o == nullptr) return SA_ERR_INVALID_ARGUMENT;
  if (n_q < 0 || q_pos0 < 0 || n_blocks < 0) return SA_ERR_INVALID_ARGUMENT;
  if (o->p < 1 || o->k < 1 || o->n_sink < 0 || o->n_window < 0) return SA_ERR_INVALID_ARGUMENT;
  if (o->regime < SA_LSA_AUTO || o->regime > SA_LSA_STREAM) return SA_ERR_INVALID_ARGUMENT;
  if (!params_supported(prm) || o->p > LSA_PSORT_MAX) return SA_ERR_UNSUPPORTED;
  const long long nb = (long long)n_blocks * prm->n_buckets;
  if (nb > (use_stream(o, nb) ? LSA_MAX_BUCKETS_STREAM : LSA_MAX_BUCKETS)) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

}  // namespace sa

using namespace sa;

extern "C" sa_status sa_lsa_build_buckets(const sa_lsa_params* prm, const void* k_idx, int32_t n_k, int32_t block0,
                                          int32_t n_blocks, void* centroids, int32_t* bucket_off,
                                          int32_t* bucket_keys, sa_device_status* status, cudaStream_t stream) {
  if (!params_ok(prm) || n_k < 0 || block0 < 0 || n_blocks < 0) return SA_ERR_INVALID_ARGUMENT;
  if ((long long)(block0 + (long long)n_blocks) * prm->n_cluster > n_k) return SA_ERR_INVALID_ARGUMENT;
  if (!params_supported(prm)) return SA_ERR_UNSUPPORTED;
  if (n_blocks > 0) {
    if (k_idx == nullptr || centroids == nullptr || bucket_off == nullptr || bucket_keys == nullptr)
      return SA_ERR_INVALID_ARGUMENT;
    if (!aligned16(k_idx) || !aligned16(centroids)) return SA_ERR_INVALID_ARGUMENT;
  }
  if (status != nullptr && cudaMemsetAsync(status, 0, sizeof(sa_device_status), stream) != cudaSuccess)
    return SA_ERR_CUDA;
  if (n_blocks == 0) return SA_OK;
  ClusterArgs a;
  a.k = static_cast<const __nv_bfloat16*>(k_idx);
  a.block0 = block0;
  a.n_pool = prm->n_pool;
  a.n_cluster = prm->n_cluster;
  a.P = prm->n_cluster / prm->n_pool;
  a.m = prm->n_buckets;
  a.cap = prm->max_bucket_keys / prm->n_pool;
  a.cent = static_cast<__nv_bfloat16*>(centroids);
  a.bucket_off = bucket_off;
  a.bucket_keys = bucket_keys;
  a.status = reinterpret_cast<uint32_t*>(status);
  const int smem = a.P * (LSA_D + LSA_MU_LD) * (int)sizeof(float);
  if (cudaFuncSetAttribute(lsa_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return SA_ERR_CUDA;
  lsa_cluster_kernel<<<n_blocks, LSA_CT, smem, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

extern "C" sa_status sa_lsa_search_workspace_size(const sa_lsa_params* prm, const sa_lsa_search_opts* o,
                                                  int32_t n_q, int32_t q_pos0, int32_t n_blocks, size_t* bytes) {
  if (bytes == nullptr) return SA_ERR_INVALID_ARGUMENT;
  const sa_status s = check_search(prm, o, n_q, q_pos0, n_blocks);
  if (s != SA_OK) return s;
  *bytes = n_q == 0 ? 0 : plan_search(prm, o, n_q, n_blocks).total;
  return SA_OK;
}

extern "C" sa_status sa_lsa_search(const sa_lsa_params* prm, const sa_lsa_search_opts* o, const void* q_idx,
                                   int32_t n_q, int32_t q_pos0, const void* centroids, const int32_t* bucket_off,
                                   const int32_t* bucket_keys, int32_t n_blocks, int32_t* J, void* ws,
                                   size_t ws_bytes, cudaStream_t stream) {
  const sa_status s = check_search(prm, o, n_q, q_pos0, n_blocks);
  if (s != SA_OK) return s;
  const SearchPlan pl = plan_search(prm, o, n_q, n_blocks);
  if (n_q > 0) {
    if (q_idx == nullptr || J == nullptr || ws == nullptr) return SA_ERR_INVALID_ARGUMENT;
    if (n_blocks > 0 && (centroids == nullptr || bucket_off == nullptr || bucket_keys == nullptr))
      return SA_ERR_INVALID_ARGUMENT;
    if (!aligned16(q_idx) || (n_blocks > 0 && !aligned16(centroids))) return SA_ERR_INVALID_ARGUMENT;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return SA_ERR_INVALID_ARGUMENT;
    if (ws_bytes < pl.total) return SA_ERR_WORKSPACE_TOO_SMALL;
  }
  if (o->status != nullptr && cudaMemsetAsync(o->status, 0, sizeof(sa_device_status), stream) != cudaSuccess)
    return SA_ERR_CUDA;
  if (n_q == 0) return SA_OK;
  uint8_t* w = static_cast<uint8_t*>(ws);
  __nv_bfloat16* qn = reinterpret_cast<__nv_bfloat16*>(w + pl.off_qn);
  const int nc = prm->n_cluster, m = prm->n_buckets, nb_all = n_blocks * m;
  const long long width = (long long)o->n_sink + o->n_window + o->k;
  const __nv_bfloat16* cent = static_cast<const __nv_bfloat16*>(centroids);
  uint32_t* status = reinterpret_cast<uint32_t*>(o->status);
  if (cudaFuncSetAttribute(lsa_score_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, LSA_SCORE_SMEM) !=
          cudaSuccess ||
      cudaFuncSetAttribute(lsa_score_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, LSA_SCORE_SMEM) !=
          cudaSuccess)
    return SA_ERR_CUDA;
  if (pl.stream) {
    const int tks = (int)sizeof(TkShared);
    if (cudaFuncSetAttribute(lsa_theta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tks) != cudaSuccess ||
        cudaFuncSetAttribute(lsa_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tks) != cudaSuccess)
      return SA_ERR_CUDA;
  }
  // the sampled centroids of the threshold estimate: every stride-th bucket
  __nv_bfloat16* cs = pl.stream ? reinterpret_cast<__nv_bfloat16*>(w + pl.off_cs) : nullptr;
  if (pl.stream && nb_all > 0 &&
      launch_gather_rows(cent, cs, nullptr, pl.n_s, LSA_D * 2, pl.stride, LSA_D * 2, stream) != cudaSuccess)
    return SA_ERR_CUDA;
  ScoreArgs base{};
  base.qn = qn;
  base.n_cluster = nc;
  base.m = m;
  base.n_blocks = n_blocks;
  base.col_stride = 1;
  base.status = status;
  base.budget = LSA_WAIT_BUDGET;
  for (int r0 = 0; r0 < n_q; r0 += pl.R) {
    const int rows = min(pl.R, n_q - r0), pos0 = q_pos0 + r0;
    lsa_qnorm_kernel<<<(rows + 255) / 256, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q_idx) + (long long)r0 * LSA_D, rows, qn);
    // buckets the chunk's last query sees (positions grow with the row)
    const int nbv = min(n_blocks, (pos0 + rows - 1) / nc) * m;
    const dim3 grid((nbv + LSA_TILE - 1) / LSA_TILE, (rows + LSA_TILE - 1) / LSA_TILE);
    base.rows = rows;
    base.pos0 = pos0;
    base.row_pos = nullptr;
    ExpandArgs ea{};
    if (!pl.stream) {
      // table regime: S written, the top-p of each row by the radix select
      float* S = reinterpret_cast<float*>(w + pl.off_S);
      int* len = reinterpret_cast<int*>(w + pl.off_len);
      int32_t* sel = reinterpret_cast<int32_t*>(w + pl.off_sel);
      if (nbv > 0) {
        ScoreArgs sa_ = base;
        sa_.cent = cent;
        sa_.n_buckets = nb_all;
        sa_.S = S;
        sa_.ld = pl.ld;
        lsa_score_kernel<false><<<grid, LSA_ST, LSA_SCORE_SMEM, stream>>>(sa_);
      }
      lsa_rowlen_kernel<<<(rows + 255) / 256, 256, 0, stream>>>(rows, pos0, nullptr, nc, m, n_blocks, len);
      if (launch_topk_table(S, rows, max(nbv, 1), pl.ld, pos0, o->p, sel, 1, nullptr, 0, len, stream) != cudaSuccess)
        return SA_ERR_CUDA;
      ea.sig_in = nullptr;
      ea.S = S;
      ea.ld = pl.ld;
      ea.sel = sel;
    } else {
      // threshold regime (appendix F.1 "Selection by threshold"): no score matrix
      float* stab = reinterpret_cast<float*>(w + pl.off_stab);
      float* theta = reinterpret_cast<float*>(w + pl.off_theta);
      unsigned long long* cand = reinterpret_cast<unsigned long long*>(w + pl.off_cand);
      int* cnt = reinterpret_cast<int*>(w + pl.off_cnt);
      int* miss = reinterpret_cast<int*>(w + pl.off_miss);
      int* frows = reinterpret_cast<int*>(w + pl.off_frows);
      int* fpos = reinterpret_cast<int*>(w + pl.off_fpos);
      int* count = reinterpret_cast<int*>(w + pl.off_count);
      unsigned long long* sig = reinterpret_cast<unsigned long long*>(w + pl.off_sig);
      if (nbv > 0) {
        ScoreArgs ss = base;              // sampled scores
        ss.cent = cs;
        ss.n_buckets = pl.n_s;
        ss.col_stride = pl.stride;
        ss.S = stab;
        ss.ld = pl.ld_s;
        const int nsv = (nbv + pl.stride - 1) / pl.stride;
        lsa_score_kernel<false>
            <<<dim3((nsv + LSA_TILE - 1) / LSA_TILE, grid.y), LSA_ST, LSA_SCORE_SMEM, stream>>>(ss);
      }
      lsa_theta_kernel<<<rows, TK_THREADS, sizeof(TkShared), stream>>>(stab, pl.ld_s, pos0, nc, m, n_blocks,
                                                                       pl.stride, o->p, pl.cap, o->test_hook, theta);
      if (cudaMemsetAsync(cnt, 0, (size_t)rows * 4, stream) != cudaSuccess) return SA_ERR_CUDA;
      if (nbv > 0) {
        ScoreArgs sc = base;              // the scan: compare with theta, list the hits
        sc.cent = cent;
        sc.n_buckets = nb_all;
        sc.theta = theta;
        sc.cand = cand;
        sc.cnt = cnt;
        sc.cap = pl.cap;
        lsa_score_kernel<true><<<grid, LSA_ST, LSA_SCORE_SMEM, stream>>>(sc);
      }
      lsa_select_kernel<<<rows, TK_THREADS, sizeof(TkShared), stream>>>(cand, cnt, pl.cap, pos0, nc, m, n_blocks,
                                                                        o->p, sig, miss, status);
      if (launch_compact_rows(miss, rows, frows, count, pos0, fpos, stream) != cudaSuccess) return SA_ERR_CUDA;
      // the fallback: the missed rows rescore their whole row (the host reads their count, as in the pages)
      int n_miss = 0;
      if (cudaMemcpyAsync(&n_miss, count, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
          cudaStreamSynchronize(stream) != cudaSuccess)
        return SA_ERR_CUDA;
      __nv_bfloat16* qnf = reinterpret_cast<__nv_bfloat16*>(w + pl.off_qnf);
      float* Sf = reinterpret_cast<float*>(w + pl.off_Sf);
      int* lenf = reinterpret_cast<int*>(w + pl.off_lenf);
      int32_t* self = reinterpret_cast<int32_t*>(w + pl.off_self);
      for (int f0 = 0; f0 < n_miss; f0 += pl.F) {
        const int nf = min(pl.F, n_miss - f0);
        if (launch_gather_rows(qn, qnf, frows + f0, nf, LSA_D * 2, 0, LSA_D * 2, stream) != cudaSuccess)
          return SA_ERR_CUDA;
        ScoreArgs sf = base;
        sf.cent = cent;
        sf.n_buckets = nb_all;
        sf.qn = qnf;
        sf.rows = nf;
        sf.row_pos = fpos + f0;
        sf.S = Sf;
        sf.ld = pl.ld;
        lsa_score_kernel<false>
            <<<dim3(grid.x, (nf + LSA_TILE - 1) / LSA_TILE), LSA_ST, LSA_SCORE_SMEM, stream>>>(sf);
        lsa_rowlen_kernel<<<(nf + 255) / 256, 256, 0, stream>>>(nf, 0, fpos + f0, nc, m, n_blocks, lenf);
        if (launch_topk_table(Sf, nf, max(nbv, 1), pl.ld, 0, o->p, self, 1, nullptr, 0, lenf, stream) !=
            cudaSuccess)
          return SA_ERR_CUDA;
        lsa_sig_from_table_kernel<<<nf, 256, 0, stream>>>(Sf, pl.ld, self, o->p, frows + f0, nf, sig);
      }
      ea.sig_in = sig;
      ea.S = nullptr;
      ea.ld = 0;
      ea.sel = nullptr;
    }
    ea.p = o->p;
    ea.psort = pl.psort;
    ea.bucket_off = bucket_off;
    ea.bucket_keys = bucket_keys;
    ea.off_stride = 0;
    ea.keys_stride = 0;
    ea.seq_lens = nullptr;
    ea.n_cluster = nc;
    ea.m = m;
    ea.rows = rows;
    ea.pos0 = pos0;
    ea.k = o->k;
    ea.n_sink = o->n_sink;
    ea.n_window = o->n_window;
    ea.J = J + (long long)r0 * width;
    lsa_expand_kernel<<<rows, TK_THREADS, 0, stream>>>(ea);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  }
  return SA_OK;
}

// ------------------------------------------------------------- decode step
namespace sa {

struct DecodePlan {
  long long ld;
  int psort;
  size_t off_qn, off_S, off_len, off_sel, total;
};

static DecodePlan plan_decode(const sa_lsa_params* prm, const sa_lsa_search_opts* o, int batch, int max_blocks) {
  DecodePlan pl{};
  const long long nb = (long long)max_blocks * prm->n_buckets;
  pl.ld = ((nb > 0 ? nb : 1) + LSA_TILE - 1) / LSA_TILE * LSA_TILE;
  pl.psort = 1;
  while (pl.psort < o->p) pl.psort <<= 1;
  size_t off = 0;
  pl.off_qn = off;
  off = up256(off + (size_t)batch * LSA_D * 2);
  pl.off_S = off;
  off = up256(off + (size_t)batch * pl.ld * 4);
  pl.off_len = off;
  off = up256(off + (size_t)batch * 4);
  pl.off_sel = off;
  off = up256(off + (size_t)batch * o->p * 4);
  pl.total = off;
  return pl;
}

static sa_status check_decode(const sa_lsa_params* prm, const sa_lsa_search_opts* o, int batch, int max_blocks) {
  if (!params_ok(prm) || o == nullptr) return SA_ERR_INVALID_ARGUMENT;
  if (batch < 0 || max_blocks < 0) return SA_ERR_INVALID_ARGUMENT;
  if (o->p < 1 || o->k < 1 || o->n_sink < 0 || o->n_window < 0) return SA_ERR_INVALID_ARGUMENT;
  if (!params_supported(prm) || o->p > LSA_PSORT_MAX) return SA_ERR_UNSUPPORTED;
  if ((long long)max_blocks * prm->n_buckets > LSA_MAX_BUCKETS) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

}  // namespace sa

extern "C" sa_status sa_lsa_decode_workspace_size(const sa_lsa_params* prm, const sa_lsa_search_opts* o,
                                                  int32_t batch, int32_t max_blocks, size_t* bytes) {
  if (bytes == nullptr) return SA_ERR_INVALID_ARGUMENT;
  const sa_status s = check_decode(prm, o, batch, max_blocks);
  if (s != SA_OK) return s;
  *bytes = batch == 0 ? 0 : plan_decode(prm, o, batch, max_blocks).total;
  return SA_OK;
}

extern "C" sa_status sa_lsa_decode(const sa_lsa_params* prm, const sa_lsa_search_opts* o, const void* q_idx,
                                   int32_t batch, const void* centroids, const int32_t* bucket_off,
                                   const int32_t* bucket_keys, int32_t max_blocks, const int32_t* n_blocks,
                                   const int32_t* seq_lens, int32_t* J, void* ws, size_t ws_bytes,
                                   cudaStream_t stream) {
  const sa_status s = check_decode(prm, o, batch, max_blocks);
  if (s != SA_OK) return s;
  const DecodePlan pl = plan_decode(prm, o, batch, max_blocks);
  if (batch > 0) {
    if (q_idx == nullptr || J == nullptr || ws == nullptr || n_blocks == nullptr || seq_lens == nullptr)
      return SA_ERR_INVALID_ARGUMENT;
    if (max_blocks > 0 && (centroids == nullptr || bucket_off == nullptr || bucket_keys == nullptr))
      return SA_ERR_INVALID_ARGUMENT;
    if (!aligned16(q_idx) || (max_blocks > 0 && !aligned16(centroids))) return SA_ERR_INVALID_ARGUMENT;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return SA_ERR_INVALID_ARGUMENT;
    if (ws_bytes < pl.total) return SA_ERR_WORKSPACE_TOO_SMALL;
  }
  if (o->status != nullptr && cudaMemsetAsync(o->status, 0, sizeof(sa_device_status), stream) != cudaSuccess)
    return SA_ERR_CUDA;
  if (batch == 0) return SA_OK;
  uint8_t* w = static_cast<uint8_t*>(ws);
  __nv_bfloat16* qn = reinterpret_cast<__nv_bfloat16*>(w + pl.off_qn);
  float* S = reinterpret_cast<float*>(w + pl.off_S);
  int* len = reinterpret_cast<int*>(w + pl.off_len);
  int32_t* sel = reinterpret_cast<int32_t*>(w + pl.off_sel);
  const int m = prm->n_buckets, nc = prm->n_cluster;
  const int nbmax = max_blocks * m;
  lsa_qnorm_kernel<<<(batch + 255) / 256, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(q_idx), batch, qn);
  DecodeScoreArgs da;
  da.cent = static_cast<const __nv_bfloat16*>(centroids);
  da.qn = qn;
  da.n_blocks = n_blocks;
  da.seq_lens = seq_lens;
  da.n_cluster = nc;
  da.m = m;
  da.max_blocks = max_blocks;
  da.S = S;
  da.ld = pl.ld;
  da.len = len;
  const dim3 grid((unsigned)max(1, (nbmax + 255) / 256), (unsigned)batch);
  lsa_decode_score_kernel<<<grid, 256, 0, stream>>>(da);
  cudaError_t e = launch_topk_table(S, batch, max(nbmax, 1), pl.ld, 0, o->p, sel, 1, nullptr, 0, len, stream);
  if (e != cudaSuccess) return SA_ERR_CUDA;
  ExpandArgs ea{};
  ea.sig_in = nullptr;
  ea.S = S;
  ea.ld = pl.ld;
  ea.sel = sel;
  ea.p = o->p;
  ea.psort = pl.psort;
  ea.bucket_off = bucket_off;
  ea.bucket_keys = bucket_keys;
  ea.off_stride = (long long)max_blocks * m;
  ea.keys_stride = (long long)max_blocks * nc;
  ea.n_cluster = nc;
  ea.m = m;
  ea.rows = batch;
  ea.pos0 = 0;
  ea.seq_lens = seq_lens;
  ea.k = o->k;
  ea.n_sink = o->n_sink;
  ea.n_window = o->n_window;
  ea.J = J;
  lsa_expand_kernel<<<batch, TK_THREADS, 0, stream>>>(ea);
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

namespace sa {
SA_DEBUG_UNIT(dbg_read_lsa)
}  // namespace sa
