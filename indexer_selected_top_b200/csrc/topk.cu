// topk.cu -- exact per-row top-k by radix select.
//
// Order: higher fp32 score first, at equal scores the lower key index first.
// This is the packed 64-bit key of Latent Sparse Attention appendix F.1
// ("Selection by threshold"): order-preserving score bits in the upper 32
// bits, the inverted id in the lower 32, so a larger packed key is a better
// score or, at equal scores, a lower id. The cut is found by radix select
// (Alabi et al. 2012; Zhang et al. 2023a, as cited there); the output is
// never sorted because the attention does not depend on the order.
//
// One CTA per row. Passes over the row in global memory histogram 12-bit
// digits of the 32-bit score key until the bucket holding the cut is small
// enough for shared memory; a last pass writes every key above that bucket
// and gathers the bucket's (key, index) pairs, which a shared-memory radix
// select over the packed 64-bit keys finishes. A bucket of identical scores
// larger than shared memory is resolved by an ordered scan (lowest indices).
#include "sa_internal.h"

namespace sa {

constexpr int TK_THREADS = 512;
constexpr int TK_CAP = 12288;          // (key, index) pairs kept in shared memory
constexpr int TK_HBITS = 12;
constexpr int TK_HBINS = 1 << TK_HBITS;
constexpr uint32_t KEY_NEG_INF = 0x007FFFFFu;   // score key of -inf

__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0u;                    // -0 sorts with +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Row description: column c of the row holds the score of key key_of(c);
// only columns [0, ncols) exist; invalid columns are skipped.
struct RowView {
  const float* s;
  int ncols;
  int vis_mode;       // 0 causal/decode (every column valid), 2 gathered (valid iff > -inf)
  const int* kept;    // vis_mode 2: kept blocks of this row
  __device__ __forceinline__ bool valid_key(uint32_t key) const { return vis_mode != 2 || key != KEY_NEG_INF; }
  __device__ __forceinline__ int key_of(int c) const { return vis_mode == 2 ? kept[c >> 6] * 64 + (c & 63) : c; }
};

struct TkShared {
  uint32_t hist[TK_HBINS];
  unsigned long long cand[TK_CAP];
  int n_out;
  int n_cand;
  int bucket;
  int above;
  int total;
  int red[TK_THREADS / 32];
};

// block-wide sum
__device__ int block_sum(int v, int* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int r = 0;
  for (int i = 0; i < TK_THREADS / 32; ++i) r += red[i];
  __syncthreads();
  return r;
}

// block-wide exclusive prefix sum (threads in order)
__device__ int block_excl_scan(int v, int* red, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) red[warp] = x;
  __syncthreads();
  int base = 0, tot = 0;
  for (int i = 0; i < TK_THREADS / 32; ++i) {
    if (i < warp) base += red[i];
    tot += red[i];
  }
  __syncthreads();
  *total = tot;
  return base + x - v;
}

// Find, in hist[0..nbins), the bucket b with sum(hist[b+1..]) < need <= sum(hist[b..]).
// Sets sh.bucket and sh.above (count strictly above the bucket).
__device__ void find_bucket(TkShared& sh, int nbins, int need) {
  // each thread owns a contiguous range of bins (from the top)
  const int per = (nbins + TK_THREADS - 1) / TK_THREADS;
  const int hi = nbins - threadIdx.x * per;              // exclusive upper bin of this thread
  const int lo = max(0, hi - per);
  int mine = 0;
  for (int b = lo; b < hi; ++b) mine += sh.hist[b];
  int tot;
  const int before = block_excl_scan(mine, sh.red, &tot);  // bins above this thread's range
  if (before < need && before + mine >= need) {
    int acc = before;
    for (int b = hi - 1; b >= lo; --b) {
      if (acc + (int)sh.hist[b] >= need) {
        sh.bucket = b;
        sh.above = acc;
        break;
      }
      acc += sh.hist[b];
    }
  }
  __syncthreads();
}

// Select the `need` largest of sh.cand[0..cnt) (unique 64-bit keys) and emit them.
template <class Emit>
__device__ void smem_select64(TkShared& sh, int cnt, int need, Emit emit) {
  uint64_t hi = 0;
  int nb = 0;
  uint64_t cut = 0;
  if (need >= cnt) {
    cut = 0;
  } else {
    while (true) {
      for (int b = threadIdx.x; b < 256; b += TK_THREADS) sh.hist[b] = 0;
      __syncthreads();
      const int sh_digit = 64 - nb - 8;
      for (int j = threadIdx.x; j < cnt; j += TK_THREADS) {
        const uint64_t key = sh.cand[j];
        if (nb == 0 || (key >> (64 - nb)) == hi) atomicAdd(&sh.hist[(key >> sh_digit) & 255u], 1u);
      }
      __syncthreads();
      find_bucket(sh, 256, need);
      const int d = sh.bucket;
      need -= sh.above;
      hi = (hi << 8) | (uint64_t)d;
      nb += 8;
      const int inb = sh.hist[d];
      __syncthreads();
      if (inb == need || nb == 64) {
        cut = hi << (64 - nb);
        break;
      }
    }
  }
  for (int j = threadIdx.x; j < cnt; j += TK_THREADS) {
    const uint64_t key = sh.cand[j];
    if (key >= cut) emit(key);
  }
  __syncthreads();
}

__device__ void topk_row(TkShared& sh, const RowView& rv, int k, int32_t* out) {
  const int tid = threadIdx.x;
  if (tid == 0) sh.n_out = 0;
  // number of valid columns
  int nvalid = rv.ncols;
  if (rv.vis_mode == 2) {
    int c = 0;
    for (int j = tid; j < rv.ncols; j += TK_THREADS) c += rv.valid_key(score_key(rv.s[j])) ? 1 : 0;
    nvalid = block_sum(c, sh.red);
  }
  __syncthreads();
  if (nvalid <= k) {
    // every valid column, in order
    for (int base = 0; base < rv.ncols; base += TK_THREADS) {
      const int j = base + tid;
      const bool v = j < rv.ncols && rv.valid_key(score_key(rv.s[j]));
      int tot;
      const int pos = block_excl_scan(v ? 1 : 0, sh.red, &tot);
      if (v) out[sh.n_out + pos] = rv.key_of(j);
      __syncthreads();
      if (tid == 0) sh.n_out += tot;
      __syncthreads();
    }
    for (int j = nvalid + tid; j < k; j += TK_THREADS) out[j] = -1;
    return;
  }
  // ---- refine the cut bucket in global memory: 12 + 12 + 8 bits ----
  uint32_t prefix = 0;
  int pbits = 0;
  int need = k;
  bool fits = false;
  while (pbits < 32) {
    const int db = (pbits == 24) ? 8 : TK_HBITS;
    const int nbins = 1 << db;
    for (int b = tid; b < nbins; b += TK_THREADS) sh.hist[b] = 0;
    __syncthreads();
    const int sdig = 32 - pbits - db;
    for (int j = tid; j < rv.ncols; j += TK_THREADS) {
      const uint32_t key = score_key(rv.s[j]);
      if (!rv.valid_key(key)) continue;
      if (pbits == 0 || (key >> (32 - pbits)) == prefix) atomicAdd(&sh.hist[(key >> sdig) & (nbins - 1)], 1u);
    }
    __syncthreads();
    find_bucket(sh, nbins, need);
    const int bsel = sh.bucket;
    need -= sh.above;
    const int inb = sh.hist[bsel];
    prefix = (prefix << db) | (uint32_t)bsel;
    pbits += db;
    __syncthreads();
    if (inb <= TK_CAP) {
      fits = true;
      break;
    }
  }
  // ---- emit every key above the bucket; gather the bucket ----
  if (tid == 0) sh.n_cand = 0;
  __syncthreads();
  for (int j = tid; j < rv.ncols; j += TK_THREADS) {
    const uint32_t key = score_key(rv.s[j]);
    if (!rv.valid_key(key)) continue;
    const uint32_t top = key >> (32 - pbits);
    if (top > prefix) {
      out[atomicAdd(&sh.n_out, 1)] = rv.key_of(j);
    } else if (top == prefix && fits) {
      const int p = atomicAdd(&sh.n_cand, 1);
      sh.cand[p] = ((unsigned long long)key << 32) | (uint32_t)(~(uint32_t)j);
    }
  }
  __syncthreads();
  if (fits) {
    const int cnt = sh.n_cand;
    smem_select64(sh, cnt, need, [&](uint64_t key) {
      const int j = (int)(~(uint32_t)(key & 0xFFFFFFFFu));
      out[atomicAdd(&sh.n_out, 1)] = rv.key_of(j);
    });
  } else {
    // more than TK_CAP identical scores at the cut: the lowest columns win
    for (int base = 0; base < rv.ncols && need > 0; base += TK_THREADS) {
      const int j = base + tid;
      bool eq = false;
      if (j < rv.ncols) {
        const uint32_t key = score_key(rv.s[j]);
        eq = rv.valid_key(key) && key == prefix;
      }
      int tot;
      const int pos = block_excl_scan(eq ? 1 : 0, sh.red, &tot);
      if (eq && pos < need) out[atomicAdd(&sh.n_out, 1)] = rv.key_of(j);
      need -= tot;
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(TK_THREADS, 1)
    topk_table_kernel(const float* scores, int n_rows, int n_cols, long long ld, int q_pos0, int k, int32_t* idx,
                      int vis_mode, const int* kept, int keep, const int* seq_lens) {
  extern __shared__ uint8_t tk_raw[];
  TkShared& sh = *reinterpret_cast<TkShared*>(tk_raw);
  const int row = blockIdx.x;
  RowView rv;
  rv.s = scores + (long long)row * ld;
  rv.vis_mode = vis_mode;
  rv.kept = nullptr;
  if (vis_mode == 0) {
    rv.ncols = max(0, min(n_cols, q_pos0 + row + 1));
  } else if (vis_mode == 1) {
    rv.ncols = seq_lens ? min(n_cols, seq_lens[row]) : n_cols;
  } else {
    rv.kept = kept + (long long)row * keep;
    int nb = 0;
    while (nb < keep && rv.kept[nb] >= 0) ++nb;
    rv.ncols = min(n_cols, nb * 64);
  }
  topk_row(sh, rv, k, idx + (long long)row * k);
}

cudaError_t launch_topk_table(const float* scores, int n_rows, int n_cols, long long ld, int q_pos0, int k,
                              int32_t* idx, int vis_mode, const int* kept, int keep, const int* seq_lens,
                              cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  const int smem = (int)sizeof(TkShared);
  cudaError_t e = cudaFuncSetAttribute(topk_table_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  topk_table_kernel<<<n_rows, TK_THREADS, smem, st>>>(scores, n_rows, n_cols, ld, q_pos0, k, idx, vis_mode, kept,
                                                       keep, seq_lens);
  return cudaGetLastError();
}

// ------------------------------------------------------------ stage-1 keep
// Kept blocks of query row t (absolute position p = q_pos0 + t): block 0, the
// current block cur = p / block, and the best keep-2 blocks of [1, cur-1] by
// (score desc, block asc); written ascending, -1 padded to `keep`.
struct BsShared {
  TkShared tk;
  uint8_t flag[16384];
};

__global__ void __launch_bounds__(TK_THREADS, 1)
    block_select_kernel(const float* bscores, int n_q, int nb, long long ld, int q_pos0, int block, int keep,
                        int* kept) {
  extern __shared__ uint8_t bs_raw[];
  BsShared& sh = *reinterpret_cast<BsShared*>(bs_raw);
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int p = q_pos0 + t;
  const int cur = p / block;
  int* out = kept + (long long)t * keep;
  const int n_other = max(0, min(cur - 1, nb - 1));
  for (int b = tid; b <= cur; b += TK_THREADS) sh.flag[b] = (b == 0 || b == cur) ? 1 : 0;
  __syncthreads();
  const float* row = bscores + (long long)t * ld;
  if (n_other <= keep - 2) {
    for (int b = 1 + tid; b <= n_other; b += TK_THREADS) sh.flag[b] = 1;
  } else {
    // all others in shared memory as packed keys (score key, ~block)
    for (int j = tid; j < n_other; j += TK_THREADS) {
      const int b = 1 + j;
      sh.tk.cand[j] = ((unsigned long long)score_key(row[b]) << 32) | (uint32_t)(~(uint32_t)b);
    }
    __syncthreads();
    smem_select64(sh.tk, n_other, keep - 2, [&](uint64_t key) {
      const int b = (int)(~(uint32_t)(key & 0xFFFFFFFFu));
      sh.flag[b] = 1;
    });
  }
  __syncthreads();
  // ascending compaction of the flags
  int n_out = 0;
  for (int base = 0; base <= cur; base += TK_THREADS) {
    const int b = base + tid;
    const bool f = b <= cur && sh.flag[b];
    int tot;
    const int pos = block_excl_scan(f ? 1 : 0, sh.tk.red, &tot);
    if (f && n_out + pos < keep) out[n_out + pos] = b;
    n_out += tot;
    __syncthreads();
  }
  for (int j = min(n_out, keep) + tid; j < keep; j += TK_THREADS) out[j] = -1;
}

cudaError_t launch_block_select(const float* bscores, int n_q, int nb, long long ld, int q_pos0, int block,
                                int keep, int* kept, cudaStream_t st) {
  if (n_q <= 0) return cudaSuccess;
  const int smem = (int)sizeof(BsShared);
  cudaError_t e = cudaFuncSetAttribute(block_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  block_select_kernel<<<n_q, TK_THREADS, smem, st>>>(bscores, n_q, nb, ld, q_pos0, block, keep, kept);
  return cudaGetLastError();
}

}  // namespace sa
