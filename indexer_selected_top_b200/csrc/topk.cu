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
#include "radix.cuh"
#include "ptx.cuh"
#include "sa_internal.h"

namespace sa {

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
                      int vis_mode, const int* kept, int keep, const int* seq_lens, const int* row_pos,
                      const int* out_rows, const int* only_flagged, const int* row_count, int row_base) {
  extern __shared__ uint8_t tk_raw[];
  TkShared& sh = *reinterpret_cast<TkShared*>(tk_raw);
  const int row = blockIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  if (only_flagged != nullptr && only_flagged[row] == 0) return;   // this row was selected already
  if (row_count != nullptr && row >= *row_count - row_base) return;  // past the rows flagged on the device
  RowView rv;
  rv.s = scores + (long long)row * ld;
  rv.vis_mode = vis_mode;
  rv.kept = nullptr;
  if (vis_mode == 0) {
    rv.ncols = max(0, min(n_cols, (row_pos ? row_pos[row] : q_pos0 + row) + 1));
    rv.vis_mode = 0;
  } else if (vis_mode == 1) {
    rv.ncols = seq_lens ? min(n_cols, seq_lens[row]) : n_cols;
  } else {
    rv.kept = kept + (long long)row * keep;
    int nb = 0;
    while (nb < keep && rv.kept[nb] >= 0) ++nb;
    rv.ncols = min(n_cols, nb * 64);
  }
  topk_row(sh, rv, k, idx + (long long)(out_rows ? out_rows[row] : row) * k);
}

cudaError_t launch_topk_table(const float* scores, int n_rows, int n_cols, long long ld, int q_pos0, int k,
                              int32_t* idx, int vis_mode, const int* kept, int keep, const int* seq_lens,
                              cudaStream_t st, const int* row_pos, const int* out_rows, const int* only_flagged,
                              const int* row_count, int row_base, bool pdl) {
  if (n_rows <= 0) return cudaSuccess;
  const int smem = (int)sizeof(TkShared);
  cudaError_t e = cudaFuncSetAttribute(topk_table_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_k(topk_table_kernel, dim3(n_rows), dim3(TK_THREADS), smem, st, pdl, scores, n_rows, n_cols, ld,
                  q_pos0, k, idx, vis_mode, kept, keep, seq_lens, row_pos, out_rows, only_flagged, row_count,
                  row_base);
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
