// stream.cu -- the streaming exact selector: top-k without a score table.
//
// Latent Sparse Attention appendix F.1 ("Selection by threshold", "Flat
// prefill"): before the scan, set a threshold theta_t per query from a
// sample of its row; the scan compares each score with theta_t once and
// appends the keys at or above it to the query's list L_t as packed 64-bit
// keys; only L_t is then ranked (radix select). When L_t holds every key
// with score >= theta_t and at least k of them, the top-k is inside it. A
// query the estimate misses -- fewer than k listed, or more than the list
// holds -- falls back to its whole row (done here by the table path on the
// missed rows only). HyScale's HyTopK also computes each query's exact top-k
// on the fly without a full score table (theflow "related" page).
//
// theta_t: the sample holds every m-th key (key m*i); query t sees the
// n_vs = min(n_s, p / m + 1) samples at positions <= p. To list about
// gamma * k of its n_vis = p + 1 keys it takes the n_theta-th largest sample
// score, n_theta = round(gamma * k * n_vs / n_vis). Rows whose visible keys
// all fit in the list take theta = -inf.
#include "radix.cuh"
#include "ptx.cuh"
#include "sa_internal.h"

namespace sa {

// dst row i = src row rows[i] (or row i * m_stride when rows is null)
__global__ void gather_rows_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, const int* rows,
                                   long long src_stride, int m_stride, int row_bytes) {
  const int i = blockIdx.x;
  const long long r = rows ? (long long)rows[i] : (long long)i * m_stride;
  const uint32_t* s = reinterpret_cast<const uint32_t*>(src + r * src_stride);
  uint32_t* d = reinterpret_cast<uint32_t*>(dst + (long long)i * row_bytes);
  for (int j = threadIdx.x; j < row_bytes / 4; j += blockDim.x) d[j] = s[j];
}

cudaError_t launch_gather_rows(const void* src, void* dst, const int* rows, int n_rows, long long src_stride,
                               int m_stride, int row_bytes, cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  if (row_bytes % 4 != 0) return cudaErrorInvalidValue;
  gather_rows_kernel<<<n_rows, 128, 0, st>>>(static_cast<const uint8_t*>(src), static_cast<uint8_t*>(dst), rows,
                                             src_stride, m_stride, row_bytes);
  return cudaGetLastError();
}

// sample keys a theta thread holds in registers (TH_REG * TK_THREADS = 16,384
// samples, the most a row of the library's plans has)
constexpr int TH_REG = 32;

static __device__ __forceinline__ float key_to_float(uint32_t key) {
  const uint32_t b = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
  return __uint_as_float(b);
}

// theta[t] for chunk row t (absolute position q_pos0 + t); stab row t holds
// the scores of samples 0..n_s-1 (entries beyond the visible ones unused)
// Decode (decode != 0): row t is sequence t's written score row; its samples
// are every m-th visible score (n_vis = seq_lens[t], or n_k).
__global__ void __launch_bounds__(TK_THREADS, 1)
    theta_kernel(const float* __restrict__ stab, int n_s, long long ld, int q_pos0, int m, int n_k, int k, int cap,
                 float gamma, int hook, float* __restrict__ theta, int decode, const int* seq_lens,
                 int* __restrict__ zero_cnt) {
  extern __shared__ uint8_t th_raw[];
  TkShared& sh = *reinterpret_cast<TkShared*>(th_raw);
  const int t = blockIdx.x, tid = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  if (zero_cnt != nullptr && tid == 0) zero_cnt[t] = 0;      // the row's list starts empty
  const int p = decode ? ((seq_lens ? min(seq_lens[t], n_k) : n_k) - 1) : q_pos0 + t;
  const int n_vis = min(n_k, p + 1);
  const int sstride = decode ? m : 1;
  float th;
  if (hook == SA_HOOK_THETA_POS_INF) {
    th = INFINITY;
  } else if (hook == SA_HOOK_THETA_NEG_INF || hook == SA_HOOK_THETA_RUNNING || n_vis <= cap) {
    th = -INFINITY;
  } else {
    const int n_vs = decode ? (n_vis + m - 1) / m : min(n_s, p / m + 1);
    const long long want = llrintf(gamma * (float)k * (float)n_vs / (float)n_vis);
    int need = (int)max(1ll, min((long long)n_vs, want));
    const float* row = stab + (long long)t * ld;
    // the samples' keys, read once (all loads in flight together) and kept in
    // registers for the three passes; a longer sample row (not planned by the
    // library) is re-read from memory in every pass
    uint32_t kr[TH_REG];
    const bool in_regs = n_vs <= TH_REG * TK_THREADS;
    if (in_regs) {
#pragma unroll
      for (int i = 0; i < TH_REG; ++i) {
        const int j = tid + i * TK_THREADS;
        kr[i] = (j < n_vs) ? score_key(row[(long long)j * sstride]) : 0u;
      }
    }
    uint32_t prefix = 0;
    int pbits = 0;
    // two 12-bit passes fix the n_theta-th key to its top 24 bits; theta is
    // the smallest key with that prefix, so it lists at least the exact
    // threshold's keys (any threshold keeps the selection exact; a third pass
    // for the last 8 bits would shorten the list by the few samples within
    // 2^-15 of it)
    while (pbits < 24) {
      const int db = TK_HBITS;
      const int nbins = 1 << db;
      for (int b = tid; b < nbins; b += TK_THREADS) sh.hist[b] = 0;
      __syncthreads();
      const int sdig = 32 - pbits - db;
      auto count = [&](uint32_t key) {
        if (pbits == 0 || (key >> (32 - pbits)) == prefix) atomicAdd(&sh.hist[(key >> sdig) & (nbins - 1)], 1u);
      };
      if (in_regs) {
#pragma unroll
        for (int i = 0; i < TH_REG; ++i)
          if (tid + i * TK_THREADS < n_vs) count(kr[i]);
      } else {
        for (int j = tid; j < n_vs; j += TK_THREADS) count(score_key(row[(long long)j * sstride]));
      }
      __syncthreads();
      find_bucket(sh, nbins, need);
      need -= sh.above;
      prefix = (prefix << db) | (uint32_t)sh.bucket;
      pbits += db;
      __syncthreads();
    }
    // the bucket below every finite score is -inf's (its other keys are NaN patterns)
    th = ((prefix << 8) < 0x00800000u) ? -INFINITY : key_to_float(prefix << 8);
  }
  if (tid == 0) theta[t] = th;
}

cudaError_t launch_theta(const float* stab, int n_rows, int n_s, long long ld, int q_pos0, int m, int n_k, int k,
                         int cap, float gamma, int hook, float* theta, cudaStream_t st, int decode,
                         const int* seq_lens, int* zero_cnt, bool pdl) {
  if (n_rows <= 0) return cudaSuccess;
  const int smem = (int)sizeof(TkShared);
  cudaError_t e = cudaFuncSetAttribute(theta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_k(theta_kernel, dim3(n_rows), dim3(TK_THREADS), smem, st, pdl, stab, n_s, ld, q_pos0, m, n_k, k, cap,
                  gamma, hook, theta, decode, seq_lens, zero_cnt);
}

// Exact top-k of each row's candidate list; rows whose list missed (fewer
// than min(k, visible) candidates, or more than cap) are flagged for the
// whole-row fallback and their index rows left to it.
__global__ void __launch_bounds__(TK_THREADS, 1)
    select_cand_kernel(const unsigned long long* __restrict__ cand, const int* __restrict__ cnt, int cap,
                       int q_pos0, int n_k, int k, int32_t* __restrict__ idx, int* __restrict__ miss,
                       uint32_t* status, int decode, const int* seq_lens) {
  extern __shared__ uint8_t sc_raw[];
  TkShared& sh = *reinterpret_cast<TkShared*>(sc_raw);
  const int t = blockIdx.x, tid = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  const int n_vis = decode ? (seq_lens ? min(seq_lens[t], n_k) : n_k) : min(n_k, q_pos0 + t + 1);
  const int need = min(k, n_vis);
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
  int32_t* out = idx + (long long)t * k;
  smem_select64(sh, c, need, [&](uint64_t key) {
    out[atomicAdd(&sh.n_out, 1)] = (int32_t)(~(uint32_t)(key & 0xFFFFFFFFu));
  });
  for (int j = need + tid; j < k; j += TK_THREADS) out[j] = -1;
}

cudaError_t launch_select_cand(const unsigned long long* cand, const int* cnt, const float* theta, int n_rows,
                               int cap, int q_pos0, int n_k, int k, int32_t* idx, int* miss_flag, uint32_t* status,
                               cudaStream_t st, int decode, const int* seq_lens, bool pdl) {
  (void)theta;
  if (n_rows <= 0) return cudaSuccess;
  if (cap > TK_CAP) return cudaErrorNotSupported;
  const int smem = (int)sizeof(TkShared);
  cudaError_t e = cudaFuncSetAttribute(select_cand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_k(select_cand_kernel, dim3(n_rows), dim3(TK_THREADS), smem, st, pdl, cand, cnt, cap, q_pos0, n_k, k,
                  idx, miss_flag, status, decode, seq_lens);
}

// Decode lists from the written score rows: every visible score >= theta[b]
// of sequence b is appended to b's list, packed as in the indexer's candidate
// mode. Grid: (row chunks of COLLECT_CHUNK scores, sequences). A CTA gathers
// its hits in shared memory and reserves their place in the list with one
// global atomic (a global atomic per warp contends on the 64 counters).
constexpr int COLLECT_CHUNK = 4096;

__global__ void __launch_bounds__(256)
    collect_cand_kernel(const float* __restrict__ rows, long long ld, int n_k, const int* __restrict__ seq_lens,
                        const float* __restrict__ theta, unsigned long long* __restrict__ cand, int* __restrict__ cnt,
                        int cap) {
  __shared__ unsigned long long hits[COLLECT_CHUNK];
  __shared__ int n_hit, base;
  const int b = blockIdx.y;
  pdl_launch_dependents();
  pdl_wait();
  const int n_vis = seq_lens ? min(seq_lens[b], n_k) : n_k;
  const float th = theta[b];
  const float* row = rows + (long long)b * ld;
  const int lo = blockIdx.x * COLLECT_CHUNK, hi = min(n_vis, lo + COLLECT_CHUNK);
  if (threadIdx.x == 0) n_hit = 0;
  __syncthreads();
  auto take = [&](float sc, int s) {
    if (sc >= th) hits[atomicAdd(&n_hit, 1)] = ((unsigned long long)score_key(sc) << 32) | (uint32_t)(~(uint32_t)s);
  };
  if (hi - lo == COLLECT_CHUNK && (ld & 3) == 0 && (reinterpret_cast<uintptr_t>(row) & 15u) == 0) {
    // a whole chunk: four 16-byte loads per thread, all in flight together
    float4 v[COLLECT_CHUNK / 1024];
#pragma unroll
    for (int i = 0; i < COLLECT_CHUNK / 1024; ++i)
      v[i] = *reinterpret_cast<const float4*>(row + lo + 4 * (threadIdx.x + 256 * i));
#pragma unroll
    for (int i = 0; i < COLLECT_CHUNK / 1024; ++i) {
      const int s = lo + 4 * (threadIdx.x + 256 * i);
      take(v[i].x, s);
      take(v[i].y, s + 1);
      take(v[i].z, s + 2);
      take(v[i].w, s + 3);
    }
  } else {
    for (int s = lo + threadIdx.x; s < hi; s += 256) take(row[s], s);
  }
  __syncthreads();
  const int n = n_hit;
  if (n == 0) return;
  if (threadIdx.x == 0) base = atomicAdd(&cnt[b], n);
  __syncthreads();
  for (int j = threadIdx.x; j < n; j += 256)
    if (base + j < cap) cand[(long long)b * cap + base + j] = hits[j];
}

cudaError_t launch_collect_cand(const float* rows, int batch, long long ld, int n_k, const int* seq_lens,
                                const float* theta, unsigned long long* cand, int* cnt, int cap, cudaStream_t st,
                                bool pdl) {
  if (batch <= 0) return cudaSuccess;
  const int chunks = (n_k + COLLECT_CHUNK - 1) / COLLECT_CHUNK;
  return launch_k(collect_cand_kernel, dim3(chunks, batch), dim3(256), 0, st, pdl, rows, ld, n_k, seq_lens, theta,
                  cand, cnt, cap);
}

// Running threshold (Latent Sparse Attention appendix F.1, "Selection by
// threshold": any k listed keys lower-bound the k-th best, so a key below the
// k-th best listed so far is never selected). One CTA per row: a list of c
// entries, k < c <= cap, is cut to its k best packed keys, written back to
// the front of the list, and the row's threshold rises to the score of the
// k-th. A list that overflowed (c > cap) lost entries and is left alone; its
// row falls back later.
__global__ void __launch_bounds__(TK_THREADS, 1)
    raise_theta_kernel(unsigned long long* __restrict__ cand, int* __restrict__ cnt, float* __restrict__ theta,
                       int cap, int k) {
  extern __shared__ uint8_t rt_raw[];
  TkShared& sh = *reinterpret_cast<TkShared*>(rt_raw);
  __shared__ unsigned long long kmin;
  const int t = blockIdx.x, tid = threadIdx.x;
  const int c = cnt[t];
  if (c <= k || c > cap) return;
  unsigned long long* row = cand + (long long)t * cap;
  for (int j = tid; j < c; j += TK_THREADS) sh.cand[j] = row[j];
  if (tid == 0) {
    sh.n_out = 0;
    kmin = ~0ull;
  }
  __syncthreads();
  smem_select64(sh, c, k, [&](uint64_t key) {
    row[atomicAdd(&sh.n_out, 1)] = key;
    atomicMin(&kmin, (unsigned long long)key);
  });
  if (tid == 0) {
    cnt[t] = k;
    const uint32_t hk = (uint32_t)(kmin >> 32);            // the k-th key's score bits, order-preserving
    const uint32_t b = (hk & 0x80000000u) ? (hk & 0x7FFFFFFFu) : ~hk;
    theta[t] = fmaxf(theta[t], __uint_as_float(b));
  }
}

cudaError_t launch_raise_theta(unsigned long long* cand, int* cnt, float* theta, int n_rows, int cap, int k,
                               cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  if (cap > TK_CAP) return cudaErrorNotSupported;
  const int smem = (int)sizeof(TkShared);
  cudaError_t e = cudaFuncSetAttribute(raise_theta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  raise_theta_kernel<<<n_rows, TK_THREADS, smem, st>>>(cand, cnt, theta, cap, k);
  return cudaGetLastError();
}

// Ordered compaction of the flagged rows: rows[] ascending, count[0], and
// pos[i] = q_pos0 + rows[i] (their absolute positions). One CTA.
__global__ void __launch_bounds__(1024) compact_rows_kernel(const int* __restrict__ flags, int n_rows,
                                                            int* __restrict__ rows, int* __restrict__ count,
                                                            int q_pos0, int* __restrict__ pos) {
  __shared__ int red[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n_rows + 1023) / 1024;
  const int lo = min(n_rows, tid * per), hi = min(n_rows, lo + per);
  int mine = 0;
  for (int i = lo; i < hi; ++i) mine += flags[i] != 0;
  int x = mine;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  __syncthreads();
  int base = 0, tot = 0;
  for (int w = 0; w < 32; ++w) {
    if (w < warp) base += red[w];
    tot += red[w];
  }
  int o = base + x - mine;
  for (int i = lo; i < hi; ++i)
    if (flags[i] != 0) {
      rows[o] = i;
      pos[o] = q_pos0 + i;
      ++o;
    }
  if (tid == 0) count[0] = tot;
}

cudaError_t launch_compact_rows(const int* flags, int n_rows, int* rows, int* count, int q_pos0, int* pos,
                                cudaStream_t st) {
  compact_rows_kernel<<<1, 1024, 0, st>>>(flags, n_rows, rows, count, q_pos0, pos);
  return cudaGetLastError();
}

}  // namespace sa
