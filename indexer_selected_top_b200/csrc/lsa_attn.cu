// lsa_attn.cu -- attention over LSA index rows on the tensor cores.
//
// An LSA index row J_i is the query's sinks, its window of the n_window most
// recent keys, and its k long-range keys (Latent Sparse Attention section 3.2;
// one J_i is shared by all query heads). The two parts have different reuse:
// consecutive queries share almost all of their sinks and windows, while
// queries that look up the same buckets share their long-range keys wherever
// they sit. So the attention runs in two passes of the grouped tcgen05 kernel
// (8 queries x 16 heads = one M = 128 tile over the union of the group's keys,
// a query's unselected keys masked in the MMA), then merges them:
//   local:  groups of 8 consecutive queries over their sinks and windows (one
//           range of at most n_window + 7 keys plus the sinks);
//   far:    groups of 8 queries whose long-range keys overlap, found by a
//           MinHash signature (the smallest hash over a row's long-range keys:
//           two rows share it with probability equal to the Jaccard similarity
//           of their key sets) sorted within windows of queries; each group's
//           union is built from per-query bitmaps over the keys in shared memory;
//   merge:  O = (e^lse_l O_l + e^lse_f O_f) / (e^lse_l + e^lse_f), lse = log of
//           the sum: softmax over the disjoint union of the two parts.
#include <cuda_bf16.h>

#include "debug.cuh"
#include "radix.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int LA_GA = kGroupQueries;     // queries per group (one M = 128 tile with 16 heads)
constexpr int LA_MAX_KEYS = 196608;      // per-query key bitmaps of a group in shared memory (192 KB)
constexpr int LA_CHUNK = 16384;          // query rows per pass (a multiple of the grouping window)
constexpr long long LA_WAIT_BUDGET = 4000000000ll;

__device__ __forceinline__ int la_round_chunk(int n) { return (n + kUnionChunk - 1) / kUnionChunk * kUnionChunk; }

// ----------------------------------------------------------- local part
// Group g holds queries 8g .. 8g + 7 (positions grow with the row). Keys: the
// sinks of its last query, then the window range from the first query's
// window start to the last query's position; a key's mask has bit qi when it is
// one of query qi's sinks or lies in its window.
__global__ void __launch_bounds__(256)
    lsa_local_union_kernel(int n_q, int q_pos0, int n_sink, int n_window, int cap, int* __restrict__ list,
                           uint8_t* __restrict__ lmask, int* __restrict__ n_list) {
  const int g = blockIdx.x;
  const int t0 = g * LA_GA, t1 = min(n_q, t0 + LA_GA) - 1;
  const int p0 = q_pos0 + t0, p1 = q_pos0 + t1;
  const int ns = min(n_sink, p1 + 1);
  const int lo = max(n_sink, p0 - n_window + 1);
  const int nw = max(0, p1 - lo + 1);
  const int total = min(ns + nw, cap);
  int* gl = list + (long long)g * cap;
  uint8_t* gm = lmask + (long long)g * cap;
  for (int e = threadIdx.x; e < la_round_chunk(total); e += 256) {
    if (e < total) {
      const int s = e < ns ? e : lo + (e - ns);
      uint32_t m = 0u;
      for (int qi = 0; qi <= t1 - t0; ++qi) {
        const int p = p0 + qi;
        const int wl = max(n_sink, p - n_window + 1);
        if (s < min(n_sink, p + 1) || (s >= wl && s <= p)) m |= 1u << qi;
      }
      gl[e] = s;
      gm[e] = (uint8_t)m;
    } else {
      gl[e] = -1;
      gm[e] = 0;
    }
  }
  if (threadIdx.x == 0) n_list[g] = total;
}

// ------------------------------------------------------------- far part
// The long-range keys of row t: the entries of J after its sinks and window,
// up to the first -1.
__device__ __forceinline__ int la_head(int pos, int n_sink, int n_window) {
  const int ns = max(0, min(n_sink, pos + 1));
  const int wl = max(n_sink, pos - n_window + 1);
  return ns + max(0, pos - wl + 1);
}

__device__ __forceinline__ uint32_t la_hash(uint32_t s) {
  uint32_t x = s * 0x9E3779B1u;
  x ^= x >> 15;
  x *= 0x2C1B3C6Du;
  x ^= x >> 12;
  return x;
}

// sig[t] = (smallest hash over row t's long-range keys) << 32 | t; rows with
// none sort last. One warp per row.
__global__ void __launch_bounds__(256)
    lsa_far_sig_kernel(const int32_t* __restrict__ J, int width, int n_q, int q_pos0, int n_sink, int n_window,
                       unsigned long long* __restrict__ sig) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= n_q) return;
  const int32_t* row = J + (long long)t * width;
  uint32_t h = 0xFFFFFFFFu;
  for (int j = la_head(q_pos0 + t, n_sink, n_window) + lane; j < width; j += 32) {
    const int s = row[j];
    if (s >= 0) h = min(h, la_hash((uint32_t)s));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) h = min(h, __shfl_xor_sync(0xffffffffu, h, o));
  if (lane == 0) sig[t] = ((unsigned long long)h << 32) | (uint32_t)t;
}

// Union of the long-range keys of group g (queries perm[8g .. 8g + 7]): one
// bitmap of n_k bits per query in shared memory, then the keys of the OR in
// ascending order with one mask bit per query, padded to whole 128-key chunks.
__global__ void __launch_bounds__(TK_THREADS)
    lsa_far_union_kernel(const int32_t* __restrict__ J, int width, const int* __restrict__ perm, int n_q,
                         int q_pos0, int n_sink, int n_window, int n_k, int cap, int* __restrict__ list,
                         uint8_t* __restrict__ lmask, int* __restrict__ n_list) {
  extern __shared__ uint32_t la_bm[];               // [8][nwords]
  __shared__ int red[TK_THREADS / 32];
  const int g = blockIdx.x, tid = threadIdx.x;
  const int nwords = (n_k + 31) >> 5;
  for (int i = tid; i < LA_GA * nwords; i += TK_THREADS) la_bm[i] = 0u;
  __syncthreads();
  for (int qi = 0; qi < LA_GA; ++qi) {
    const int t = perm[g * LA_GA + qi];
    if (t < 0 || t >= n_q) continue;
    const int32_t* row = J + (long long)t * width;
    for (int j = la_head(q_pos0 + t, n_sink, n_window) + tid; j < width; j += TK_THREADS) {
      const int s = row[j];
      if (s >= 0 && s < n_k) atomicOr(&la_bm[qi * nwords + (s >> 5)], 1u << (s & 31));
    }
  }
  __syncthreads();
  const int per = (nwords + TK_THREADS - 1) / TK_THREADS;
  const int w0 = min(nwords, tid * per), w1 = min(nwords, w0 + per);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) {
    uint32_t u = 0u;
#pragma unroll
    for (int qi = 0; qi < LA_GA; ++qi) u |= la_bm[qi * nwords + w];
    cnt += __popc(u);
  }
  int tot;
  int o = block_excl_scan(cnt, red, &tot);
  if (tid == 0) SA_DBG_CHECK(tot <= cap, SA_DBG_LSA_FAR_UNION, tot);
  const int total = min(tot, cap);
  int* gl = list + (long long)g * cap;
  uint8_t* gm = lmask + (long long)g * cap;
  for (int w = w0; w < w1; ++w) {
    uint32_t word[LA_GA];
    uint32_t u = 0u;
#pragma unroll
    for (int qi = 0; qi < LA_GA; ++qi) {
      word[qi] = la_bm[qi * nwords + w];
      u |= word[qi];
    }
    while (u != 0u) {
      const int b = __ffs(u) - 1;
      u &= u - 1u;
      uint32_t m = 0u;
#pragma unroll
      for (int qi = 0; qi < LA_GA; ++qi) m |= ((word[qi] >> b) & 1u) << qi;
      if (o < cap) {
        gl[o] = w * 32 + b;
        gm[o] = (uint8_t)m;
      }
      ++o;
    }
  }
  for (int i = total + tid; i < la_round_chunk(total); i += TK_THREADS) {
    gl[i] = -1;
    gm[i] = 0;
  }
  if (tid == 0) n_list[g] = total;
}

// ---------------------------------------------------------------- merge
// One warp per (query, head) row of head_dim values.
__global__ void __launch_bounds__(256)
    lsa_merge_kernel(const __nv_bfloat16* __restrict__ oa, const float* __restrict__ la,
                     const __nv_bfloat16* __restrict__ ob, const float* __restrict__ lb, long long rows, int dh,
                     __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const float a = la[r], b = lb[r];
  const float m = fmaxf(a, b);
  float wa = 0.f, wb = 0.f;
  if (m != -INFINITY) {
    wa = a == -INFINITY ? 0.f : expf(a - m);
    wb = b == -INFINITY ? 0.f : expf(b - m);
  }
  const float inv = (wa + wb) > 0.f ? 1.f / (wa + wb) : 0.f;
  for (int i = lane; i < dh; i += 32) {
    const float v = (wa * __bfloat162float(oa[r * dh + i]) + wb * __bfloat162float(ob[r * dh + i])) * inv;
    out[r * dh + i] = __float2bfloat16_rn(v);
  }
  if (lane == 0 && lse != nullptr) lse[r] = (wa + wb) > 0.f ? m + logf(wa + wb) : -INFINITY;
}

// ------------------------------------------------------------------ plan
struct LaPlan {
  int R, groups, cap_l, cap_f, wperm;
  size_t off_ll, off_ml, off_nl, off_sig, off_perm, off_lf, off_mf, off_nf, off_ol, off_sl, off_of, off_sf, total;
};

static size_t la_up(size_t x) { return (x + 255) & ~size_t(255); }

static int ceil_to(int x, int m) { return (x + m - 1) / m * m; }

static LaPlan la_plan(const sa_attn_in* at, int width, int n_sink, int n_window) {
  LaPlan p{};
  const int W = group_window();
  p.R = ceil_to(max(1, min(at->n_q, LA_CHUNK)), W);
  p.groups = p.R / LA_GA;
  p.wperm = p.R;
  p.cap_l = ceil_to(n_sink + n_window + LA_GA, kUnionChunk);
  p.cap_f = ceil_to(LA_GA * max(1, width - n_sink - n_window), kUnionChunk);
  const size_t rowsz = (size_t)p.R * at->n_q_heads;
  size_t off = 0;
  p.off_ll = off;
  off = la_up(off + (size_t)p.groups * p.cap_l * 4);
  p.off_ml = off;
  off = la_up(off + (size_t)p.groups * p.cap_l);
  p.off_nl = off;
  off = la_up(off + (size_t)p.groups * 4);
  p.off_sig = off;
  off = la_up(off + (size_t)p.R * 8);
  p.off_perm = off;
  off = la_up(off + (size_t)p.wperm * 4);
  p.off_lf = off;
  off = la_up(off + (size_t)p.groups * p.cap_f * 4);
  p.off_mf = off;
  off = la_up(off + (size_t)p.groups * p.cap_f);
  p.off_nf = off;
  off = la_up(off + (size_t)p.groups * 4);
  p.off_ol = off;
  off = la_up(off + rowsz * at->head_dim * 2);
  p.off_sl = off;
  off = la_up(off + rowsz * 4);
  p.off_of = off;
  off = la_up(off + rowsz * at->head_dim * 2);
  p.off_sf = off;
  off = la_up(off + rowsz * 4);
  p.total = off;
  return p;
}

static sa_status la_check(const sa_attn_in* at, int width, int q_pos0, int n_sink, int n_window) {
  if (at == nullptr || at->batch != 0 || at->n_q < 0 || at->n_k <= 0) return SA_ERR_INVALID_ARGUMENT;
  if (width < 1 || q_pos0 < 0 || n_sink < 0 || n_window < 0 || n_sink + (long long)n_window > width)
    return SA_ERR_INVALID_ARGUMENT;
  if (q_pos0 + (long long)at->n_q > at->n_k) return SA_ERR_INVALID_ARGUMENT;   // every query's own key is cached
  if (!tc_attention_supported(at->n_q_heads, at->head_dim) || at->n_k > LA_MAX_KEYS) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

}  // namespace sa

using namespace sa;

extern "C" sa_status sa_lsa_attention_workspace_size(const sa_attn_in* attn, int32_t width, int32_t q_pos0,
                                                     int32_t n_sink, int32_t n_window, size_t* bytes) {
  if (bytes == nullptr) return SA_ERR_INVALID_ARGUMENT;
  const sa_status s = la_check(attn, width, q_pos0, n_sink, n_window);
  if (s != SA_OK) return s;
  *bytes = attn->n_q == 0 ? 0 : la_plan(attn, width, n_sink, n_window).total;
  return SA_OK;
}

extern "C" sa_status sa_lsa_attention(const sa_attn_in* attn, const int32_t* J, int32_t width, int32_t q_pos0,
                                      int32_t n_sink, int32_t n_window, void* out, float* lse,
                                      sa_device_status* status, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const sa_status s = la_check(attn, width, q_pos0, n_sink, n_window);
  if (s != SA_OK) return s;
  const LaPlan pl = la_plan(attn, width, n_sink, n_window);
  if (attn->n_q > 0) {
    if (J == nullptr || out == nullptr || attn->q == nullptr || attn->k_cache == nullptr ||
        attn->v_cache == nullptr || ws == nullptr)
      return SA_ERR_INVALID_ARGUMENT;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return SA_ERR_INVALID_ARGUMENT;
    if (ws_bytes < pl.total) return SA_ERR_WORKSPACE_TOO_SMALL;
  }
  if (status != nullptr && cudaMemsetAsync(status, 0, sizeof(sa_device_status), stream) != cudaSuccess)
    return SA_ERR_CUDA;
  if (attn->n_q == 0) return SA_OK;
  uint8_t* w = static_cast<uint8_t*>(ws);
  int* list_l = reinterpret_cast<int*>(w + pl.off_ll);
  uint8_t* mask_l = w + pl.off_ml;
  int* nl_l = reinterpret_cast<int*>(w + pl.off_nl);
  unsigned long long* sig = reinterpret_cast<unsigned long long*>(w + pl.off_sig);
  int* perm = reinterpret_cast<int*>(w + pl.off_perm);
  int* list_f = reinterpret_cast<int*>(w + pl.off_lf);
  uint8_t* mask_f = w + pl.off_mf;
  int* nl_f = reinterpret_cast<int*>(w + pl.off_nf);
  __nv_bfloat16* o_l = reinterpret_cast<__nv_bfloat16*>(w + pl.off_ol);
  float* s_l = reinterpret_cast<float*>(w + pl.off_sl);
  __nv_bfloat16* o_f = reinterpret_cast<__nv_bfloat16*>(w + pl.off_of);
  float* s_f = reinterpret_cast<float*>(w + pl.off_sf);
  const int hq = attn->n_q_heads, dh = attn->head_dim;
  const float scale = attn->softmax_scale > 0.f ? attn->softmax_scale : 1.f / sqrtf((float)dh);
  uint32_t* st = reinterpret_cast<uint32_t*>(status);
  const int nwords = (attn->n_k + 31) / 32;
  const int bm_smem = LA_GA * nwords * 4;
  if (cudaFuncSetAttribute(lsa_far_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bm_smem) !=
      cudaSuccess)
    return SA_ERR_CUDA;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(attn->q);
  for (int r0 = 0; r0 < attn->n_q; r0 += pl.R) {
    const int rows = min(pl.R, attn->n_q - r0), pos0 = q_pos0 + r0;
    const int groups = (rows + LA_GA - 1) / LA_GA;
    const int32_t* Jc = J + (long long)r0 * width;
    const __nv_bfloat16* qc = q + (long long)r0 * hq * dh;
    // local: consecutive groups over sinks and windows
    lsa_local_union_kernel<<<groups, 256, 0, stream>>>(rows, pos0, n_sink, n_window, pl.cap_l, list_l, mask_l, nl_l);
    cudaError_t e = launch_attention_tc(qc, attn->k_cache, attn->v_cache, list_l, mask_l, nl_l, nullptr, groups, rows,
                                        pl.cap_l, scale, o_l, s_l, st, LA_WAIT_BUDGET, stream);
    if (e != cudaSuccess) return SA_ERR_CUDA;
    // far: signature groups over the long-range keys
    lsa_far_sig_kernel<<<(rows + 7) / 8, 256, 0, stream>>>(Jc, width, rows, pos0, n_sink, n_window, sig);
    if (launch_group_sort(sig, rows, perm, stream) != cudaSuccess) return SA_ERR_CUDA;
    const int fgroups = ceil_to(rows, group_window()) / LA_GA;
    lsa_far_union_kernel<<<fgroups, TK_THREADS, bm_smem, stream>>>(Jc, width, perm, rows, pos0, n_sink, n_window,
                                                                   attn->n_k, pl.cap_f, list_f, mask_f, nl_f);
    e = launch_attention_tc(qc, attn->k_cache, attn->v_cache, list_f, mask_f, nl_f, perm, fgroups, rows, pl.cap_f,
                            scale, o_f, s_f, st, LA_WAIT_BUDGET, stream);
    if (e != cudaSuccess) return SA_ERR_CUDA;
    // merge the two softmax parts
    const long long mrows = (long long)rows * hq;
    lsa_merge_kernel<<<(unsigned)((mrows + 7) / 8), 256, 0, stream>>>(
        o_l, s_l, o_f, s_f, mrows, dh, static_cast<__nv_bfloat16*>(out) + (long long)r0 * hq * dh,
        lse == nullptr ? nullptr : lse + (long long)r0 * hq);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  }
  return SA_OK;
}

namespace sa {
SA_DEBUG_UNIT(dbg_read_lsa_attn)
}  // namespace sa
