// group.cu -- attention over the keys a group of queries selected together.
//
// The plain prefill attention (attn.cu) gathers every query's selected K/V
// rows on its own: at 2048 keys of 512 bytes per query that is 1 MiB of
// scattered reads per query, and the kernel runs at the L2 gather rate.
// Queries that attend to nearly the same keys can share those reads. In the
// two-stage method the queries that keep the same key blocks (HISA section 3)
// select mostly the same keys; the grouping kernel below sorts every window
// of GW consecutive queries by three MinHashes of its kept-block set
// (lexicographically), so runs of GA queries in that order tend to keep the
// same blocks. The grouped kernel then
// takes GA queries per CTA (one warp each), forms the union of their index
// sets with a per-key mask of the queries that chose the key, gathers each
// union key once into a ring shared by the CTA, and lets every warp attend
// over the union with its own mask. Each query still attends exactly to its
// own index set (softmax does not depend on the order of the keys, Latent
// Sparse Attention section 3.2); the grouping only changes the schedule.
//
// A group whose union does not fit the CTA's tables (more than GU_MAX key
// blocks of 64, more than GL_MAX keys, or n_k above GK_MAX) is processed one
// query at a time instead, with the query's keys split over the warps and the
// warp states merged, which is the plain kernel's schedule.
#include <cuda_bf16.h>

#include "attn_common.cuh"
#include "debug.cuh"
#include "ptx.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int GW = 2048;             // queries per grouping window
static_assert(GW == 2048, "the sort key holds a query's index in its window in 11 bits");
constexpr int GA = kGroupQueries;    // queries per attention group (one warp each)
constexpr int GT = GA * 32;          // threads per grouped CTA
constexpr int GCH = 64;              // keys per ring stage
constexpr int GST = 3;               // ring stages
constexpr int GU_MAX = 512;          // union blocks of 64 keys
constexpr int GL_MAX = 16384;        // union keys
constexpr int GK_MAX = 1 << 20;      // keys per cache covered by the block bitmap
constexpr int GK_WORDS = GK_MAX / 2048;

// ---------------------------------------------------------------- grouping
static __device__ __forceinline__ uint32_t block_hash(uint32_t b) {
  uint32_t x = b * 0x9E3779B1u;
  x ^= x >> 15;
  x *= 0x2C1B3C6Du;
  x ^= x >> 12;
  return x;
}

// The signature of query t: the smallest hash over its kept blocks under
// three hash functions, leaving out block 0 and the query's own block, which
// every query keeps (HISA section 3: the first and the local block are always
// in). Two queries agree on one MinHash with probability equal to the Jaccard
// similarity of their block sets; sorting by the first, then the second, then
// the third keeps a run of equal first hashes ordered by how much more its
// members share, so fewer groups straddle two runs (on the 64K two-stage
// workload an 8-query group's union of kept blocks is 1.08 x its queries' mean
// kept count, against 1.32 with one MinHash). With `sel` (the top-k's
// selection bitmaps over the kept blocks' keys) only the blocks holding at
// least min_sel selected keys count: the blocks a query draws most of its keys
// from mark its neighbourhood better than the blocks it kept at the margin.
// The sort key packs the three minima (17, 18 and 18 high bits) above the
// query's index in its window (11 bits); the first field stops at 0x1FFFE so
// no key equals the empty slot's all-ones. One warp per query: lane j reads
// kept slots j and j + 32.
__global__ void __launch_bounds__(256) group_signature_kernel(const int* __restrict__ kept, int keep,
                                                              const uint32_t* __restrict__ sel, int min_sel, int n_q,
                                                              int q_pos0, int block,
                                                              unsigned long long* __restrict__ sig) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= n_q) return;
  const int cur = (q_pos0 + t) / block;
  uint32_t h1 = 0xFFFFFFFFu, h2 = 0xFFFFFFFFu, h3 = 0xFFFFFFFFu;
  for (int j = lane; j < keep; j += 32) {
    const int b = kept[(long long)t * keep + j];
    bool use = b >= 0 && b != 0 && b != cur;
    if (use && sel != nullptr) {
      const uint32_t* sr = sel + (long long)t * keep * 2;
      use = __popc(sr[2 * j]) + __popc(sr[2 * j + 1]) >= min_sel;
    }
    if (use) {
      h1 = min(h1, block_hash(3u * (uint32_t)b));
      h2 = min(h2, block_hash(3u * (uint32_t)b + 1u));
      h3 = min(h3, block_hash(3u * (uint32_t)b + 2u));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    h1 = min(h1, __shfl_xor_sync(0xffffffffu, h1, o));
    h2 = min(h2, __shfl_xor_sync(0xffffffffu, h2, o));
    h3 = min(h3, __shfl_xor_sync(0xffffffffu, h3, o));
  }
  if (lane == 0)
    sig[t] = ((unsigned long long)min(h1 >> 15, 0x1FFFEu) << 47) | ((unsigned long long)(h2 >> 14) << 29) |
             ((unsigned long long)(h3 >> 14) << 11) | (unsigned long long)(t & (GW - 1));
}

// perm[w * GW + i] = the query at rank i of window w in (signature, query)
// order, -1 past n_q. A key's low 11 bits are its query's index in the window
// (the keys of the two-stage grouping above, and (hash << 32 | t) keys, whose
// t has those bits).
__global__ void __launch_bounds__(1024) group_sort_kernel(const unsigned long long* __restrict__ sig, int n_q,
                                                          int* __restrict__ perm) {
  __shared__ unsigned long long key[GW];
  const int w0 = blockIdx.x * GW;
  for (int i = threadIdx.x; i < GW; i += 1024) key[i] = (w0 + i < n_q) ? sig[w0 + i] : ~0ull;
  __syncthreads();
  // bitonic sort, ascending
  for (int size = 2; size <= GW; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < GW / 2; i += 1024) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const unsigned long long a = key[lo], b = key[hi];
        if ((a > b) == up) {
          key[lo] = b;
          key[hi] = a;
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < GW; i += 1024) {
    const unsigned long long k = key[i];
    perm[w0 + i] = (k == ~0ull) ? -1 : w0 + (int)(k & (unsigned long long)(GW - 1));
  }
}

int group_perm_len(int n_q) { return (n_q + GW - 1) / GW * GW; }

cudaError_t launch_group_queries(const int* kept, int keep, const uint32_t* sel, int min_sel, int n_q, int q_pos0,
                                 int block, unsigned long long* sig, int* perm, cudaStream_t st) {
  if (n_q <= 0) return cudaSuccess;
  if (keep <= 0 || block <= 0) return cudaErrorInvalidValue;
  group_signature_kernel<<<(n_q + 7) / 8, 256, 0, st>>>(kept, keep, sel, min_sel, n_q, q_pos0, block, sig);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  group_sort_kernel<<<(n_q + GW - 1) / GW, 1024, 0, st>>>(sig, n_q, perm);
  return cudaGetLastError();
}

cudaError_t launch_group_sort(const unsigned long long* sig, int n_q, int* perm, cudaStream_t st) {
  if (n_q <= 0) return cudaSuccess;
  group_sort_kernel<<<(n_q + GW - 1) / GW, 1024, 0, st>>>(sig, n_q, perm);
  return cudaGetLastError();
}

int group_window() { return GW; }

// ------------------------------------------------------- grouped attention
template <int DH>
struct GaCfg {
  static constexpr int ROWB = DH * 2;
  static constexpr int SEGS = ROWB / 16;
  static constexpr int STAGE_BYTES = 2 * GCH * ROWB;                 // K rows, then V rows
  static constexpr int RING = GST * STAGE_BYTES;
  static constexpr int MERGE_BYTES = GA * (16 * DH + 32) * 4;
  // the union build borrows the ring for the per-key masks and the bitmap
  static constexpr int MASK_BYTES = GU_MAX * 64;
  static constexpr int BUILD_BYTES = MASK_BYTES + 2 * GK_WORDS * 4;
  static_assert(RING >= MERGE_BYTES && RING >= BUILD_BYTES, "ring too small for its other uses");
  static constexpr int OFF_LIST = RING;
  static constexpr int OFF_LMASK = OFF_LIST + GL_MAX * 4;
  static constexpr int OFF_UB = OFF_LMASK + GL_MAX;
  static constexpr int OFF_MISC = OFF_UB + GU_MAX * 4;
  static constexpr int SMEM = OFF_MISC + 64 * 4;
};

template <int HQ, int DH>
__global__ void __launch_bounds__(GT, 1)
    grouped_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                        const __nv_bfloat16* __restrict__ vc, const int32_t* __restrict__ idx,
                        const int* __restrict__ perm, int n_q, int k, int n_k, float scale_log2,
                        __nv_bfloat16* __restrict__ out, float* __restrict__ lse, bool ungrouped) {
  using C = GaCfg<DH>;
  using W = AttnWarp<HQ, DH, 1>;
  extern __shared__ __align__(128) uint8_t ga_smem[];
  uint32_t* maskw = reinterpret_cast<uint32_t*>(ga_smem);                       // [GU_MAX * 16]  (build only)
  uint32_t* bits = reinterpret_cast<uint32_t*>(ga_smem + C::MASK_BYTES);       // [GK_WORDS]     (build only)
  int* wpre = reinterpret_cast<int*>(ga_smem + C::MASK_BYTES + GK_WORDS * 4);  // [GK_WORDS]     (build only)
  int* list = reinterpret_cast<int*>(ga_smem + C::OFF_LIST);                   // union keys, ascending
  uint8_t* lmask = ga_smem + C::OFF_LMASK;                                      // their query masks
  int* ub2blk = reinterpret_cast<int*>(ga_smem + C::OFF_UB);                   // union block -> block
  int* misc = reinterpret_cast<int*>(ga_smem + C::OFF_MISC);
  int* qt = misc;                  // [GA] the group's queries (-1: none)
  int* red = misc + GA;            // [GA] scan partials
  int& n_ub = misc[2 * GA];
  int& n_list = misc[2 * GA + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid < GA) {
    const int j = blockIdx.x * GA + tid;
    const int t = perm ? perm[j] : j;
    qt[tid] = (t >= 0 && t < n_q) ? t : -1;
  }
  __syncthreads();
  bool any = false;
#pragma unroll
  for (int w = 0; w < GA; ++w) any |= qt[w] >= 0;
  if (!any) return;

  // ---- union of the group's index sets ----
  bool grouped = n_k <= GK_MAX && !ungrouped;
  const int nwords = (n_k + 2047) / 2048;
  // the group's index rows, staged in the list area (which the union
  // overwrites only after its last read of them) when they fit; a row read
  // from global memory entry by entry would leave every thread waiting on
  // one dependent load per entry
  const bool staged = (long long)GA * k <= GL_MAX;
  auto row_at = [&](int qi, int j) -> int {
    return staged ? list[qi * k + j] : idx[(long long)qt[qi] * k + j];
  };
  if (grouped) {
    if (staged) {
      const bool vec = (k & 3) == 0 && (reinterpret_cast<uintptr_t>(idx) & 15u) == 0;
      for (int qi = 0; qi < GA; ++qi) {
        const int t = qt[qi];
        int* dst = list + qi * k;
        if (t >= 0 && vec) {
          const int32_t* row = idx + (long long)t * k;
          for (int j = tid * 4; j < k; j += GT * 4) cp_async16(smem_u32(dst + j), row + j);
        } else {
          for (int j = tid; j < k; j += GT) dst[j] = t >= 0 ? idx[(long long)t * k + j] : -1;
        }
      }
      cp_async_commit();
      cp_async_wait<0>();
    }
    for (int i = tid; i < nwords; i += GT) bits[i] = 0u;
    __syncthreads();
    // pass 1: which 64-key blocks hold a selected key
    for (int qi = 0; qi < GA; ++qi) {
      if (qt[qi] < 0) continue;
      for (int j = tid; j < k; j += GT) {
        const int s = row_at(qi, j);
        if (s >= 0 && s < n_k) atomicOr(&bits[s >> 11], 1u << ((s >> 6) & 31));
      }
    }
    __syncthreads();
    // union block numbering in ascending block order
    if (warp == 0) {
      const int per = (nwords + 31) / 32;
      const int lo = min(nwords, lane * per), hi = min(nwords, lo + per);
      int cnt = 0;
      for (int i = lo; i < hi; ++i) cnt += __popc(bits[i]);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int p = incl - cnt;
      for (int i = lo; i < hi; ++i) {
        wpre[i] = p;
        uint32_t b = bits[i];
        while (b) {
          const int bit = __ffs(b) - 1;
          b &= b - 1;
          if (p < GU_MAX) ub2blk[p] = i * 32 + bit;
          ++p;
        }
      }
      if (lane == 31) n_ub = incl;
    }
    __syncthreads();
    grouped = n_ub <= GU_MAX;
  }
  if (grouped) {
    for (int i = tid; i < n_ub * 16; i += GT) maskw[i] = 0u;
    __syncthreads();
    // pass 2: per-key masks of the queries that selected the key
    for (int qi = 0; qi < GA; ++qi) {
      if (qt[qi] < 0) continue;
      for (int j = tid; j < k; j += GT) {
        const int s = row_at(qi, j);
        if (s < 0 || s >= n_k) continue;
        const int wi = s >> 11, b = (s >> 6) & 31;
        const int ub = wpre[wi] + __popc(bits[wi] & ((1u << b) - 1u));
        const int slot = ub * 64 + (s & 63);
        atomicOr(&maskw[slot >> 2], (1u << qi) << (8 * (slot & 3)));
      }
    }
    __syncthreads();
    // ordered compaction of the selected union keys
    const int n_slot = n_ub * 64;
    const int per = (n_slot + GT - 1) / GT;
    const int lo = min(n_slot, tid * per), hi = min(n_slot, lo + per);
    const uint8_t* mb = reinterpret_cast<const uint8_t*>(maskw);
    int cnt = 0;
    for (int i = lo; i < hi; ++i) cnt += mb[i] != 0;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < GA; ++w) {
      before += (w < warp) ? red[w] : 0;
      total += red[w];
    }
    if (total <= GL_MAX) {
      int p = before + incl - cnt;
      for (int i = lo; i < hi; ++i) {
        const uint8_t m = mb[i];
        if (m) {
          list[p] = ub2blk[i >> 6] * 64 + (i & 63);
          lmask[p] = m;
          ++p;
        }
      }
      for (int i = total + tid; i < (total + GCH - 1) / GCH * GCH; i += GT) {
        list[i] = -1;
        lmask[i] = 0;
      }
    }
    grouped = total <= GL_MAX;
    if (tid == 0) n_list = total;
    __syncthreads();   // the masks (in the ring) are consumed; the list is complete
  }

  // ---- the ring loop over a key list ----
  // grouped: every warp takes the 16-key chunks holding one of its keys;
  // single: the chunks go round-robin over the warps, every listed key valid
  constexpr int SEGS = C::SEGS;
  constexpr int RPP = GT / SEGS;        // rows per loader pass
  auto issue = [&](int stage, int slot) {
    const uint32_t kdst = smem_u32(ga_smem + slot * C::STAGE_BYTES);
    const uint32_t vdst = kdst + GCH * C::ROWB;
    const int seg = tid % SEGS;
#pragma unroll
    for (int i = 0; i < GCH / RPP; ++i) {
      const int r = i * RPP + tid / SEGS;
      const int s = list[stage * GCH + r];
      const long long off = (long long)(s >= 0 ? s : 0) * DH + seg * 8;
      cp_async16(kdst + W::off(r, seg), kc + off);
      cp_async16(vdst + W::off(r, seg), vc + off);
    }
  };
  uint32_t qa[W::KK][4];
  float o[W::NT][4], m_r[2], l_r[2];
  auto run = [&](int n_ent, bool by_mask) {
    const int n_st = (n_ent + GCH - 1) / GCH;
#pragma unroll
    for (int i = 0; i < GST - 1; ++i) {
      if (i < n_st) issue(i, i);
      cp_async_commit();
    }
    for (int i = 0; i < n_st; ++i) {
      cp_async_wait<GST - 2>();
      __syncthreads();
      if (i + GST - 1 < n_st) issue(i + GST - 1, (i + GST - 1) % GST);
      cp_async_commit();
      const uint32_t base = smem_u32(ga_smem + (i % GST) * C::STAGE_BYTES);
#pragma unroll
      for (int sub = 0; sub < GCH / AT_CHUNK; ++sub) {
        const int c = i * (GCH / AT_CHUNK) + sub;
        if (c * AT_CHUNK >= n_ent) break;
        const int e = c * AT_CHUNK + (lane & (AT_CHUNK - 1));
        uint32_t valid;
        if (by_mask) {
          valid = __ballot_sync(0xffffffffu, lane < AT_CHUNK && ((lmask[e] >> warp) & 1u));
        } else {
          if (c % GA != warp) continue;
          valid = __ballot_sync(0xffffffffu, lane < AT_CHUNK && list[e] >= 0);
        }
        if (valid == 0u) continue;
        W::step(qa, base + sub * AT_CHUNK * C::ROWB, base + GCH * C::ROWB + sub * AT_CHUNK * C::ROWB, valid, lane,
                scale_log2, o, m_r, l_r);
      }
    }
    cp_async_wait<0>();
    __syncthreads();
  };

  if (grouped) {
    const int t = qt[warp];
    W::load_q(q, t, lane, qa);
    W::init(o, m_r, l_r);
    run(n_list, true);
    W::reduce_l(l_r);
    if (t >= 0) W::store(out + (long long)t * HQ * DH, lse ? lse + (long long)t * HQ : nullptr, lane, o, m_r, l_r);
    return;
  }

  // one query at a time, its keys split over the warps
  for (int qi = 0; qi < GA; ++qi) {
    const int t = qt[qi];
    if (t < 0) continue;
    W::load_q(q, t, lane, qa);
    W::init(o, m_r, l_r);
    const int32_t* row = idx + (long long)t * k;
    for (int j0 = 0; j0 < k; j0 += GL_MAX) {
      const int n = min(GL_MAX, k - j0);
      for (int j = tid; j < (n + GCH - 1) / GCH * GCH; j += GT) {
        const int s = j < n ? row[j0 + j] : -1;
        list[j] = (s >= 0 && s < n_k) ? s : -1;
      }
      __syncthreads();
      run(n, false);
    }
    W::reduce_l(l_r);
    float* slots = reinterpret_cast<float*>(ga_smem);
    W::to_slot(slots + warp * (16 * DH + 32), lane, o, m_r, l_r);
    __syncthreads();
    for (int e = tid; e < HQ * DH; e += GT) {
      const int h = e / DH, col = e % DH;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < GA; ++w) M = fmaxf(M, slots[w * (16 * DH + 32) + 16 * DH + h]);
      const float Ms = (M == -INFINITY) ? 0.f : M;
      float L = 0.f, acc = 0.f;
#pragma unroll
      for (int w = 0; w < GA; ++w) {
        const float* bw = slots + w * (16 * DH + 32);
        const float f = exp2f(bw[16 * DH + h] - Ms);
        L += bw[16 * DH + 16 + h] * f;
        acc += bw[h * DH + col] * f;
      }
      out[((long long)t * HQ + h) * DH + col] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
      if (lse != nullptr && col == 0)
        lse[(long long)t * HQ + h] = L > 0.f ? (Ms + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
    __syncthreads();
  }
}

template <int HQ, int DH>
static cudaError_t launch_grouped_t(const void* q, const void* kc, const void* vc, const int32_t* idx,
                                   const int* perm, int n_groups, int n_q, int k, int n_k, float scale, void* out,
                                   float* lse, bool ungrouped, cudaStream_t st) {
  using C = GaCfg<DH>;
  auto kern = grouped_attn_kernel<HQ, DH>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<n_groups, GT, C::SMEM, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)kc, (const __nv_bfloat16*)vc,
                                      idx, perm, n_q, k, n_k, scale * 1.4426950408889634f, (__nv_bfloat16*)out, lse,
                                      ungrouped);
  return cudaGetLastError();
}

cudaError_t launch_attention_grouped(const void* q, const void* kc, const void* vc, const int32_t* idx,
                                     const int* perm, int n_perm, int n_q, int k, int n_k, int hq, int dh,
                                     float scale, void* out, float* lse, bool ungrouped, cudaStream_t st) {
  if (n_q <= 0) return cudaSuccess;
  const int n_groups = ((perm ? n_perm : n_q) + GA - 1) / GA;
  if (hq == 16 && dh == 128)
    return launch_grouped_t<16, 128>(q, kc, vc, idx, perm, n_groups, n_q, k, n_k, scale, out, lse, ungrouped, st);
  if (hq == 8 && dh == 128)
    return launch_grouped_t<8, 128>(q, kc, vc, idx, perm, n_groups, n_q, k, n_k, scale, out, lse, ungrouped, st);
  if (hq == 16 && dh == 64)
    return launch_grouped_t<16, 64>(q, kc, vc, idx, perm, n_groups, n_q, k, n_k, scale, out, lse, ungrouped, st);
  if (hq == 8 && dh == 64)
    return launch_grouped_t<8, 64>(q, kc, vc, idx, perm, n_groups, n_q, k, n_k, scale, out, lse, ungrouped, st);
  return cudaErrorNotSupported;
}

}  // namespace sa

namespace sa {

// ------------------------------------------------------ union of a group
// Two-stage rows: a query's selected keys are the set bits of its selection
// bitmap over its kept blocks' candidates (column c = 64 * slot + offset).
// The union of the group is built block-wise: the group's kept blocks in
// ascending order (a bitmap over all blocks, ranked by popcount), a table of
// each query's slot of every union block, then one mask byte per union key
// (8 keys at a time by an 8 x 8 bit transpose), compacted in key order.
int group_union_cap(int k) { return (GA * k + kUnionChunk - 1) / kUnionChunk * kUnionChunk; }

__global__ void __launch_bounds__(256) group_union_kernel(const int* __restrict__ kept, int keep,
                                                          const uint32_t* __restrict__ sel, const int* __restrict__ perm,
                                                          int n_q, int n_k, int cap, int* __restrict__ list,
                                                          uint8_t* __restrict__ lmask, int* __restrict__ n_list) {
  constexpr int KB = 64;                         // kept blocks per query (at most)
  __shared__ int qt[GA];
  __shared__ int kb[GA][KB];
  __shared__ uint32_t sw[GA][2 * KB];
  __shared__ uint32_t bits[GK_WORDS];
  __shared__ int wpre[GK_WORDS];
  __shared__ signed char slot[GA][GA * KB];
  __shared__ int ub2blk[GA * KB];
  __shared__ int red[8];
  __shared__ int s_nub;
  extern __shared__ __align__(8) uint8_t ga_union_smem[];   // [GA * KB * 64] per-key query masks
  const int g = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid < GA) {
    const int j = g * GA + tid;
    const int t = perm ? perm[j] : j;
    qt[tid] = (t >= 0 && t < n_q) ? t : -1;
  }
  const int nwords = ((n_k + 63) / 64 + 31) / 32;
  for (int i = tid; i < nwords; i += 256) bits[i] = 0u;
  __syncthreads();
  const int words = 2 * keep;
  for (int i = tid; i < GA * KB; i += 256) {
    const int qi = i / KB, c = i % KB, t = qt[qi];
    kb[qi][c] = (t >= 0 && c < keep) ? kept[(long long)t * keep + c] : -1;
  }
  for (int i = tid; i < GA * 2 * KB; i += 256) {
    const int qi = i / (2 * KB), w = i % (2 * KB), t = qt[qi];
    sw[qi][w] = (t >= 0 && w < words) ? sel[(long long)t * words + w] : 0u;
  }
  __syncthreads();
  for (int i = tid; i < GA * KB; i += 256) {
    const int b = kb[i / KB][i % KB];
    if (b >= 0) atomicOr(&bits[b >> 5], 1u << (b & 31));
  }
  __syncthreads();
  if (warp == 0) {
    const int per = (nwords + 31) / 32;
    const int lo = min(nwords, lane * per), hi = min(nwords, lo + per);
    int cnt = 0;
    for (int i = lo; i < hi; ++i) cnt += __popc(bits[i]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int p = incl - cnt;
    for (int i = lo; i < hi; ++i) {
      wpre[i] = p;
      uint32_t b = bits[i];
      while (b) {
        const int bit = __ffs(b) - 1;
        b &= b - 1;
        ub2blk[p++] = i * 32 + bit;
      }
    }
    if (lane == 31) s_nub = incl;
  }
  __syncthreads();
  const int n_ub = s_nub;                         // <= GA * KB: every union block is some query's kept block
  for (int i = tid; i < GA * GA * KB; i += 256) (&slot[0][0])[i] = -1;
  __syncthreads();
  for (int i = tid; i < GA * KB; i += 256) {
    const int qi = i / KB, c = i % KB, b = kb[qi][c];
    if (b >= 0) slot[qi][wpre[b >> 5] + __popc(bits[b >> 5] & ((1u << (b & 31)) - 1u))] = (signed char)c;
  }
  __syncthreads();
  // per union key, the byte of the group's queries that selected it: for 8
  // keys of a union block, byte q of `m` holds query q's selection bits of
  // those keys; an 8 x 8 bit transpose turns it into one byte per key
  uint8_t* mb = ga_union_smem;
  for (int i = tid; i < n_ub * 8; i += 256) {
    const int u = i >> 3, b8 = (i & 7) * 8;
    unsigned long long m = 0ull;
#pragma unroll
    for (int qi = 0; qi < GA; ++qi) {
      const int sl = slot[qi][u];
      if (sl >= 0) {
        const int c = sl * 64 + b8;
        m |= (unsigned long long)((sw[qi][c >> 5] >> (c & 31)) & 0xFFu) << (8 * qi);
      }
    }
    unsigned long long t = (m ^ (m >> 7)) & 0x00AA00AA00AA00AAull;
    m ^= t ^ (t << 7);
    t = (m ^ (m >> 14)) & 0x0000CCCC0000CCCCull;
    m ^= t ^ (t << 14);
    t = (m ^ (m >> 28)) & 0x00000000F0F0F0F0ull;
    m ^= t ^ (t << 28);
    *reinterpret_cast<unsigned long long*>(mb + u * 64 + b8) = m;
  }
  __syncthreads();
  const int n_slot = n_ub * 64;
  const int per = (n_slot + 255) / 256;
  const int lo = min(n_slot, tid * per), hi = min(n_slot, lo + per);
  int cnt = 0;
  for (int e = lo; e < hi; ++e) cnt += mb[e] != 0;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) red[warp] = incl;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    before += (w < warp) ? red[w] : 0;
    total += red[w];
  }
  if (tid == 0) SA_DBG_CHECK(total <= cap, SA_DBG_GROUP_UNION, total);
  total = min(total, cap);                        // cannot bind: each query selects at most k keys
  int* gl = list + (long long)g * cap;
  uint8_t* gm = lmask + (long long)g * cap;
  int p = before + incl - cnt;
  for (int e = lo; e < hi; ++e) {
    const uint8_t m = mb[e];
    if (m != 0) {
      if (p < cap) {
        gl[p] = ub2blk[e >> 6] * 64 + (e & 63);
        gm[p] = m;
      }
      ++p;
    }
  }
  for (int i = total + tid; i < (total + kUnionChunk - 1) / kUnionChunk * kUnionChunk; i += 256) {
    gl[i] = -1;
    gm[i] = 0;
  }
  if (tid == 0) n_list[g] = total;
}

cudaError_t launch_group_union(const int* kept, int keep, const uint32_t* sel, const int* perm, int n_perm, int n_q,
                               int n_k, int cap, int* list, uint8_t* lmask, int* n_list, cudaStream_t st) {
  if (n_q <= 0) return cudaSuccess;
  if (keep <= 0 || keep > 64 || n_k > GK_MAX || cap % kUnionChunk != 0) return cudaErrorNotSupported;
  const int n_groups = ((perm ? n_perm : n_q) + GA - 1) / GA;
  constexpr int smem = GA * 64 * 64;   // one mask byte per key of up to GA * 64 union blocks
  cudaError_t e = cudaFuncSetAttribute(group_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  group_union_kernel<<<n_groups, 256, smem, st>>>(kept, keep, sel, perm, n_q, n_k, cap, list, lmask, n_list);
  return cudaGetLastError();
}

}  // namespace sa

namespace sa {

// ------------------------------------------------- union of kept blocks
// Per group: the blocks any of its queries kept, ascending, and for each the
// slot (position in the query's kept list) of every query that kept it. The
// two-stage stage 2 scores each union block once for the whole group.
int group_blocks_cap() { return GA * 64; }

__global__ void __launch_bounds__(256) group_blocks_kernel(const int* __restrict__ kept, int keep,
                                                           const int* __restrict__ perm, int n_q, int n_k,
                                                           int* __restrict__ gb_n, int* __restrict__ gb_blk,
                                                           unsigned long long* __restrict__ gb_slot) {
  constexpr int KB = 64, CAP = GA * KB;
  __shared__ int qt[GA];
  __shared__ int kb[GA][KB];
  __shared__ uint32_t bits[GK_WORDS];
  __shared__ int wpre[GK_WORDS];
  __shared__ unsigned long long slots[CAP];
  __shared__ int ub2blk[CAP];
  __shared__ int s_nub;
  const int g = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid < GA) {
    const int j = g * GA + tid;
    const int t = perm ? perm[j] : j;
    qt[tid] = (t >= 0 && t < n_q) ? t : -1;
  }
  const int nwords = ((n_k + 63) / 64 + 31) / 32;
  for (int i = tid; i < nwords; i += 256) bits[i] = 0u;
  for (int i = tid; i < CAP; i += 256) slots[i] = ~0ull;
  __syncthreads();
  for (int i = tid; i < GA * KB; i += 256) {
    const int qi = i / KB, c = i % KB, t = qt[qi];
    const int b = (t >= 0 && c < keep) ? kept[(long long)t * keep + c] : -1;
    kb[qi][c] = b;
    if (b >= 0) atomicOr(&bits[b >> 5], 1u << (b & 31));
  }
  __syncthreads();
  if (warp == 0) {
    const int per = (nwords + 31) / 32;
    const int lo = min(nwords, lane * per), hi = min(nwords, lo + per);
    int cnt = 0;
    for (int i = lo; i < hi; ++i) cnt += __popc(bits[i]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int p = incl - cnt;
    for (int i = lo; i < hi; ++i) {
      wpre[i] = p;
      uint32_t b = bits[i];
      while (b) {
        const int bit = __ffs(b) - 1;
        b &= b - 1;
        ub2blk[p++] = i * 32 + bit;
      }
    }
    if (lane == 31) s_nub = incl;
  }
  __syncthreads();
  // every query writes its own byte of each of its blocks' slot words
  uint8_t* sb = reinterpret_cast<uint8_t*>(slots);
  for (int i = tid; i < GA * KB; i += 256) {
    const int qi = i / KB, c = i % KB, b = kb[qi][c];
    if (b >= 0) sb[(wpre[b >> 5] + __popc(bits[b >> 5] & ((1u << (b & 31)) - 1u))) * 8 + qi] = (uint8_t)c;
  }
  __syncthreads();
  const int n_ub = s_nub;
  for (int u = tid; u < n_ub; u += 256) {
    gb_blk[(long long)g * CAP + u] = ub2blk[u];
    gb_slot[(long long)g * CAP + u] = slots[u];
  }
  if (tid == 0) gb_n[g] = n_ub;
}

cudaError_t launch_group_blocks(const int* kept, int keep, const int* perm, int n_perm, int n_q, int n_k, int* gb_n,
                                int* gb_blk, unsigned long long* gb_slot, cudaStream_t st) {
  if (n_q <= 0) return cudaSuccess;
  if (keep <= 0 || keep > 64 || n_k > GK_MAX) return cudaErrorNotSupported;
  const int n_groups = ((perm ? n_perm : n_q) + GA - 1) / GA;
  group_blocks_kernel<<<n_groups, 256, 0, st>>>(kept, keep, perm, n_q, n_k, gb_n, gb_blk, gb_slot);
  return cudaGetLastError();
}

}  // namespace sa

namespace sa {
SA_DEBUG_UNIT(dbg_read_group)
}  // namespace sa
