// topk_fast.cu -- exact top-k of rows of at most 4096 scores with the keys
// held in registers (TF_PER per thread), one CTA per row.
//
// Same order as topk.cu: higher score first, lower key index on ties (the
// packed key of Latent Sparse Attention appendix F.1), found by radix select.
// Radix passes start below the bits that every valid key of the row shares
// (block AND / OR of the keys), so a row whose scores sit within one octave
// does not spend passes on its common exponent bits; each pass histograms an
// 8-bit digit in per-warp shared histograms and stops early once the bucket
// holding the cut is taken whole. Ties at the cut take the lowest positions by
// an ordered block scan.
#include "sa_internal.h"

namespace sa {

// Tuning knobs: keys per thread (32 or 16; the CTA holds 4096 keys either way)
// and resident CTAs per SM the registers are sized for. 16 keys x 256 threads
// at 6 CTAs per SM measured fastest (the passes are latency-bound; the few
// registers this leaves cost a small spill).
#ifndef SA_TF_PER
#define SA_TF_PER 16
#endif
#ifndef SA_TF_MINB
#define SA_TF_MINB 6
#endif
constexpr int TF_PER = SA_TF_PER;                  // keys per thread
constexpr int TF_THREADS = 4096 / TF_PER;
constexpr int TF_MAXN = TF_THREADS * TF_PER;       // 4096

static __device__ __forceinline__ uint32_t tf_key(float x) {
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct TfShared {
  uint32_t hist[TF_THREADS / 32][256];
  int red[TF_THREADS / 32];
  uint32_t redu[2][TF_THREADS / 32];
  int bucket, above, inb, n_out;
  int kb[64];
};

// Row modes: 0 = causal table row (columns [0, min(n_cols, p + 1)) all valid,
// key = column); 2 = two-stage candidate row (columns [0, 64 * #kept), key =
// 64 * kept[c / 64] + c % 64, valid iff score > -inf).
__global__ void __launch_bounds__(TF_THREADS, SA_TF_MINB)
    topk_fast_kernel(const float* __restrict__ scores, int n_rows, long long ld, int n_cols, int q_pos0,
                     const int* __restrict__ row_pos, const int* __restrict__ kept, int keep, int k,
                     int32_t* __restrict__ idx, uint32_t* __restrict__ sel) {
  __shared__ TfShared sh;
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool gathered = kept != nullptr;
  int n;
  if (gathered) {
    // kept lists are -1 padded at the tail: the kept count is one block count
    int kbv = -1;
    if (tid < 64) {
      kbv = tid < keep ? kept[(long long)row * keep + tid] : -1;
      sh.kb[tid] = kbv;
    }
    const int nb = __syncthreads_count(kbv >= 0);
    n = min(n_cols, nb * 64);
  } else {
    n = max(0, min(n_cols, (row_pos ? row_pos[row] : q_pos0 + row) + 1));
  }
  // keys of columns [tid * 32, tid * 32 + 32); invalid -> 0 (below every valid key)
  const float* src = scores + row * ld;
  uint32_t key[TF_PER];
  int nv = 0;
  uint32_t andk = 0xFFFFFFFFu, ork = 0u;
  const int c0 = tid * TF_PER;
  float vals[TF_PER];
  if ((ld & 3) == 0 && c0 + TF_PER <= n && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
    const float4* s4 = reinterpret_cast<const float4*>(src + c0);
#pragma unroll
    for (int i = 0; i < TF_PER / 4; ++i) {
      const float4 v = s4[i];
      vals[4 * i] = v.x;
      vals[4 * i + 1] = v.y;
      vals[4 * i + 2] = v.z;
      vals[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < TF_PER; ++i) vals[i] = (c0 + i < n) ? src[c0 + i] : 0.f;
  }
#pragma unroll
  for (int i = 0; i < TF_PER; ++i) {
    uint32_t kk = 0u;
    if (c0 + i < n) {
      kk = tf_key(vals[i]);
      if (gathered && kk == 0x007FFFFFu) kk = 0u;     // -inf: an invisible key
    }
    key[i] = kk;
    if (kk != 0u) {
      ++nv;
      andk &= kk;
      ork |= kk;
    }
  }
  // block reductions: valid count, AND and OR of the valid keys
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    nv += __shfl_xor_sync(0xffffffffu, nv, o);
    andk &= __shfl_xor_sync(0xffffffffu, andk, o);
    ork |= __shfl_xor_sync(0xffffffffu, ork, o);
  }
  if (lane == 0) {
    sh.red[warp] = nv;
    sh.redu[0][warp] = andk;
    sh.redu[1][warp] = ork;
  }
  if (tid == 0) sh.n_out = 0;
  __syncthreads();
  nv = 0;
  andk = 0xFFFFFFFFu;
  ork = 0u;
#pragma unroll
  for (int w = 0; w < TF_THREADS / 32; ++w) {
    nv += sh.red[w];
    andk &= sh.redu[0][w];
    ork |= sh.redu[1][w];
  }
  int32_t* out = idx + (long long)row * k;
  // the thread's TF_PER columns lie in one 64-key block: its first key id
  // (gathered rows: the block's key base) is looked up once
  static_assert(64 % TF_PER == 0, "a thread's columns share one kept block");
  const int key0 = gathered ? (c0 < 64 * 64 ? sh.kb[c0 >> 6] * 64 + (c0 & 63) : 0) : c0;
  auto key_of = [&](int c) { return key0 + (c - c0); };
  // ordered emission of the positions whose flag is set (block scan over
  // (thread, element)); returns the thread's emitted elements as a bit mask
  auto emit_ordered = [&](auto flag, int base, int limit) -> uint32_t {
    int mine = 0;
#pragma unroll
    for (int i = 0; i < TF_PER; ++i) mine += flag(i) ? 1 : 0;
    int x = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) sh.red[warp] = x;
    __syncthreads();
    int before = 0;
#pragma unroll
    for (int w = 0; w < TF_THREADS / 32; ++w)
      if (w < warp) before += sh.red[w];
    int p = base + before + x - mine;
    uint32_t emitted = 0u;
#pragma unroll
    for (int i = 0; i < TF_PER; ++i)
      if (flag(i)) {
        if (p < limit) {
          out[p] = key_of(c0 + i);
          emitted |= 1u << i;
        }
        ++p;
      }
    return emitted;
  };
  // selection bitmap of a gathered row: word i covers columns [32 i, 32 i + 32)
  auto put_sel = [&](uint32_t word) {
    if constexpr (TF_PER == 32) {
      if (sel != nullptr && tid < keep * 2) sel[(long long)row * keep * 2 + tid] = word;
    } else {
      const uint32_t hi = __shfl_down_sync(0xffffffffu, word, 1);   // the next thread's 16 columns
      if (sel != nullptr && (tid & 1) == 0 && tid / 2 < keep * 2)
        sel[(long long)row * keep * 2 + tid / 2] = (word & 0xFFFFu) | (hi << 16);
    }
  };
  if (nv <= k) {
    put_sel(emit_ordered([&](int i) { return key[i] != 0u; }, 0, k));
    for (int j = nv + tid; j < k; j += TF_THREADS) out[j] = -1;
    return;
  }
  // radix select below the bits every valid key shares
  const uint32_t diff = andk ^ ork;                    // nonzero: nv > k >= 1 keys, not all equal
  int hi = diff ? 31 - __clz(diff) : -1;               // highest bit that differs
  uint32_t prefix = andk, pmask = diff ? ~((2u << hi) - 1u) : 0xFFFFFFFFu;
  if (hi == 31) pmask = 0u;
  prefix &= pmask;
  int need = k;
  uint32_t cut = prefix;
  int ties = -1;
  bool done = (hi < 0);
  if (done) ties = need;                               // every valid key equal
  while (!done) {
    const int lo = max(0, hi - 7);
    const int nbits = hi - lo + 1;
    for (int b = tid; b < (TF_THREADS / 32) * 256; b += TF_THREADS) (&sh.hist[0][0])[b] = 0u;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < TF_PER; ++i) {
      const uint32_t kk = key[i];
      if (kk != 0u && (kk & pmask) == prefix) atomicAdd(&sh.hist[warp][(kk >> lo) & ((1u << nbits) - 1u)], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits [255 - 8l - 7, 255 - 8l] (from the top)
      uint32_t hb[8];
      int mine = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int d = 255 - 8 * lane - j;
        uint32_t v = 0;
#pragma unroll
        for (int w = 0; w < TF_THREADS / 32; ++w) v += sh.hist[w][d];
        hb[j] = v;
        mine += v;
      }
      int incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int before = incl - mine;
      if (before < need && incl >= need) {
        int acc = before;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (acc + (int)hb[j] >= need) {
            sh.bucket = 255 - 8 * lane - j;
            sh.above = acc;
            sh.inb = hb[j];
            break;
          }
          acc += hb[j];
        }
      }
    }
    __syncthreads();
    need -= sh.above;
    prefix |= (uint32_t)sh.bucket << lo;
    pmask |= ((1u << nbits) - 1u) << lo;
    if (sh.inb == need) {                              // the whole bucket is taken
      cut = prefix;
      ties = -1;
      done = true;
    } else if (lo == 0) {                              // full key: `need` lowest positions of key == prefix
      cut = prefix;
      ties = need;
      done = true;
    }
    hi = lo - 1;
    __syncthreads();
  }
  // every key strictly above the cut (or, for a bucket taken whole, at or above)
  int base = 0;
  uint32_t word = 0u;
  {
    const bool whole = ties < 0;
#pragma unroll
    for (int i = 0; i < TF_PER; ++i) {
      const uint32_t kk = key[i];
      const bool take = kk != 0u && (whole ? kk >= cut : kk > cut);
      if (take) {
        out[atomicAdd(&sh.n_out, 1)] = key_of(c0 + i);
        word |= 1u << i;
      }
    }
    __syncthreads();
    base = sh.n_out;
  }
  if (ties > 0) word |= emit_ordered([&](int i) { return key[i] != 0u && key[i] == cut; }, base, base + ties);
  put_sel(word);
}

cudaError_t launch_topk_fast(const float* scores, int n_rows, long long ld, int n_cols, int q_pos0, const int* row_pos,
                             const int* kept, int keep, int k, int32_t* idx, cudaStream_t st, uint32_t* sel) {
  if (n_rows <= 0) return cudaSuccess;
  if ((kept != nullptr ? keep * 64 : n_cols) > TF_MAXN) return cudaErrorNotSupported;
  topk_fast_kernel<<<n_rows, TF_THREADS, 0, st>>>(scores, n_rows, ld, n_cols, q_pos0, row_pos, kept, keep, k, idx,
                                                  kept != nullptr ? sel : nullptr);
  return cudaGetLastError();
}

}  // namespace sa
