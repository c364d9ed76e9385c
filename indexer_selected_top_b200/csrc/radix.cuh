// radix.cuh -- CTA-wide pieces of the exact radix select (one CTA per row):
// the order-preserving score key, block reductions/scans, bucket search in a
// histogram, and a shared-memory select over unique packed 64-bit keys
// (score key << 32 | inverted id: a larger key is a better score or, at equal
// scores, a lower id -- Latent Sparse Attention appendix F.1).
#pragma once
#include <cstdint>

namespace sa {

constexpr int TK_THREADS = 512;
constexpr int TK_CAP = 12288;          // (key, index) pairs kept in shared memory
constexpr int TK_HBITS = 12;
constexpr int TK_HBINS = 1 << TK_HBITS;
constexpr uint32_t KEY_NEG_INF = 0x007FFFFFu;   // score key of -inf

static __device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0u;                    // -0 sorts with +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

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
static __device__ int block_sum(int v, int* red) {
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
static __device__ int block_excl_scan(int v, int* red, int* total) {
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
static __device__ void find_bucket(TkShared& sh, int nbins, int need) {
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
static __device__ void smem_select64(TkShared& sh, int cnt, int need, Emit emit) {
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

}  // namespace sa
