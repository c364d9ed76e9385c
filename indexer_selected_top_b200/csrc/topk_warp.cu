// topk_warp.cu -- the stage-1 block keep: the best keep - 2 block scores of
// each query row, one warp per row.
//
// Same order as topk.cu (higher score first, lower index on ties; the packed
// key of Latent Sparse Attention appendix F.1) and the same radix select,
// restated for one warp: the row's order-preserving 32-bit score keys sit in
// shared memory, each pass histograms the next 8-bit digit of the keys that
// still match the prefix (per-instruction match aggregation keeps the shared
// atomics low), and the pass stops early once the bucket holding the cut is
// taken whole. Ties at the cut take the lowest positions by an ordered ballot
// scan. Rows of at most 4096 blocks (longer ones go to block_select_kernel).
#include "sa_internal.h"

namespace sa {

constexpr int TW_WARPS = 4;

__device__ __forceinline__ uint32_t tw_key(float x) {
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Finds the cut of the `need` largest keys among keys[0..n) (keys[i] counts
// iff valid(i)). Result (cut, ties): if ties < 0 the selection is every key
// >= cut; otherwise it is every key > cut plus the `ties` lowest positions of
// the keys == cut.
template <class Valid>
__device__ void warp_cut(const uint32_t* keys, int n, int need, uint32_t* hist, Valid valid, uint32_t& cut,
                         int& ties) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, mask = 0;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int i0 = 0; i0 < n; i0 += 32) {
      const int i = i0 + lane;
      bool in = false;
      uint32_t dig = 0;
      if (i < n && valid(i)) {
        const uint32_t kk = keys[i];
        in = (kk & mask) == prefix;
        dig = (kk >> shift) & 255u;
      }
      const unsigned act = __ballot_sync(0xffffffffu, in);
      if (in) {
        const unsigned peers = __match_any_sync(act, dig);
        if ((__ffs(peers) - 1) == lane) atomicAdd(&hist[dig], __popc(peers));
      }
    }
    __syncwarp();
    // lane l owns bins [248 - 8l, 255 - 8l] (from the top)
    uint32_t hb[8];
    int mine = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      hb[j] = hist[255 - 8 * lane - j];
      mine += hb[j];
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int before = incl - mine;
    const bool here = before < need && incl >= need;
    const unsigned who = __ballot_sync(0xffffffffu, here);
    const int src = __ffs(who) - 1;
    int d = 0, above = 0, inb = 0;
    if (lane == src) {
      int acc = before;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (acc + (int)hb[j] >= need) {
          d = 255 - 8 * lane - j;
          above = acc;
          inb = hb[j];
          break;
        }
        acc += hb[j];
      }
    }
    d = __shfl_sync(0xffffffffu, d, src);
    above = __shfl_sync(0xffffffffu, above, src);
    inb = __shfl_sync(0xffffffffu, inb, src);
    need -= above;
    prefix |= (uint32_t)d << shift;
    mask |= 255u << shift;
    if (inb == need) {             // the whole bucket is taken
      cut = prefix;                // select key >= smallest key with this prefix
      ties = -1;
      __syncwarp();
      return;
    }
  }
  cut = prefix;                    // full 32-bit key: take `need` lowest positions of key == cut
  ties = need;
  __syncwarp();
}

constexpr int BW_MAXB = 4096;                 // blocks per row held in shared memory

__global__ void __launch_bounds__(TW_WARPS * 32)
    block_keep_warp_kernel(const float* __restrict__ bscores, int n_q, long long ld, int q_pos0, int block, int keep,
                           int* __restrict__ kept, int cap) {
  extern __shared__ uint32_t bw_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // per warp: cap block keys, a 256-bin histogram, cap / 32 flag words
  uint32_t* keys = bw_smem + warp * (cap + 256 + cap / 32);
  uint32_t* hist = keys + cap;
  uint32_t* flags = hist + 256;
  const int t = blockIdx.x * TW_WARPS + warp;
  if (t >= n_q) return;
  const int cur = (q_pos0 + t) / block;
  const int n_other = max(0, cur - 1);             // blocks 1 .. cur-1
  int* out = kept + (long long)t * keep;
  const int nw = (cur + 1 + 31) / 32;
  for (int j = lane; j < nw; j += 32) flags[j] = 0u;
  __syncwarp();
  if (lane == 0) {
    flags[0] |= 1u;
    flags[cur >> 5] |= 1u << (cur & 31);
  }
  const float* row = bscores + (long long)t * ld;
  if (n_other <= keep - 2) {
    for (int b = 1 + lane; b <= n_other; b += 32) atomicOr(&flags[b >> 5], 1u << (b & 31));
  } else {
    // the row's scores, eight loads per lane in flight before any is stored
    for (int i0 = 0; i0 < n_other; i0 += 32 * 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + lane + 32 * u;
        v[u] = (i < n_other) ? row[1 + i] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + lane + 32 * u;
        if (i < n_other) keys[i] = tw_key(v[u]);
      }
    }
    __syncwarp();
    uint32_t cut;
    int ties;
    warp_cut(keys, n_other, keep - 2, hist, [](int) { return true; }, cut, ties);
    for (int i0 = 0; i0 < n_other; i0 += 32) {
      const int i = i0 + lane;
      bool take = false;
      if (i < n_other) {
        const uint32_t kk = keys[i];
        take = (ties < 0) ? (kk >= cut) : (kk > cut);
      }
      if (take) atomicOr(&flags[(1 + i) >> 5], 1u << ((1 + i) & 31));
    }
    if (ties > 0) {
      for (int i0 = 0; i0 < n_other && ties > 0; i0 += 32) {
        const int i = i0 + lane;
        const bool eq = i < n_other && keys[i] == cut;
        const unsigned b = __ballot_sync(0xffffffffu, eq);
        const int r = __popc(b & ((1u << lane) - 1));
        if (eq && r < ties) atomicOr(&flags[(1 + i) >> 5], 1u << ((1 + i) & 31));
        ties -= min(ties, __popc(b));
      }
    }
  }
  __syncwarp();
  // ascending compaction of the flags (one 32-block word per lane step)
  int pos = 0;
  for (int w0 = 0; w0 < nw; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t f = (w < nw) ? flags[w] : 0u;
    const int c = __popc(f);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int p = pos + incl - c;
    uint32_t bits = f;
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      if (p < keep) out[p] = w * 32 + bit;
      ++p;
    }
    pos += __shfl_sync(0xffffffffu, incl, 31);
  }
  for (int j = min(pos, keep) + lane; j < keep; j += 32) out[j] = -1;
}

cudaError_t launch_block_keep_warp(const float* bscores, int n_q, long long ld, int q_pos0, int block, int keep,
                                   int* kept, cudaStream_t st) {
  if (n_q <= 0) return cudaSuccess;
  if ((q_pos0 + n_q - 1) / block >= BW_MAXB) return cudaErrorNotSupported;
  // shared memory sized by the largest current block of the call (not the
  // 4096-block maximum), so more CTAs fit per SM
  const int cap = ((q_pos0 + n_q - 1) / block + 1 + 31) / 32 * 32;
  const int smem = TW_WARPS * (cap + 256 + cap / 32) * 4;
  cudaError_t e = cudaFuncSetAttribute(block_keep_warp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  block_keep_warp_kernel<<<(n_q + TW_WARPS - 1) / TW_WARPS, TW_WARPS * 32, smem, st>>>(bscores, n_q, ld, q_pos0, block,
                                                                                       keep, kept, cap);
  return cudaGetLastError();
}

}  // namespace sa
