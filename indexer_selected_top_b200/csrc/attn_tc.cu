// attn_tc.cu -- grouped sparse attention on tcgen05 tensor cores.
//
// A group of 8 queries x 16 query heads is one M = 128 tile: rows r =
// 16 * query + head, so the two contractions of attention over the group's
// shared keys are dense MMAs with the accumulators in tensor memory:
//   S = Q K^T   (M 128 rows, N 128 keys, K 128 dims)  -> TMEM, two buffers
//   O += P V    (M 128 rows, N 128 dims, K 128 keys)  -> TMEM
// Q and P are the MMAs' A operands and live in tensor memory too (Q loaded
// once per group, P written by the softmax over the S columns it has read),
// so shared memory only carries the gathered K and V rows.
// Every query still attends only to its own index set J_t (Latent Sparse
// Attention section 3.2): the keys of a chunk come from the union of the
// group's sets, and a per-key byte mask says which of the 8 queries selected
// each one. The mask is applied by the tensor core itself (16 extra K dims,
// see TC_MASK_BF16): keys a row's query did not select get a logit below
// -2^99 and a softmax weight of exactly 0, so the row's softmax runs over J_t.
// The union lists (ascending keys, padded with -1 / mask 0 to whole chunks)
// come from group_union_kernel.
//
// One persistent CTA per SM loops over its groups; chunks are counted across
// groups, so the K/V ring and the S buffers run on from one group to the
// next, and the next group's first S products overlap the O write-back of
// the one before (its first O += P V waits until that O has been read).
// Roles (288 threads): warp 0 allocates TMEM and one lane issues the MMAs;
// warps 1-4 gather 32 keys each of every chunk (16-byte cp.async, whole rows
// per 16 lanes) into 128-byte-swizzled tiles, publishing them on an mbarrier
// that completes when the copies land; warps 5-8 run the softmax, one thread
// per row (TMEM lane): a pass for the row max, then a pass writing P in bf16
// while the row sum l (and with it lse) is kept in fp32. The running max is
// lazy: the O row is rescaled in TMEM only when the max grows by more than
// 2^8, so P stays below 256 and the final O / l uses one consistent reference.
// K/V tiles: each 256-byte row is split into two 128-byte halves (dims 0-63,
// 64-127), each half a [128 keys x 128 B] SW128 tile. For S the K tile is a
// K-major B operand; for O the same V tiles are an MN-major B operand (dims
// contiguous), 8 keys per 1024-byte swizzle atom.
#include <cuda_bf16.h>

#include "attn_common.cuh"
#include "ptx.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int TC_GA = 8;               // queries per group
constexpr int TC_HQ = 16;
constexpr int TC_DH = 128;
constexpr int TC_CH = kUnionChunk;     // keys per chunk (the union lists are padded to whole chunks)
constexpr int TC_ST = 3;               // K/V ring stages
constexpr int TC_LW = 4;               // loader warps (32 keys of every chunk each)
constexpr int TC_THREADS = 32 * (1 + TC_LW + 4);
// tensor memory columns
constexpr int TC_O_COL = 0;                        // O: 128 fp32 columns
constexpr int TC_S_COL = TC_DH;                    // S buffers: 2 x 128 fp32 columns (P overwrites the first 64)
constexpr int TC_Q_COL = TC_S_COL + 2 * TC_CH;     // Q: 128 dims as 64 columns of bf16 pairs
constexpr int TC_QX_COL = TC_Q_COL + TC_DH / 2;    // Q mask dims: 16 dims as 8 columns
constexpr float TC_RESCALE = 8.0f;     // log2 growth of the row max that forces a rescale
// The mask enters S through the MMA: Q gets 16 extra dims holding a one-hot
// of the row's query, K gets 16 extra dims holding -2^100 (bf16 0xF180) for
// each query of the group that did not select the key and 0 otherwise. A
// selected key's S is then exactly Q.K; an unselected one is below -2^99.
// (A finite bias: -inf times the zeros of the other rows would give NaN.)
constexpr uint16_t TC_MASK_BF16 = 0xF180;  // -2^100
constexpr float TC_MASKED = -1e29f;        // raw S below this: a masked key

// 2^x by the MUFU unit (ex2.approx.ftz: relative error near 2^-22, +0 for
// -inf and for results below the normal range)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Publishes a loader thread's copies on `bar`: the arrive-on from cp.async
// fires once this thread's earlier cp.async copies have landed, and the plain
// arrive counts the thread, so the phase completes after both.
__device__ __forceinline__ void cp_async_publish(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
  mbar_arrive(bar);
}

// Descriptor of an unswizzled K-major operand: 8-row x 16-byte core
// matrices; sbo = distance between 8-row groups, lbo = between the two
// 8-element halves of the 16-element K step.
__device__ __forceinline__ uint64_t umma_desc_noswz(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  return d;   // layout type 0: no swizzle
}

struct TcSmem {
  static constexpr int KV_HALF = TC_CH * 128;             // 16 KB: 128 keys x 64 dims
  static constexpr int KX = TC_CH * 32;                   // K mask dims: [2 halves][128 keys][16 B]
  static constexpr int STAGE = 4 * KV_HALF + KX;          // K0 K1 V0 V1 KX = 68 KB
  static constexpr int OFF_KV = 0;
  static constexpr int OFF_BAR = OFF_KV + TC_ST * STAGE;
  // full[ST] empty[ST] sfull[2] pfull[2] pvdone[2] qfull drain ofree
  static constexpr int N_BAR = 2 * TC_ST + 9;
  static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
  static constexpr int SMEM = OFF_MISC + 64 + 1024;      // + slack for 1024-byte alignment
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
};

__global__ void __launch_bounds__(TC_THREADS, 1)
    tc_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                   const __nv_bfloat16* __restrict__ vc, const int* __restrict__ list,
                   const uint8_t* __restrict__ lmask, const int* __restrict__ n_list, const int* __restrict__ perm,
                   int n_groups, int n_q, int cap, float scale_log2, __nv_bfloat16* __restrict__ out,
                   float* __restrict__ lse, uint32_t* status, long long budget) {
  using L = TcSmem;
  extern __shared__ uint8_t tc_raw[];
  uint8_t* sm = smem_align1024(tc_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = full + TC_ST;
  uint64_t* sfull = empty + TC_ST;
  uint64_t* pfull = sfull + 2;
  uint64_t* pvdone = pfull + 2;
  uint64_t* qfull = pvdone + 2;
  uint64_t* drain = qfull + 1;
  uint64_t* ofree = drain + 1;                   // the softmax has read the group's O
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + L::OFF_MISC);
  uint32_t* tmem_slot = misc;
  volatile uint32_t* abort_flag = misc + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the CTA's groups: blockIdx.x, + gridDim.x, ... (one CTA per SM). Chunks
  // are counted across them (c), so the K/V ring, the two S buffers and their
  // barrier phases run on from one group to the next; a group with no keys
  // touches none of them
  auto group_at = [&](int it) -> int {
    const long long g = (long long)it * gridDim.x + blockIdx.x;
    return g < n_groups ? (int)g : -1;
  };
  auto n_chunks = [&](int g) { return (n_list[g] + TC_CH - 1) / TC_CH; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_ST; ++s) {
      mbar_init(&full[s], 32 * TC_LW);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sfull[b], 1);
      mbar_init(&pfull[b], 128);
      mbar_init(&pvdone[b], 1);
    }
    mbar_init(qfull, 128);
    mbar_init(drain, 1);
    mbar_init(ofree, 128);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc<512>(tmem_slot);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, status, budget};

  if (warp == 0) {
    // ============================ MMA issuer ============================
    // S(c) = Q K^T of chunk c into S buffer c % 2 (Q and its mask dims read
    // from tensor memory); O += P(c) V(c) with P read from the S buffer the
    // softmax overwrote. S(c + 1) is issued before O += P(c) V(c), once the
    // buffer's previous P has been consumed; a group's first O += P V (which
    // starts O afresh) waits until the softmax has read the previous group's O.
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc<1, 128, TC_CH>();
      constexpr uint32_t idesc_o = umma_idesc_bmn<1, 128, TC_DH>();
      auto issue_s = [&](int c) -> bool {
        const int s = c % TC_ST, b = c & 1;
        if (!mbar_wait(&full[s], (c / TC_ST) & 1, wc, 40)) return false;
        if (c >= 2 && !mbar_wait(&pvdone[b], ((c - 2) >> 1) & 1, wc, 41)) return false;
        tc_fence_after();
        const uint32_t k_base = smem_u32(sm + L::OFF_KV + s * L::STAGE);
        const uint32_t d = tmem + TC_S_COL + b * TC_CH;
#pragma unroll
        for (int kk = 0; kk < TC_DH / 16; ++kk) {
          const uint64_t bd = umma_smem_desc<128>(k_base + (kk >> 2) * L::KV_HALF + (kk & 3) * 32);
          mma_bf16_ts(d, tmem + TC_Q_COL + kk * 8, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        // the mask dims: one more K step adds the -2^100 bias where the row's query did not select the key
        mma_bf16_ts(d, tmem + TC_QX_COL, umma_desc_noswz(k_base + 4 * L::KV_HALF, L::KX / 2, 128), idesc_s, 1u);
        mma_commit(&sfull[b]);
        return true;
      };
      int c0 = 0, gi = 0;                // chunks and non-empty groups before this one
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int g = group_at(it);
        if (g < 0) break;
        const int nch = n_chunks(g);
        if (nch == 0) continue;
        ok = mbar_wait(qfull, gi & 1, wc, 42);
        if (!ok) break;
        tc_fence_after();
        ok = issue_s(c0);
        for (int j = 0; ok && j < nch; ++j) {
          const int c = c0 + j;
          if (j + 1 < nch && !issue_s(c + 1)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&pfull[c & 1], (c >> 1) & 1, wc, 43)) {
            ok = false;
            break;
          }
          if (j == 0 && gi > 0 && !mbar_wait(ofree, (gi - 1) & 1, wc, 48)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t v_base = smem_u32(sm + L::OFF_KV + (c % TC_ST) * L::STAGE + 2 * L::KV_HALF);
          const uint32_t p_col = tmem + TC_S_COL + (c & 1) * TC_CH;
#pragma unroll
          for (int kk = 0; kk < TC_CH / 16; ++kk) {
            // 16 keys = two 8-key atoms of 1024 B; the two 64-dim halves 16 KB apart
            const uint64_t bd = umma_desc_sw128(v_base + kk * 2048, L::KV_HALF, 1024);
            mma_bf16_ts(tmem + TC_O_COL, p_col + kk * 8, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[c % TC_ST]);
          mma_commit(&pvdone[c & 1]);
        }
        c0 += nch;
        ++gi;
      }
      // every MMA issued has completed before tensor memory is released
      mma_commit(drain);
      mbar_wait_drain(drain, 0, wc);
    }
  } else if (warp <= TC_LW) {
    // ============================ K/V gather ============================
    // loader warp lw gathers keys [32 lw, 32 lw + 32) of every chunk and
    // their mask dims, and publishes them without waiting (the barrier phase
    // completes once all loaders' copies have landed). The next chunk's keys
    // and masks are read before waiting for its ring stage.
    const int lw = warp - 1;
    const int seg = lane & 15, half = seg >> 3, c16 = seg & 7;
    int c = 0;                               // chunks of the earlier groups
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int g = group_at(it);
      if (g < 0) break;
      const int nch = n_chunks(g);
      if (nch == 0) continue;
      const int* glist = list + (long long)g * cap;
      const uint8_t* gmask = lmask + (long long)g * cap;
      int key = glist[lw * 32 + lane];
      uint32_t msk = gmask[lw * 32 + lane];
      for (int j = 0; j < nch; ++j, ++c) {
        const int s = c % TC_ST;
        int n_key = 0;
        uint32_t n_msk = 0u;
        if (j + 1 < nch) {
          n_key = glist[(j + 1) * TC_CH + lw * 32 + lane];
          n_msk = gmask[(j + 1) * TC_CH + lw * 32 + lane];
        }
        if (c >= TC_ST && !mbar_wait(&empty[s], ((c / TC_ST) - 1) & 1, wc, 44)) {
          ok = false;
          break;
        }
        const int kr = max(key, 0);                   // padding (-1): any valid row, its mask byte is 0
        uint8_t* st = sm + L::OFF_KV + s * L::STAGE;
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
          const int rl = 2 * i + (lane >> 4);         // this warp's row
          const int r = lw * 32 + rl;                 // row of the chunk
          const long long src = (long long)__shfl_sync(0xffffffffu, kr, rl) * TC_DH + seg * 8;
          const uint32_t off = half * L::KV_HALF + r * 128 + ((c16 ^ (r & 7)) << 4);
          cp_async16(smem_u32(st + off), kc + src);
          cp_async16(smem_u32(st + 2 * L::KV_HALF + off), vc + src);
        }
        // mask dims of this lane's key: dims 0-7 carry the bias for the
        // queries that did not select it, dims 8-15 are 0
        {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t lo = ((msk >> (2 * e)) & 1u) ? 0u : TC_MASK_BF16;
            const uint32_t hi = ((msk >> (2 * e + 1)) & 1u) ? 0u : TC_MASK_BF16;
            w[e] = lo | (hi << 16);
          }
          uint8_t* kx = st + 4 * L::KV_HALF;
          const int row = lw * 32 + lane;
          *reinterpret_cast<uint4*>(kx + row * 16) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(kx + L::KX / 2 + row * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        cp_async_publish(&full[s]);
        key = n_key;
        msk = n_msk;
      }
    }
    cp_async_wait_all();   // no copy may land after the CTA has left
  } else {
    // ============================== softmax ==============================
    const int qw = warp & 3;                  // TMEM lane quarter of this warp
    const int r = qw * 32 + lane;             // row = 16 * query + head
    const int qi = r >> 4, h = r & 15;
    const uint32_t t_row = tmem + (uint32_t(qw * 32) << 16);
    int c0 = 0, gi = 0;                       // chunks and non-empty groups before this one
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int g = group_at(it);
      if (g < 0) break;
      const int nch = n_chunks(g);
      const int tq = perm ? perm[g * TC_GA + qi] : g * TC_GA + qi;
      const int t = (tq >= 0 && tq < n_q) ? tq : -1;
      if (nch == 0) {                         // no keys: a zero row and lse = -inf
        if (t >= 0) {
          __nv_bfloat16* dst = out + ((long long)t * TC_HQ + h) * TC_DH;
          for (int i = 0; i < TC_DH; i += 8) *reinterpret_cast<uint4*>(dst + i) = make_uint4(0u, 0u, 0u, 0u);
          if (lse != nullptr) lse[(long long)t * TC_HQ + h] = -INFINITY;
        }
        continue;
      }
      {
        // this row of Q (bf16 pairs: column c holds dims 2c, 2c + 1) and the
        // one-hot of its query in the mask dims; every S product of the
        // previous group has completed (this thread waited for the last)
        uint32_t qv[32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          if (t >= 0) {
            const uint4* src = reinterpret_cast<const uint4*>(q + ((long long)t * TC_HQ + h) * TC_DH + hh * 64);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint4 v = src[i];
              qv[4 * i] = v.x;
              qv[4 * i + 1] = v.y;
              qv[4 * i + 2] = v.z;
              qv[4 * i + 3] = v.w;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) qv[i] = 0u;
          }
          tmem_st32(t_row + TC_Q_COL + hh * 32, *reinterpret_cast<const float(*)[32]>(qv));
        }
        uint32_t qx[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          qx[e] = (qi == 2 * e ? 0x3F80u : 0u) | (qi == 2 * e + 1 ? 0x3F800000u : 0u);   // bf16 1.0 at dim qi
        tmem_st8(t_row + TC_QX_COL, qx);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(qfull);
      }
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < nch; ++j) {
        const int c = c0 + j, b = c & 1;
        const uint32_t s_row = t_row + TC_S_COL + b * TC_CH;
        ok = __all_sync(0xffffffffu, mbar_wait(&sfull[b], (c >> 1) & 1, wc, 45));
        if (!ok) break;
        tc_fence_after();
        // pass 1: the row max over the chunk (masked keys sit below -2^99;
        // the scale is positive, so it commutes with the max)
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int cb = 0; cb < TC_CH / 32; ++cb) {
          float sv[32];
          tmem_ld32(s_row + cb * 32, sv);
          tmem_ld_wait();
          tmem_regs_ready(sv);
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) mq[cc & 3] = fmaxf(mq[cc & 3], sv[cc]);
        }
        float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
        mx = mx < TC_MASKED ? -INFINITY : mx * scale_log2;    // no key of the chunk is the row's
        const float m_new = fmaxf(m_used, mx);
        const bool resc = m_used != -INFINITY && m_new > m_used + TC_RESCALE;
        if (m_used == -INFINITY) m_used = m_new;          // the row's O is still 0
        if (__any_sync(0xffffffffu, resc)) {
          // O must hold every earlier chunk of the group before it is rescaled in place
          ok = __all_sync(0xffffffffu, mbar_wait(&pvdone[(c - 1) & 1], ((c - 1) >> 1) & 1, wc, 47));
          if (!ok) break;
          tc_fence_after();
          const float alpha = resc ? exp2f(m_used - m_new) : 1.f;
#pragma unroll
          for (int cb = 0; cb < TC_DH / 32; ++cb) {
            float ov[32];
            tmem_ld32(t_row + TC_O_COL + cb * 32, ov);
            tmem_ld_wait();
            tmem_regs_ready(ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= alpha;
            tmem_st32(t_row + TC_O_COL + cb * 32, ov);
          }
          tmem_st_wait();
          if (resc) {
            l *= alpha;
            m_used = m_new;
          }
        }
        // pass 2: p = 2^(s * scale_log2 - m) (one FMA and one ex2 per key; a
        // masked key lands far below the normal range and gives exactly 0),
        // packed to bf16 pairs over the S columns already read: keys 32 cb ..
        // 32 cb + 31 go to columns 16 cb .. 16 cb + 15
        const float msub = m_used == -INFINITY ? 0.f : m_used;
        float2 l2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int cb = 0; cb < TC_CH / 32; ++cb) {
          float sv[32];
          tmem_ld32(s_row + cb * 32, sv);
          tmem_ld_wait();
          tmem_regs_ready(sv);
          uint32_t pw[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = ex2_approx(fmaf(sv[2 * e], scale_log2, -msub));
            const float p1 = ex2_approx(fmaf(sv[2 * e + 1], scale_log2, -msub));
            const __nv_bfloat162 pv = __floats2bfloat162_rn(p0, p1);
            l2 = __fadd2_rn(l2, make_float2(p0, p1));      // the row sum in fp32, as lse needs
            pw[e] = *reinterpret_cast<const uint32_t*>(&pv);
          }
          tmem_st16(s_row + cb * 16, pw);
        }
        l += l2.x + l2.y;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&pfull[b]);
      }
      if (!ok) break;
      // epilogue: O / l in bf16, lse in natural log; then O is free for the
      // next group's first O += P V
      const int cl = c0 + nch - 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&pvdone[cl & 1], (cl >> 1) & 1, wc, 49));
      if (!ok) break;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* dst = out + ((long long)(t < 0 ? 0 : t) * TC_HQ + h) * TC_DH;
#pragma unroll
      for (int cb = 0; cb < TC_DH / 32; ++cb) {
        float ov[32];
        tmem_ld32(t_row + TC_O_COL + cb * 32, ov);
        tmem_ld_wait();
        tmem_regs_ready(ov);
        if (t >= 0) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 pk;
            pk.x = pack_bf16(ov[i] * inv, ov[i + 1] * inv);
            pk.y = pack_bf16(ov[i + 2] * inv, ov[i + 3] * inv);
            pk.z = pack_bf16(ov[i + 4] * inv, ov[i + 5] * inv);
            pk.w = pack_bf16(ov[i + 6] * inv, ov[i + 7] * inv);
            *reinterpret_cast<uint4*>(dst + cb * 32 + i) = pk;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(ofree);
      if (t >= 0 && lse != nullptr)
        lse[(long long)t * TC_HQ + h] = l > 0.f ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
      c0 += nch;
      ++gi;
    }
  }

  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc<512>(tmem);
  }
}

bool tc_attention_supported(int hq, int dh) { return hq == TC_HQ && dh == TC_DH; }

cudaError_t launch_attention_tc(const void* q, const void* kc, const void* vc, const int* list, const uint8_t* lmask,
                                const int* n_list, const int* perm, int n_groups, int n_q, int cap, float scale,
                                void* out, float* lse, uint32_t* status, long long budget, cudaStream_t st) {
  if (n_groups <= 0) return cudaSuccess;
  if (cap % TC_CH != 0) return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(tc_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TcSmem::SMEM);
  if (e != cudaSuccess) return e;
  // one persistent CTA per SM (at most one per group)
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int grid = n_groups < sms ? n_groups : sms;
  tc_attn_kernel<<<grid, TC_THREADS, TcSmem::SMEM, st>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)kc, (const __nv_bfloat16*)vc, list, lmask, n_list, perm,
      n_groups, n_q, cap, scale * 1.4426950408889634f, (__nv_bfloat16*)out, lse, status, budget);
  return cudaGetLastError();
}

}  // namespace sa
