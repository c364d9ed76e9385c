// attn_tc.cu -- grouped sparse attention on tcgen05 tensor cores.
//
// A group of 8 queries x 16 query heads is one M = 128 tile: rows r =
// 16 * query + head, so the two contractions of attention over the group's
// shared keys are dense MMAs with the accumulators in tensor memory:
//   S = Q K^T   (M 128 rows, N 64 keys, K 128 dims)   -> TMEM, two buffers
//   O += P V    (M 128 rows, N 128 dims, K 64 keys)   -> TMEM
// Every query still attends only to its own index set J_t (Latent Sparse
// Attention section 3.2): the keys of a chunk come from the union of the
// group's sets, and a per-key byte mask says which of the 8 queries selected
// each one. The mask is applied by the tensor core itself (16 extra K dims,
// see TC_MASK_BF16): keys a row's query did not select get a logit below
// -2^99 and a softmax weight of exactly 0, so the row's softmax runs over J_t. The union lists (ascending keys, whole
// chunks of 64, padded with -1 / mask 0) come from group_union_kernel.
//
// Roles (288 threads): warp 0 allocates TMEM and one lane issues the MMAs;
// warps 1-4 gather whole chunks of K and V rows in turn (16-byte cp.async,
// whole rows per 16 lanes) into 128-byte-swizzled tiles, publishing each on
// an mbarrier that completes when the copies land; warps 5-8 run the
// softmax, one thread per row (TMEM lane); P enters the MMA in bf16 while the row sum l
// (and with it lse) is kept in fp32. The softmax keeps a running max per row and
// rescales the O row in TMEM only when the max grows by more than 2^8, so P
// stays below 256 and the final O / l uses one consistent reference.
// K/V tiles: each 256-byte row is split into two 128-byte halves (dims 0-63,
// 64-127), each half a [64 keys x 128 B] SW128 tile. For S the K tile is a
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
constexpr int TC_ROWS = TC_GA * TC_HQ; // 128
constexpr int TC_CH = 64;              // keys per chunk
constexpr int TC_ST = 4;               // K/V ring stages
constexpr int TC_NSB = 3;              // S accumulators in TMEM (S = Q K^T runs ahead of O += P V)
constexpr int TC_NPB = 3;              // P buffers in shared memory
constexpr int TC_LW = 4;               // loader warps
constexpr int TC_THREADS = 32 * (1 + TC_LW + 4);
constexpr int TC_O_COL = TC_NSB * TC_CH;   // TMEM column of O
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
  static constexpr int Q_HALF = TC_ROWS * 128;            // 16 KB
  static constexpr int KV_HALF = TC_CH * 128;             // 8 KB
  static constexpr int QX = TC_ROWS * 32;                 // Q mask dims: [2 halves][128 rows][16 B]
  static constexpr int KX = TC_CH * 32;                   // K mask dims: [2 halves][64 keys][16 B]
  static constexpr int STAGE = 4 * KV_HALF + 1024 * ((KX + 1023) / 1024);   // K0 K1 V0 V1 KX
  static constexpr int P_BYTES = TC_ROWS * 128;           // 128 rows x 64 keys bf16
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_QX = OFF_Q + 2 * Q_HALF;
  static constexpr int OFF_KV = OFF_QX + 1024 * ((QX + 1023) / 1024);
  static constexpr int OFF_P = OFF_KV + TC_ST * STAGE;
  static constexpr int OFF_BAR = OFF_P + TC_NPB * P_BYTES;
  // full[ST] empty[ST] sfull[NSB] sfree[NSB] pfull[NPB] pvdone[NPB] qfull drain
  static constexpr int N_BAR = 2 * TC_ST + 2 * TC_NSB + 2 * TC_NPB + 2;
  static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
  static constexpr int SMEM = OFF_MISC + 64 + 1024;      // + slack for 1024-byte alignment
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

__global__ void __launch_bounds__(TC_THREADS, 1)
    tc_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                   const __nv_bfloat16* __restrict__ vc, const int* __restrict__ list,
                   const uint8_t* __restrict__ lmask, const int* __restrict__ n_list, const int* __restrict__ perm,
                   int n_q, int cap, float scale_log2, __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                   uint32_t* status, long long budget) {
  using L = TcSmem;
  extern __shared__ uint8_t tc_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = full + TC_ST;
  uint64_t* sfull = empty + TC_ST;
  uint64_t* sfree = sfull + TC_NSB;
  uint64_t* pfull = sfree + TC_NSB;
  uint64_t* pvdone = pfull + TC_NPB;
  uint64_t* qfull = pvdone + TC_NPB;
  uint64_t* drain = qfull + 1;
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + L::OFF_MISC);
  uint32_t* tmem_slot = misc;
  volatile uint32_t* abort_flag = misc + 1;
  int* qt = reinterpret_cast<int*>(misc + 2);     // [TC_GA]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x;
  const int nl = n_list[g];
  const int nch = (nl + TC_CH - 1) / TC_CH;
  const int* glist = list + (long long)g * cap;
  const uint8_t* gmask = lmask + (long long)g * cap;

  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_ST; ++s) {
      mbar_init(&full[s], 32);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < TC_NSB; ++b) {
      mbar_init(&sfull[b], 1);
      mbar_init(&sfree[b], 128);
    }
    for (int b = 0; b < TC_NPB; ++b) {
      mbar_init(&pfull[b], 128);
      mbar_init(&pvdone[b], 1);
    }
    mbar_init(qfull, 128);
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (threadIdx.x < TC_GA) {
    const int j = g * TC_GA + threadIdx.x;
    const int t = perm ? perm[j] : j;
    qt[threadIdx.x] = (t >= 0 && t < n_q) ? t : -1;
  }
  if (warp == 0) tmem_alloc<512>(tmem_slot);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, status, budget};

  if (warp == 0) {
    // ============================ MMA issuer ============================
    // S = Q K^T of chunk i goes to S buffer i % NSB as soon as the chunk has
    // landed and the softmax has read that buffer's previous chunk, so it
    // runs up to NSB - 1 chunks ahead of O += P V
    if (lane == 0 && nch > 0) {
      constexpr uint32_t idesc_s = umma_idesc<1, 128, TC_CH>();
      constexpr uint32_t idesc_o = umma_idesc_bmn<1, 128, TC_DH>();
      const uint32_t q_base = smem_u32(sm + L::OFF_Q);
      const uint64_t qx_desc = umma_desc_noswz(smem_u32(sm + L::OFF_QX), L::QX / 2, 128);
      int n_s = 0;                          // S products issued
      auto issue_s = [&]() -> bool {
        const int i = n_s, s = i % TC_ST, b = i % TC_NSB;
        if (!mbar_wait(&full[s], (i / TC_ST) & 1, wc, 40)) return false;
        if (i >= TC_NSB && !mbar_wait(&sfree[b], ((i / TC_NSB) - 1) & 1, wc, 41)) return false;
        tc_fence_after();
        const uint32_t k_base = smem_u32(sm + L::OFF_KV + s * L::STAGE);
#pragma unroll
        for (int kk = 0; kk < TC_DH / 16; ++kk) {
          const uint64_t ad = umma_smem_desc<128>(q_base + (kk >> 2) * L::Q_HALF + (kk & 3) * 32);
          const uint64_t bd = umma_smem_desc<128>(k_base + (kk >> 2) * L::KV_HALF + (kk & 3) * 32);
          mma_bf16(tmem + b * TC_CH, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        // the mask dims: one more K step adds the -2^100 bias where the row's query did not select the key
        mma_bf16(tmem + b * TC_CH, qx_desc, umma_desc_noswz(k_base + 4 * L::KV_HALF, L::KX / 2, 128), idesc_s, 1u);
        mma_commit(&sfull[b]);
        ++n_s;
        return true;
      };
      bool ok = mbar_wait(qfull, 0, wc, 42);
      if (ok) tc_fence_after();
      for (int j = 0; ok && j < nch; ++j) {
        while (ok && n_s < nch && n_s < j + TC_NSB) ok = issue_s();
        if (!ok || !mbar_wait(&pfull[j % TC_NPB], (j / TC_NPB) & 1, wc, 43)) break;
        tc_fence_after();
        const uint32_t v_base = smem_u32(sm + L::OFF_KV + (j % TC_ST) * L::STAGE + 2 * L::KV_HALF);
        const uint32_t p_base = smem_u32(sm + L::OFF_P + (j % TC_NPB) * L::P_BYTES);
#pragma unroll
        for (int kk = 0; kk < TC_CH / 16; ++kk) {
          const uint64_t ad = umma_smem_desc<128>(p_base + kk * 32);
          // 16 keys = two 8-key atoms of 1024 B; the two 64-dim halves 8 KB apart
          const uint64_t bd = umma_desc_sw128(v_base + kk * 2048, L::KV_HALF, 1024);
          mma_bf16(tmem + TC_O_COL, ad, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[j % TC_ST]);
        mma_commit(&pvdone[j % TC_NPB]);
      }
      // every MMA issued has completed before tensor memory is released
      mma_commit(drain);
      mbar_wait_drain(drain, 0, wc);
    }
  } else if (warp <= TC_LW) {
    // ============================ K/V gather ============================
    // loader warp lw owns chunks lw, lw + TC_LW, ...: it gathers a whole
    // chunk, writes its mask dims, and publishes it without waiting (the
    // barrier phase completes once the copies have landed). The next chunk's
    // keys and masks are read before waiting for its ring stage.
    const int lw = warp - 1;
    const int seg = lane & 15, half = seg >> 3, c16 = seg & 7;
    int k_lo = 0, k_hi = 0;
    uint32_t m_lo = 0u, m_hi = 0u;
    if (lw < nch) {
      k_lo = glist[lw * TC_CH + lane];
      k_hi = glist[lw * TC_CH + 32 + lane];
      m_lo = gmask[lw * TC_CH + lane];
      m_hi = gmask[lw * TC_CH + 32 + lane];
    }
    for (int j = lw; j < nch; j += TC_LW) {
      const int s = j % TC_ST;
      const int jn = j + TC_LW;
      int n_klo = 0, n_khi = 0;
      uint32_t n_mlo = 0u, n_mhi = 0u;
      if (jn < nch) {
        n_klo = glist[jn * TC_CH + lane];
        n_khi = glist[jn * TC_CH + 32 + lane];
        n_mlo = gmask[jn * TC_CH + lane];
        n_mhi = gmask[jn * TC_CH + 32 + lane];
      }
      if (j >= TC_ST && !mbar_wait(&empty[s], ((j / TC_ST) - 1) & 1, wc, 44)) break;
      k_lo = max(k_lo, 0);                    // padding (-1): any valid row, its mask byte is 0
      k_hi = max(k_hi, 0);
      uint8_t* st = sm + L::OFF_KV + s * L::STAGE;
#pragma unroll 8
      for (int i = 0; i < TC_CH / 2; ++i) {
        const int r = 2 * i + (lane >> 4);
        const int key = __shfl_sync(0xffffffffu, i < 16 ? k_lo : k_hi, r & 31);
        const long long src = (long long)key * TC_DH + seg * 8;
        const uint32_t off = half * L::KV_HALF + r * 128 + ((c16 ^ (r & 7)) << 4);
        cp_async16(smem_u32(st + off), kc + src);
        cp_async16(smem_u32(st + 2 * L::KV_HALF + off), vc + src);
      }
      // mask dims of keys lane and 32 + lane: dims 0-7 carry the bias for
      // the queries that did not select the key, dims 8-15 are 0
      uint8_t* kx = st + 4 * L::KV_HALF;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint32_t m = hh ? m_hi : m_lo;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t lo = ((m >> (2 * e)) & 1u) ? 0u : TC_MASK_BF16;
          const uint32_t hi = ((m >> (2 * e + 1)) & 1u) ? 0u : TC_MASK_BF16;
          w[e] = lo | (hi << 16);
        }
        const int key_row = hh * 32 + lane;
        *reinterpret_cast<uint4*>(kx + key_row * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(kx + L::KX / 2 + key_row * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      cp_async_publish(&full[s]);
      k_lo = n_klo;
      k_hi = n_khi;
      m_lo = n_mlo;
      m_hi = n_mhi;
    }
    cp_async_wait_all();   // no copy may land after the CTA has left
  } else {
    // ============================== softmax ==============================
    const int qw = warp & 3;                  // TMEM lane quarter of this warp
    const int r = qw * 32 + lane;             // row = 16 * query + head
    const int qi = r >> 4, h = r & 15;
    const int t = qt[qi];
    const uint32_t t_row = tmem + (uint32_t(qw * 32) << 16);
    {
      // this row of the Q tile (two 128-byte halves, swizzled) and its mask dims
      uint8_t* qa = sm + L::OFF_Q;
      if (t >= 0) {
        const __nv_bfloat16* src = q + ((long long)t * TC_HQ + h) * TC_DH;
#pragma unroll
        for (int sg = 0; sg < 16; ++sg)
          cp_async16(smem_u32(qa + (sg >> 3) * L::Q_HALF + r * 128 + (((sg & 7) ^ (r & 7)) << 4)), src + sg * 8);
        cp_async_commit();
        cp_async_wait<0>();
      } else {
#pragma unroll
        for (int sg = 0; sg < 16; ++sg)
          *reinterpret_cast<uint4*>(qa + (sg >> 3) * L::Q_HALF + r * 128 + (((sg & 7) ^ (r & 7)) << 4)) =
              make_uint4(0u, 0u, 0u, 0u);
      }
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        w[e] = (qi == 2 * e ? 0x3F80u : 0u) | (qi == 2 * e + 1 ? 0x3F800000u : 0u);   // bf16 1.0 at dim qi
      uint8_t* qx = sm + L::OFF_QX;
      *reinterpret_cast<uint4*>(qx + r * 16) = make_uint4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<uint4*>(qx + L::QX / 2 + r * 16) = make_uint4(0u, 0u, 0u, 0u);
      fence_proxy_async_smem();
      mbar_arrive(qfull);
    }
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nch; ++j) {
      const int b = j % TC_NSB, pb = j % TC_NPB;
      ok = __all_sync(0xffffffffu, mbar_wait(&sfull[b], (j / TC_NSB) & 1, wc, 45));
      if (!ok) break;
      tc_fence_after();
      float sv[TC_CH];
      tmem_ld32(t_row + b * TC_CH, *reinterpret_cast<float(*)[32]>(sv));
      tmem_ld32(t_row + b * TC_CH + 32, *reinterpret_cast<float(*)[32]>(sv + 32));
      tmem_ld_wait();
      tmem_regs_ready(*reinterpret_cast<float(*)[32]>(sv));
      tmem_regs_ready(*reinterpret_cast<float(*)[32]>(sv + 32));
      tc_fence_before();
      mbar_arrive(&sfree[b]);
      // the row max over the chunk (masked keys sit below -2^99; the scale
      // is positive, so it commutes with the max)
      float mq[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
      for (int c = 4; c < TC_CH; ++c) mq[c & 3] = fmaxf(mq[c & 3], sv[c]);
      float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      mx = mx < TC_MASKED ? -INFINITY : mx * scale_log2;    // no key of the chunk is the row's
      const float m_new = fmaxf(m_used, mx);
      const bool resc = m_used != -INFINITY && m_new > m_used + TC_RESCALE;
      if (m_used == -INFINITY) m_used = m_new;          // the row's O is still 0
      if (__any_sync(0xffffffffu, resc)) {
        // O must hold every earlier chunk before it is rescaled in place
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&pvdone[(j - 1) % TC_NPB], ((j - 1) / TC_NPB) & 1, wc, 47));
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
      // P buffer pb is free once the O update of chunk j - NPB has completed
      if (j >= TC_NPB) {
        ok = __all_sync(0xffffffffu, mbar_wait(&pvdone[pb], ((j / TC_NPB) - 1) & 1, wc, 48));
        if (!ok) break;
      }
      uint8_t* prow = sm + L::OFF_P + pb * L::P_BYTES + (r >> 3) * 1024 + (r & 7) * 128;
      // p = 2^(s * scale_log2 - m): one FMA and one ex2 per key; a masked
      // key lands far below the normal range and gives exactly 0. A row with
      // no valid key yet subtracts 0.
      const float msub = m_used == -INFINITY ? 0.f : m_used;
      float2 l2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int c8 = 0; c8 < TC_CH / 8; ++c8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = ex2_approx(fmaf(sv[c8 * 8 + 2 * e], scale_log2, -msub));
          const float p1 = ex2_approx(fmaf(sv[c8 * 8 + 2 * e + 1], scale_log2, -msub));
          const __nv_bfloat162 pv = __floats2bfloat162_rn(p0, p1);
          l2 = __fadd2_rn(l2, make_float2(p0, p1));      // the row sum in fp32, as lse needs
          w[e] = *reinterpret_cast<const uint32_t*>(&pv);
        }
        *reinterpret_cast<uint4*>(prow + ((c8 ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      l += l2.x + l2.y;
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&pfull[pb]);
    }
    // epilogue: O / l in bf16, lse in natural log
    if (ok && nch > 0) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&pvdone[(nch - 1) % TC_NPB], ((nch - 1) / TC_NPB) & 1, wc, 49));
      if (ok) {
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
      }
    }
    if (t >= 0 && (ok || nch == 0)) {
      if (nch == 0) {
        __nv_bfloat16* dst = out + ((long long)t * TC_HQ + h) * TC_DH;
        for (int i = 0; i < TC_DH; i += 8) *reinterpret_cast<uint4*>(dst + i) = make_uint4(0u, 0u, 0u, 0u);
      }
      if (lse != nullptr)
        lse[(long long)t * TC_HQ + h] = l > 0.f ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
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
  tc_attn_kernel<<<n_groups, TC_THREADS, TcSmem::SMEM, st>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)kc, (const __nv_bfloat16*)vc, list, lmask, n_list, perm, n_q,
      cap, scale * 1.4426950408889634f, (__nv_bfloat16*)out, lse, status, budget);
  return cudaGetLastError();
}

}  // namespace sa
