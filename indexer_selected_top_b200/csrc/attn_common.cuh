// attn_common.cuh -- the per-chunk math shared by the attention kernels.
//
// One warp holds the 16 query heads of one query as the M = 16 rows of
// mma.sync m16n8k16 and consumes 16 gathered keys at a time: S = Q K^T,
// base-2 online softmax in fp32, O += P V (Latent Sparse Attention section
// 3.2: every query head attends over the same selected keys). K and V chunks
// sit in shared memory as rows of DH bf16 whose 16-byte segments are either
// padded (LAYOUT 0) or XOR-swizzled by row (LAYOUT 1), so the ldmatrix reads
// of 8 consecutive rows hit 8 different bank groups.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

namespace sa {

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// every cp.async of this thread, committed to a group or not, has landed
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

constexpr int AT_CHUNK = 16;   // keys per mma step (the k of m16n8k16 in P V)

template <int HQ, int DH, int LAYOUT>
struct AttnWarp {
  static constexpr int ROWB = DH * 2;                  // bytes per K or V row
  static constexpr int PITCH = ROWB + (LAYOUT == 0 ? 16 : 0);
  static constexpr int SEGS = ROWB / 16;               // 16-byte segments per row
  static constexpr int NT = DH / 8;                    // O n-tiles
  static constexpr int KK = DH / 16;                   // k-steps of Q.K

  // byte offset of 16-byte segment `seg` of row `row` inside a K or V chunk
  static __device__ __forceinline__ uint32_t off(int row, int seg) {
    if constexpr (LAYOUT == 0) return (uint32_t)(row * PITCH + seg * 16);
    return (uint32_t)(row * PITCH + ((seg ^ (row & 7)) * 16));
  }

  // Q fragments of one query (rows = heads; rows >= HQ and t < 0 are zero)
  static __device__ __forceinline__ void load_q(const __nv_bfloat16* q, long long t, int lane,
                                                uint32_t (&qa)[KK][4]) {
    const int g = lane >> 2, c4 = lane & 3;
    const __nv_bfloat16* qt = q + (t < 0 ? 0ll : t) * HQ * DH;
#pragma unroll
    for (int kk = 0; kk < KK; ++kk) {
      const int c0 = kk * 16 + 2 * c4;
      auto ld = [&](int r, int col) -> uint32_t {
        if (r >= HQ || t < 0) return 0u;
        return *reinterpret_cast<const uint32_t*>(qt + r * DH + col);
      };
      qa[kk][0] = ld(g, c0);
      qa[kk][1] = ld(g + 8, c0);
      qa[kk][2] = ld(g, c0 + 8);
      qa[kk][3] = ld(g + 8, c0 + 8);
    }
  }

  // One chunk of 16 keys at shared addresses kb (K rows) and vb (V rows).
  // valid bit j: key j of the chunk belongs to this query; this lane only
  // reads bits 2*c4, 2*c4+1, 2*c4+8 and 2*c4+9 (its S columns).
  static __device__ __forceinline__ void step(const uint32_t (&qa)[KK][4], uint32_t kb, uint32_t vb, uint32_t valid,
                                              int lane, float scale_log2, float (&o)[NT][4], float (&m_r)[2],
                                              float (&l_r)[2]) {
    const int c4 = lane & 3;
    // S = Q K^T : two n-tiles of 8 keys, each split into two independent
    // accumulation chains over the head dimension
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    float s2[4] = {0.f, 0.f, 0.f, 0.f}, s3[4] = {0.f, 0.f, 0.f, 0.f};
    const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int kk = 0; kk < KK; ++kk) {
      const int key = (mi >> 1) * 8 + rr;
      const int col = (kk * 2 + (mi & 1)) * 16;
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kb + off(key, col / 16), b0, b1, b2, b3);
      if (kk & 1) {
        mma16816(s2, qa[kk], b0, b1);
        mma16816(s3, qa[kk], b2, b3);
      } else {
        mma16816(s0, qa[kk], b0, b1);
        mma16816(s1, qa[kk], b2, b3);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s0[e] += s2[e];
      s1[e] += s3[e];
    }
    // mask, scale to base-2 logits
    const int kc0 = 2 * c4;
    const bool v0 = (valid >> kc0) & 1u, v1 = (valid >> (kc0 + 1)) & 1u;
    const bool v8 = (valid >> (kc0 + 8)) & 1u, v9 = (valid >> (kc0 + 9)) & 1u;
    float x[8];
    x[0] = v0 ? s0[0] * scale_log2 : -INFINITY;
    x[1] = v1 ? s0[1] * scale_log2 : -INFINITY;
    x[2] = v0 ? s0[2] * scale_log2 : -INFINITY;
    x[3] = v1 ? s0[3] * scale_log2 : -INFINITY;
    x[4] = v8 ? s1[0] * scale_log2 : -INFINITY;
    x[5] = v9 ? s1[1] * scale_log2 : -INFINITY;
    x[6] = v8 ? s1[2] * scale_log2 : -INFINITY;
    x[7] = v9 ? s1[3] * scale_log2 : -INFINITY;
    float cm0 = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[4], x[5]));
    float cm1 = fmaxf(fmaxf(x[2], x[3]), fmaxf(x[6], x[7]));
    cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, 1));
    cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, 2));
    cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, 1));
    cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, 2));
    const float mn0 = fmaxf(m_r[0], cm0), mn1 = fmaxf(m_r[1], cm1);
    const float ms0 = (mn0 == -INFINITY) ? 0.f : mn0;
    const float ms1 = (mn1 == -INFINITY) ? 0.f : mn1;
    const float a0 = exp2f(m_r[0] - ms0), a1 = exp2f(m_r[1] - ms1);
    float p[8];
    p[0] = exp2f(x[0] - ms0);
    p[1] = exp2f(x[1] - ms0);
    p[2] = exp2f(x[2] - ms1);
    p[3] = exp2f(x[3] - ms1);
    p[4] = exp2f(x[4] - ms0);
    p[5] = exp2f(x[5] - ms0);
    p[6] = exp2f(x[6] - ms1);
    p[7] = exp2f(x[7] - ms1);
    l_r[0] = l_r[0] * a0 + ((p[0] + p[1]) + (p[4] + p[5]));
    l_r[1] = l_r[1] * a1 + ((p[2] + p[3]) + (p[6] + p[7]));
    m_r[0] = mn0;
    m_r[1] = mn1;
    if (__any_sync(0xffffffffu, a0 != 1.f || a1 != 1.f)) {   // the running max moved
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        o[n][0] *= a0;
        o[n][1] *= a0;
        o[n][2] *= a1;
        o[n][3] *= a1;
      }
    }
    uint32_t pa[4];
    pa[0] = pack_bf16(p[0], p[1]);
    pa[1] = pack_bf16(p[2], p[3]);
    pa[2] = pack_bf16(p[4], p[5]);
    pa[3] = pack_bf16(p[6], p[7]);
    // O += P V : V via transposed ldmatrix
#pragma unroll
    for (int n2 = 0; n2 < NT / 2; ++n2) {
      const int key = (mi & 1) * 8 + rr;
      const int col = (n2 * 2 + (mi >> 1)) * 16;
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vb + off(key, col / 16), b0, b1, b2, b3);
      mma16816(o[2 * n2], pa, b0, b1);
      mma16816(o[2 * n2 + 1], pa, b2, b3);
    }
  }

  static __device__ __forceinline__ void init(float (&o)[NT][4], float (&m_r)[2], float (&l_r)[2]) {
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    m_r[0] = m_r[1] = -INFINITY;
    l_r[0] = l_r[1] = 0.f;
  }

  // complete the row sums across the quad that shares a row
  static __device__ __forceinline__ void reduce_l(float (&l_r)[2]) {
    l_r[0] += __shfl_xor_sync(0xffffffffu, l_r[0], 1);
    l_r[0] += __shfl_xor_sync(0xffffffffu, l_r[0], 2);
    l_r[1] += __shfl_xor_sync(0xffffffffu, l_r[1], 1);
    l_r[1] += __shfl_xor_sync(0xffffffffu, l_r[1], 2);
  }

  // write one warp's state (after reduce_l) into a merge slot of 16 * DH + 32 floats
  static __device__ __forceinline__ void to_slot(float* mo, int lane, const float (&o)[NT][4], const float (&m_r)[2],
                                                 const float (&l_r)[2]) {
    const int g = lane >> 2, c4 = lane & 3;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int col = n * 8 + 2 * c4;
      mo[g * DH + col] = o[n][0];
      mo[g * DH + col + 1] = o[n][1];
      mo[(g + 8) * DH + col] = o[n][2];
      mo[(g + 8) * DH + col + 1] = o[n][3];
    }
    if (c4 == 0) {
      mo[16 * DH + g] = m_r[0];
      mo[16 * DH + g + 8] = m_r[1];
      mo[16 * DH + 16 + g] = l_r[0];
      mo[16 * DH + 16 + g + 8] = l_r[1];
    }
  }

  // final O (bf16) and lse (natural log) of one query from one warp's state
  // (after reduce_l); a query with no valid key gets O = 0 and lse = -inf
  static __device__ __forceinline__ void store(__nv_bfloat16* out_t, float* lse_t, int lane, const float (&o)[NT][4],
                                               const float (&m_r)[2], const float (&l_r)[2]) {
    const int g = lane >> 2, c4 = lane & 3;
    const float inv0 = l_r[0] > 0.f ? 1.f / l_r[0] : 0.f, inv1 = l_r[1] > 0.f ? 1.f / l_r[1] : 0.f;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int col = n * 8 + 2 * c4;
      if (g < HQ)
        *reinterpret_cast<__nv_bfloat162*>(out_t + g * DH + col) = __floats2bfloat162_rn(o[n][0] * inv0, o[n][1] * inv0);
      if (g + 8 < HQ)
        *reinterpret_cast<__nv_bfloat162*>(out_t + (g + 8) * DH + col) =
            __floats2bfloat162_rn(o[n][2] * inv1, o[n][3] * inv1);
    }
    if (lse_t != nullptr && c4 == 0) {
      const float ms0 = (m_r[0] == -INFINITY) ? 0.f : m_r[0], ms1 = (m_r[1] == -INFINITY) ? 0.f : m_r[1];
      if (g < HQ) lse_t[g] = l_r[0] > 0.f ? (ms0 + log2f(l_r[0])) * 0.69314718055994531f : -INFINITY;
      if (g + 8 < HQ) lse_t[g + 8] = l_r[1] > 0.f ? (ms1 + log2f(l_r[1])) * 0.69314718055994531f : -INFINITY;
    }
  }
};

}  // namespace sa
