// attn.cu -- softmax attention over selected keys of one shared KV head.
//
// O[t,h] = sum_{s in J_t} softmax_s(scale * Q[t,h] . K[s]) V[s], one index
// set J_t shared by every query head (Latent Sparse Attention section 3.2;
// J_t rows of KV slots padded with -1, appendix F.1 "Attention kernels").
//
// Gather-bound, not MMA-bound: per selected key a 2 x head_dim bf16 row pair
// (512 B at head_dim 128) feeds 4 * 16 * 128 flops. Each warp runs its own
// ring of AT_STAGES chunks of 16 keys, gathered with 16-byte cp.async where
// each warp instruction moves whole rows (16 lanes per 256-byte row, so every
// L2 sector is fetched once; measured faster here than one bulk copy per row).
// Rows are padded by 16 bytes so the ldmatrix reads of 8 consecutive rows hit
// 8 different bank groups. The 16
// query heads are exactly the M = 16 of mma.sync m16n8k16 (below the M >= 64
// of tcgen05), so one gathered row serves all heads. Online softmax in fp32
// (base 2); the CTA's warps merge their partial states through shared memory.
// Decode splits a sequence's keys over several CTAs and merges their
// (O, lse) in a second kernel (flash-decoding style; the pages add a
// split-KV sparse decode kernel for context parallelism, appendix F.1).
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "sa_internal.h"

namespace sa {

// Tuning knobs (compile-time): warps per CTA, ring depth per warp, and the
// shared-memory row layout (0: rows padded by 16 bytes; 1: unpadded rows with
// the 16-byte segments XOR-swizzled by row).
#ifndef SA_AT_WARPS
#define SA_AT_WARPS 4
#endif
#ifndef SA_AT_STAGES
#define SA_AT_STAGES 3
#endif
#ifndef SA_AT_LAYOUT
#define SA_AT_LAYOUT 1
#endif
constexpr int AT_WARPS = SA_AT_WARPS;
constexpr int AT_CHUNK = 16;
constexpr int AT_STAGES = SA_AT_STAGES;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
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

template <int HQ, int DH>
struct AtCfg {
  static constexpr int ROWB = DH * 2;                  // bytes per K or V row
  static constexpr int PITCH = ROWB + (SA_AT_LAYOUT == 0 ? 16 : 0);   // row pitch in shared memory
  static constexpr int STAGE_BYTES = 2 * AT_CHUNK * PITCH;
  static constexpr int WARP_BYTES = AT_STAGES * STAGE_BYTES;
  static constexpr int NT = DH / 8;                    // O n-tiles
  static constexpr int KK = DH / 16;                   // k-steps of Q.K
  static constexpr int MERGE_BYTES = AT_WARPS * (16 * DH + 32) * 4;
  static constexpr int RING = AT_WARPS * WARP_BYTES > MERGE_BYTES ? AT_WARPS * WARP_BYTES : MERGE_BYTES;
  static constexpr int SMEM = RING;                    // + the index slice, appended at launch
};

// index slice per CTA (entries), rounded up to whole chunks
__host__ __device__ inline int at_slice(int k, int splits) {
  return ((k + splits - 1) / splits + AT_CHUNK - 1) / AT_CHUNK * AT_CHUNK;
}

// byte offset of 16-byte segment `seg` of row `row` inside a K or V chunk
template <int PITCH>
__device__ __forceinline__ uint32_t at_off(int row, int seg) {
  if constexpr (SA_AT_LAYOUT == 0) return (uint32_t)(row * PITCH + seg * 16);
  return (uint32_t)(row * PITCH + ((seg ^ (row & 7)) * 16));
}

template <int HQ, int DH>
__global__ void __launch_bounds__(AT_WARPS * 32)
    sparse_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                       const __nv_bfloat16* __restrict__ vc, const int32_t* __restrict__ idx, int n_q, int k, int n_k,
                       float scale_log2, int batch, __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                       float* __restrict__ part_o, float* __restrict__ part_lse, int splits, uint32_t* status) {
  using C = AtCfg<HQ, DH>;
  extern __shared__ __align__(128) uint8_t at_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x, sp = blockIdx.y;
  const int g = lane >> 2, c4 = lane & 3;
  uint8_t* wbuf = at_smem + warp * C::WARP_BYTES;
  int* sidx = reinterpret_cast<int*>(at_smem + C::SMEM);     // this CTA's index slice

  const __nv_bfloat16* kbase = kc + (batch ? (long long)t * n_k * DH : 0ll);
  const __nv_bfloat16* vbase = vc + (batch ? (long long)t * n_k * DH : 0ll);
  const int32_t* irow = idx + (long long)t * k;

  // this CTA's slice of the index row, in chunks of 16, staged in shared
  // memory once (invalid entries become -1)
  const int per = at_slice(k, splits);
  const int j_lo = sp * per, j_hi = min(k, j_lo + per);
  const int nchunks = (j_hi > j_lo) ? (j_hi - j_lo + AT_CHUNK - 1) / AT_CHUNK : 0;
  for (int j = threadIdx.x; j < nchunks * AT_CHUNK; j += AT_WARPS * 32) {
    int s = (j_lo + j < j_hi) ? irow[j_lo + j] : -1;
    sidx[j] = (s >= 0 && s < n_k) ? s : -1;
  }
  __syncthreads();
  (void)status;   // no spin-waits here: cp.async groups complete in hardware

  // Q fragments (rows = heads; rows >= HQ are zero)
  uint32_t qa[C::KK][4];
  {
    const __nv_bfloat16* qt = q + (long long)t * HQ * DH;
#pragma unroll
    for (int kk = 0; kk < C::KK; ++kk) {
      const int c0 = kk * 16 + 2 * c4;
      auto ld = [&](int r, int col) -> uint32_t {
        if (r >= HQ) return 0u;
        return *reinterpret_cast<const uint32_t*>(qt + r * DH + col);
      };
      qa[kk][0] = ld(g, c0);
      qa[kk][1] = ld(g + 8, c0);
      qa[kk][2] = ld(g, c0 + 8);
      qa[kk][3] = ld(g + 8, c0 + 8);
    }
  }

  // loader: 32 / SEGS rows per warp instruction, SEGS lanes per row; an
  // invalid key loads row 0 (finite data, masked out below)
  constexpr int SEGS = C::ROWB / 16;
  constexpr int RPI = 32 / SEGS;
  auto issue = [&](int chunk_local, int st) {
    const int chunk = warp + chunk_local * AT_WARPS;
    const int* cidx = sidx + chunk * AT_CHUNK;
    const uint32_t kdst = smem_u32(wbuf + st * C::STAGE_BYTES);
    const uint32_t vdst = kdst + AT_CHUNK * C::PITCH;
    const int seg = lane % SEGS;
#pragma unroll
    for (int i = 0; i < AT_CHUNK / RPI; ++i) {
      const int r = i * RPI + lane / SEGS;
      const int s = cidx[r];
      const long long off = (long long)(s >= 0 ? s : 0) * DH + seg * 8;
      cp_async16(kdst + at_off<C::PITCH>(r, seg), kbase + off);
      cp_async16(vdst + at_off<C::PITCH>(r, seg), vbase + off);
    }
  };

  const int my_chunks = (nchunks > warp) ? (nchunks - warp + AT_WARPS - 1) / AT_WARPS : 0;
#pragma unroll
  for (int i = 0; i < AT_STAGES - 1; ++i) {
    if (i < my_chunks) issue(i, i);
    cp_async_commit();
  }

  float o[C::NT][4];
#pragma unroll
  for (int n = 0; n < C::NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};

  for (int i = 0; i < my_chunks; ++i) {
    const int st = i % AT_STAGES;
    cp_async_wait<AT_STAGES - 2>();
    __syncwarp();
    const uint32_t kb = smem_u32(wbuf + st * C::STAGE_BYTES);
    const uint32_t vb = kb + AT_CHUNK * C::PITCH;
    const int* cidx = sidx + (warp + i * AT_WARPS) * AT_CHUNK;
    // S = Q K^T : two n-tiles of 8 keys, each split into two independent
    // accumulation chains over the head dimension
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    float s2[4] = {0.f, 0.f, 0.f, 0.f}, s3[4] = {0.f, 0.f, 0.f, 0.f};
    const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int kk = 0; kk < C::KK; ++kk) {
      const int key = (mi >> 1) * 8 + rr;
      const int col = (kk * 2 + (mi & 1)) * 16;
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kb + at_off<C::PITCH>(key, col / 16), b0, b1, b2, b3);
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
    const bool v0 = cidx[kc0] >= 0, v1 = cidx[kc0 + 1] >= 0, v8 = cidx[kc0 + 8] >= 0, v9 = cidx[kc0 + 9] >= 0;
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
      for (int n = 0; n < C::NT; ++n) {
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
    for (int n2 = 0; n2 < C::NT / 2; ++n2) {
      const int key = (mi & 1) * 8 + rr;
      const int col = (n2 * 2 + (mi >> 1)) * 16;
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vb + at_off<C::PITCH>(key, col / 16), b0, b1, b2, b3);
      mma16816(o[2 * n2], pa, b0, b1);
      mma16816(o[2 * n2 + 1], pa, b2, b3);
    }
    // refill the stage read one iteration ago (its ldmatrix reads are done)
    __syncwarp();
    if (i + AT_STAGES - 1 < my_chunks) issue(i + AT_STAGES - 1, (i + AT_STAGES - 1) % AT_STAGES);
    cp_async_commit();
  }
  cp_async_wait<0>();

  // quad-reduce l
  l_r[0] += __shfl_xor_sync(0xffffffffu, l_r[0], 1);
  l_r[0] += __shfl_xor_sync(0xffffffffu, l_r[0], 2);
  l_r[1] += __shfl_xor_sync(0xffffffffu, l_r[1], 1);
  l_r[1] += __shfl_xor_sync(0xffffffffu, l_r[1], 2);

  // ---- merge the warps through shared memory ----
  __syncthreads();
  float* mo = reinterpret_cast<float*>(at_smem) + warp * (16 * DH + 32);
#pragma unroll
  for (int n = 0; n < C::NT; ++n) {
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
  __syncthreads();
  const float* base = reinterpret_cast<const float*>(at_smem);
  for (int e = threadIdx.x; e < HQ * DH; e += AT_WARPS * 32) {
    const int h = e / DH, col = e % DH;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < AT_WARPS; ++w) M = fmaxf(M, base[w * (16 * DH + 32) + 16 * DH + h]);
    const float Ms = (M == -INFINITY) ? 0.f : M;
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < AT_WARPS; ++w) {
      const float* bw = base + w * (16 * DH + 32);
      const float f = exp2f(bw[16 * DH + h] - Ms);
      L += bw[16 * DH + 16 + h] * f;
      acc += bw[h * DH + col] * f;
    }
    const float ov = (L > 0.f) ? acc / L : 0.f;
    const float lv = (L > 0.f) ? (Ms + log2f(L)) * 0.69314718055994531f : -INFINITY;
    if (splits == 1) {
      out[((long long)t * HQ + h) * DH + col] = __float2bfloat16_rn(ov);
      if (lse != nullptr && col == 0) lse[(long long)t * HQ + h] = lv;
    } else {
      part_o[(((long long)t * splits + sp) * HQ + h) * DH + col] = ov;
      if (col == 0) part_lse[((long long)t * splits + sp) * HQ + h] = lv;
    }
  }
}

// merge of the splits: one CTA per (sequence, head), one thread per column
template <int HQ, int DH>
__global__ void __launch_bounds__(DH) attn_combine_kernel(const float* __restrict__ part_o,
                                                          const float* __restrict__ part_lse, int n_q, int splits,
                                                          __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  const int t = blockIdx.x / HQ, h = blockIdx.x % HQ, col = threadIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, part_lse[((long long)t * splits + s) * HQ + h]);
  float L = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const float f = __expf(part_lse[((long long)t * splits + s) * HQ + h] - M);
      L += f;
      acc += f * part_o[(((long long)t * splits + s) * HQ + h) * DH + col];
    }
  }
  out[((long long)t * HQ + h) * DH + col] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
  if (lse != nullptr && col == 0) lse[(long long)t * HQ + h] = (L > 0.f) ? M + logf(L) : -INFINITY;
}

template <int HQ, int DH>
static cudaError_t launch_attn_t(const void* q, const void* kc, const void* vc, const int32_t* idx, int n_q, int k,
                                 int n_k, float scale, int batch, void* out, float* lse, float* part_o,
                                 float* part_lse, int splits, uint32_t* status, cudaStream_t st) {
  using C = AtCfg<HQ, DH>;
  auto kern = sparse_attn_kernel<HQ, DH>;
  const int smem = C::SMEM + at_slice(k, splits) * 4;
  if (smem > 227 * 1024) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  const float scale_log2 = scale * 1.4426950408889634f;
  kern<<<dim3(n_q, splits), AT_WARPS * 32, smem, st>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)kc, (const __nv_bfloat16*)vc, idx, n_q, k, n_k, scale_log2,
      batch, (__nv_bfloat16*)out, lse, part_o, part_lse, splits, status);
  e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  attn_combine_kernel<HQ, DH><<<n_q * HQ, DH, 0, st>>>(part_o, part_lse, n_q, splits, (__nv_bfloat16*)out, lse);
  return cudaGetLastError();
}

cudaError_t launch_attention(const void* q, const void* kc, const void* vc, const int32_t* idx, int n_q, int k,
                             int n_k, int hq, int dh, float scale, int batch, void* out, float* lse, float* part_o,
                             float* part_lse, int splits, cudaStream_t st, uint32_t* status) {
  if (n_q <= 0) return cudaSuccess;
  if (hq == 16 && dh == 128)
    return launch_attn_t<16, 128>(q, kc, vc, idx, n_q, k, n_k, scale, batch, out, lse, part_o, part_lse, splits,
                                  status, st);
  if (hq == 8 && dh == 128)
    return launch_attn_t<8, 128>(q, kc, vc, idx, n_q, k, n_k, scale, batch, out, lse, part_o, part_lse, splits,
                                 status, st);
  if (hq == 16 && dh == 64)
    return launch_attn_t<16, 64>(q, kc, vc, idx, n_q, k, n_k, scale, batch, out, lse, part_o, part_lse, splits,
                                 status, st);
  if (hq == 8 && dh == 64)
    return launch_attn_t<8, 64>(q, kc, vc, idx, n_q, k, n_k, scale, batch, out, lse, part_o, part_lse, splits,
                                status, st);
  return cudaErrorNotSupported;
}

}  // namespace sa
