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
// The 16 query heads are exactly the M = 16 of mma.sync m16n8k16 (below the
// M >= 64 of tcgen05), so one gathered row serves all heads; the per-chunk
// math lives in attn_common.cuh. The CTA's warps merge their partial states
// through shared memory. Prefill over index sets that overlap between queries
// has a grouped kernel (group.cu) that gathers shared keys once.
// Decode splits a sequence's keys over several CTAs and merges their
// (O, lse) in a second kernel (flash-decoding style; the pages add a
// split-KV sparse decode kernel for context parallelism, appendix F.1).
#include <cuda_bf16.h>

#include "attn_common.cuh"
#include "debug.cuh"
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
constexpr int AT_STAGES = SA_AT_STAGES;

template <int HQ, int DH>
struct AtCfg {
  static constexpr int ROWB = DH * 2;                  // bytes per K or V row
  static constexpr int PITCH = ROWB + (SA_AT_LAYOUT == 0 ? 16 : 0);   // row pitch in shared memory
  static constexpr int STAGE_BYTES = 2 * AT_CHUNK * PITCH;
  static constexpr int WARP_BYTES = AT_STAGES * STAGE_BYTES;
  static constexpr int MERGE_BYTES = AT_WARPS * (16 * DH + 32) * 4;
  static constexpr int RING = AT_WARPS * WARP_BYTES > MERGE_BYTES ? AT_WARPS * WARP_BYTES : MERGE_BYTES;
  static constexpr int SMEM = RING;                    // + the index slice, appended at launch
};

// index slice per CTA (entries), rounded up to whole chunks
__host__ __device__ inline int at_slice(int k, int splits) {
  return ((k + splits - 1) / splits + AT_CHUNK - 1) / AT_CHUNK * AT_CHUNK;
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
  uint8_t* wbuf = at_smem + warp * C::WARP_BYTES;
  int* sidx = reinterpret_cast<int*>(at_smem + C::SMEM);     // this CTA's index slice

  const __nv_bfloat16* kbase = kc + (batch ? (long long)t * n_k * DH : 0ll);
  const __nv_bfloat16* vbase = vc + (batch ? (long long)t * n_k * DH : 0ll);
  const int32_t* irow = idx + (long long)t * k;
  pdl_launch_dependents();
  pdl_wait();                 // decode chain: the index rows come from the previous kernel

  // this CTA's slice of the index row, in chunks of 16, staged in shared
  // memory once (invalid entries become -1)
  const int per = at_slice(k, splits);
  const int j_lo = sp * per, j_hi = min(k, j_lo + per);
  const int nchunks = (j_hi > j_lo) ? (j_hi - j_lo + AT_CHUNK - 1) / AT_CHUNK : 0;
  for (int j = threadIdx.x; j < nchunks * AT_CHUNK; j += AT_WARPS * 32) {
    int s = (j_lo + j < j_hi) ? irow[j_lo + j] : -1;
    SA_DBG_CHECK(s < n_k, SA_DBG_ATTN_INDEX, s);
    sidx[j] = (s >= 0 && s < n_k) ? s : -1;
  }
  __syncthreads();
  (void)status;   // no spin-waits here: cp.async groups complete in hardware

  using W = AttnWarp<HQ, DH, SA_AT_LAYOUT>;
  uint32_t qa[W::KK][4];
  W::load_q(q, t, lane, qa);

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
      cp_async16(kdst + W::off(r, seg), kbase + off);
      cp_async16(vdst + W::off(r, seg), vbase + off);
    }
  };

  const int my_chunks = (nchunks > warp) ? (nchunks - warp + AT_WARPS - 1) / AT_WARPS : 0;
#pragma unroll
  for (int i = 0; i < AT_STAGES - 1; ++i) {
    if (i < my_chunks) issue(i, i);
    cp_async_commit();
  }

  float o[W::NT][4], m_r[2], l_r[2];
  W::init(o, m_r, l_r);

  for (int i = 0; i < my_chunks; ++i) {
    const int st = i % AT_STAGES;
    cp_async_wait<AT_STAGES - 2>();
    __syncwarp();
    const uint32_t kb = smem_u32(wbuf + st * C::STAGE_BYTES);
    const uint32_t vb = kb + AT_CHUNK * C::PITCH;
    const int* cidx = sidx + (warp + i * AT_WARPS) * AT_CHUNK;
    const uint32_t valid = __ballot_sync(0xffffffffu, lane < AT_CHUNK && cidx[lane & (AT_CHUNK - 1)] >= 0);
    W::step(qa, kb, vb, valid, lane, scale_log2, o, m_r, l_r);
    // refill the stage read one iteration ago (its ldmatrix reads are done)
    __syncwarp();
    if (i + AT_STAGES - 1 < my_chunks) issue(i + AT_STAGES - 1, (i + AT_STAGES - 1) % AT_STAGES);
    cp_async_commit();
  }
  cp_async_wait<0>();

  W::reduce_l(l_r);

  // ---- merge the warps through shared memory ----
  __syncthreads();
  W::to_slot(reinterpret_cast<float*>(at_smem) + warp * (16 * DH + 32), lane, o, m_r, l_r);
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
  pdl_wait();
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
                                 float* part_lse, int splits, uint32_t* status, cudaStream_t st, bool pdl) {
  using C = AtCfg<HQ, DH>;
  auto kern = sparse_attn_kernel<HQ, DH>;
  const int smem = C::SMEM + at_slice(k, splits) * 4;
  if (smem > 227 * 1024) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  const float scale_log2 = scale * 1.4426950408889634f;
  e = launch_k(kern, dim3(n_q, splits), dim3(AT_WARPS * 32), smem, st, pdl, (const __nv_bfloat16*)q,
               (const __nv_bfloat16*)kc, (const __nv_bfloat16*)vc, idx, n_q, k, n_k, scale_log2, batch,
               (__nv_bfloat16*)out, lse, part_o, part_lse, splits, status);
  if (e != cudaSuccess || splits == 1) return e;
  return launch_k(attn_combine_kernel<HQ, DH>, dim3(n_q * HQ), dim3(DH), 0, st, pdl, (const float*)part_o,
                  (const float*)part_lse, n_q, splits, (__nv_bfloat16*)out, lse);
}

cudaError_t launch_attention(const void* q, const void* kc, const void* vc, const int32_t* idx, int n_q, int k,
                             int n_k, int hq, int dh, float scale, int batch, void* out, float* lse, float* part_o,
                             float* part_lse, int splits, cudaStream_t st, uint32_t* status, bool pdl) {
  if (n_q <= 0) return cudaSuccess;
  if (hq == 16 && dh == 128)
    return launch_attn_t<16, 128>(q, kc, vc, idx, n_q, k, n_k, scale, batch, out, lse, part_o, part_lse, splits,
                                  status, st, pdl);
  if (hq == 8 && dh == 128)
    return launch_attn_t<8, 128>(q, kc, vc, idx, n_q, k, n_k, scale, batch, out, lse, part_o, part_lse, splits,
                                 status, st, pdl);
  if (hq == 16 && dh == 64)
    return launch_attn_t<16, 64>(q, kc, vc, idx, n_q, k, n_k, scale, batch, out, lse, part_o, part_lse, splits,
                                 status, st, pdl);
  if (hq == 8 && dh == 64)
    return launch_attn_t<8, 64>(q, kc, vc, idx, n_q, k, n_k, scale, batch, out, lse, part_o, part_lse, splits,
                                status, st, pdl);
  return cudaErrorNotSupported;
}

}  // namespace sa

namespace sa {
SA_DEBUG_UNIT(dbg_read_attn)
}  // namespace sa
