// pool.cu -- block keys for the two-stage indexer, and a table filler.
//
// Block key of block b = mean of the dequantised index keys of its `block`
// keys (a block is scored by the mean of its keys: MoBA, as summarised in
// Latent Sparse Attention section 2.2; HISA's block-level coarse filter).
// The sum runs in fp64 in key order (every product e4m3 * fp32 scale is exact
// in fp64), is divided by the block size and rounded to fp32; the result is
// stored like any index key: e4m3 bytes with one fp32 scale per block
// (amax / 448, 1 for a zero block), so stage 1 runs the same FP8 indexer.
#include <cuda_fp8.h>

#include "sa_internal.h"

namespace sa {

__global__ void pool_blocks_kernel(const uint8_t* __restrict__ k, const float* __restrict__ k_scale, int block,
                                   uint8_t* __restrict__ blk, float* __restrict__ blk_scale) {
  // one CTA per block, one thread per dimension (d = blockDim.x = 128)
  __shared__ float red[4];
  const int b = blockIdx.x, j = threadIdx.x, d = blockDim.x;
  double acc = 0.0;
  for (int s = b * block; s < (b + 1) * block; ++s) {
    __nv_fp8_e4m3 v;
    v.__x = k[(long long)s * d + j];
    acc += (double)float(v) * (double)k_scale[s];
  }
  const float mean = __double2float_rn(acc / (double)block);
  float a = fabsf(mean);
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((j & 31) == 0) red[j >> 5] = a;
  __syncthreads();
  float amax = 0.f;
  for (int w = 0; w < (d + 31) / 32; ++w) amax = fmaxf(amax, red[w]);
  const float scale = (amax > 0.f) ? __fdiv_rn(amax, 448.0f) : 1.0f;
  blk[(long long)b * d + j] = (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(mean, scale), __NV_SATFINITE, __NV_E4M3);
  if (j == 0) blk_scale[b] = scale;
}

cudaError_t launch_pool_blocks(const uint8_t* k, const float* k_scale, int n_blocks, int block, uint8_t* blk,
                               float* blk_scale, cudaStream_t st) {
  if (n_blocks <= 0) return cudaSuccess;
  pool_blocks_kernel<<<n_blocks, 128, 0, st>>>(k, k_scale, block, blk, blk_scale);
  return cudaGetLastError();
}

// scores[i * ld + s] = -inf for q_pos0 + i < s < n_k (the invisible part of
// a causal score table that the indexer's tiles do not cover).
__global__ void fill_upper_kernel(float* scores, int n_q, int n_k, long long ld, int q_pos0) {
  const int i = blockIdx.y;
  const int first = q_pos0 + i + 1;
  for (long long s = first + (long long)blockIdx.x * blockDim.x + threadIdx.x; s < n_k;
       s += (long long)gridDim.x * blockDim.x)
    scores[(long long)i * ld + s] = -INFINITY;
}

cudaError_t launch_fill_upper(float* scores, int n_q, int n_k, long long ld, int q_pos0, cudaStream_t st) {
  if (n_q <= 0 || n_k <= 0) return cudaSuccess;
  const int gx = max(1, min(64, (n_k + 255) / 256));
  fill_upper_kernel<<<dim3(gx, n_q), 256, 0, st>>>(scores, n_q, n_k, ld, q_pos0);
  return cudaGetLastError();
}

}  // namespace sa
