// quant.cu -- per-row FP8 e4m3 encoding of index vectors on the device.
//
// The indexer reads its queries and keys as OCP FP8 e4m3 bytes with one fp32
// scale per row (Latent Sparse Attention section 2.1: a lower-precision
// indexer). A serving loop appends one index key per token at every decode
// step; this kernel encodes such rows where they are produced: scale =
// amax / 448 (1 for an all-zero row), bytes = e4m3(x / scale), rounding to
// nearest with ties to even and saturating at +-448 (the conversion
// intrinsic's SATFINITE mode). One warp per row.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "sa_internal.h"

namespace sa {

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const T* __restrict__ x, long long n_rows, int d,
                                                            uint8_t* __restrict__ out, float* __restrict__ scale) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const T* xr = x + row * d;
  float amax = 0.f;
  for (int i = lane; i < d; i += 32) amax = fmaxf(amax, fabsf(to_f32(xr[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  uint8_t* orow = out + row * d;
  for (int i = lane; i < d; i += 32)
    orow[i] = (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(to_f32(xr[i]), s), __NV_SATFINITE, __NV_E4M3);
  if (lane == 0) scale[row] = s;
}

}  // namespace sa

using namespace sa;

extern "C" sa_status sa_quantize_rows_e4m3(const void* x, sa_dtype dtype, int64_t n_rows, int32_t d, uint8_t* out,
                                           float* scale, cudaStream_t stream) {
  if (n_rows < 0 || d < 1 || d > 4096) return SA_ERR_INVALID_ARGUMENT;
  if (n_rows == 0) return SA_OK;
  if (x == nullptr || out == nullptr || scale == nullptr) return SA_ERR_INVALID_ARGUMENT;
  const long long blocks = (n_rows + 7) / 8;
  if (blocks > 0x7FFFFFFFll) return SA_ERR_INVALID_ARGUMENT;
  if (dtype == SA_F32)
    quantize_rows_kernel<float><<<(unsigned)blocks, 256, 0, stream>>>(static_cast<const float*>(x), n_rows, d, out,
                                                                      scale);
  else if (dtype == SA_BF16)
    quantize_rows_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), n_rows, d, out, scale);
  else
    return SA_ERR_UNSUPPORTED;
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}
