// noalloc.cu -- decode attention that needs no caller-provided workspace.
//
// sa_sparse_attn in decode mode splits each sequence's selected keys over
// several CTAs and merges their partial results; those partials normally live
// in the caller's workspace. Some callers cannot hand us any extra device
// memory: a plugin inside a serving engine that owns every device allocation
// and passes only input and output pointers, or a decode loop whose memory is
// fixed after start-up and which may not call the CUDA allocator (cudaMalloc
// and cudaFree can synchronise the device). For them this entry point keeps
// the partials in a fixed array compiled into the library.
#include <mutex>

#include "sa_internal.h"

namespace sa {

// Partial results of the split-K decode attention: normalised O per (sequence,
// split, head) and its log-sum-exp. Sized for batch * splits * heads *
// head_dim <= 2^21 floats (8 MiB) and batch * splits * heads <= 2^17.
constexpr size_t kNoAllocMaxPartialFloats = size_t(1) << 21;
constexpr size_t kNoAllocMaxLseFloats = size_t(1) << 17;

static __device__ __align__(256) float g_partials[kNoAllocMaxPartialFloats + kNoAllocMaxLseFloats];

// Device address of g_partials, looked up once per device. In host code the
// symbol name is only a host-side stand-in, so kernels must be given this
// address instead.
static std::mutex g_addr_mu;
static float* g_addr[64] = {nullptr};

static cudaError_t partials_address(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_addr_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_partials);
    if (e != cudaSuccess) return e;
    g_addr[dev] = static_cast<float*>(p);
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace sa

using namespace sa;

extern "C" sa_status sa_sparse_attn_decode_noalloc(const sa_attn_in* at, const int32_t* idx, int32_t k, void* out,
                                                   float* lse, cudaStream_t stream) {
  if (at == nullptr || at->batch <= 0 || at->n_q != at->batch || at->n_k <= 0) return SA_ERR_INVALID_ARGUMENT;
  if (k <= 0 || idx == nullptr || out == nullptr || at->q == nullptr || at->k_cache == nullptr ||
      at->v_cache == nullptr)
    return SA_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(at->q) & 15u) || (reinterpret_cast<uintptr_t>(at->k_cache) & 15u) ||
      (reinterpret_cast<uintptr_t>(at->v_cache) & 15u))
    return SA_ERR_INVALID_ARGUMENT;
  if (!(at->head_dim == 64 || at->head_dim == 128) || !(at->n_q_heads == 16 || at->n_q_heads == 8))
    return SA_ERR_UNSUPPORTED;
  if (!(at->softmax_scale >= 0.f) || at->softmax_scale > 3.0e38f) return SA_ERR_INVALID_ARGUMENT;
  // one split per 256 selected keys (the fixed array is sized for that)
  const int splits = (k + 255) / 256;
  const size_t n_part = (size_t)at->batch * splits * at->n_q_heads * at->head_dim;
  const size_t n_lse = (size_t)at->batch * splits * at->n_q_heads;
  if (n_part > kNoAllocMaxPartialFloats || n_lse > kNoAllocMaxLseFloats) return SA_ERR_WORKSPACE_TOO_SMALL;
  float* base = nullptr;
  if (partials_address(&base) != cudaSuccess) return SA_ERR_CUDA;
  const float scale = at->softmax_scale > 0.f ? at->softmax_scale : 1.0f / sqrtf((float)at->head_dim);
  // every (sequence, split, head) partial is written before the merge reads
  // it, so the array needs no clearing between calls
  const cudaError_t e = launch_attention(at->q, at->k_cache, at->v_cache, idx, at->batch, k, at->n_k, at->n_q_heads,
                                         at->head_dim, scale, at->batch, out, lse, base,
                                         base + kNoAllocMaxPartialFloats, splits, stream);
  if (e == cudaSuccess) return SA_OK;
  return e == cudaErrorNotSupported ? SA_ERR_UNSUPPORTED : SA_ERR_CUDA;
}
