// expand.cu -- attention index rows with sinks and a local window around the
// selected keys.
//
// Served index sets combine a few attention-sink keys at the start of the
// sequence, a window of the most recent keys, and the k long-range keys the
// indexer selected (Latent Sparse Attention section 3.2). A selected key the
// sinks or the window already hold is skipped, so no key repeats. One warp per
// row: the sinks and the window are ranges, and the kept entries of the
// selected row are compacted in their order with ballots.
#include "sa_internal.h"

namespace sa {

__global__ void __launch_bounds__(256) expand_sinks_window_kernel(const int32_t* __restrict__ idx, int n_q, int k,
                                                                  int q_pos0, int n_sink, int n_window,
                                                                  int32_t* __restrict__ out) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= n_q) return;
  const long long width = (long long)n_sink + n_window + k;
  int32_t* o = out + (long long)t * width;
  const int p = q_pos0 + t;
  const int n_s = max(0, min(n_sink, p + 1));                  // sinks 0 .. n_s - 1
  const int w_lo = max(n_sink, p - n_window + 1);              // window w_lo .. p
  const int n_w = max(0, p - w_lo + 1);
  for (int i = lane; i < n_s; i += 32) o[i] = i;
  for (int i = lane; i < n_w; i += 32) o[n_s + i] = w_lo + i;
  int pos = n_s + n_w;
  const int32_t* row = idx + (long long)t * k;
  for (int j0 = 0; j0 < k; j0 += 32) {
    const int j = j0 + lane;
    const int s = j < k ? row[j] : -1;
    const bool keep = s >= 0 && s >= n_sink && s < w_lo;     // neither a sink nor in the window
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) o[pos + __popc(bal & ((1u << lane) - 1u))] = s;
    pos += __popc(bal);
  }
  for (long long i = pos + lane; i < width; i += 32) o[i] = -1;
}

}  // namespace sa

using namespace sa;

extern "C" sa_status sa_expand_sinks_window(const int32_t* idx, int32_t n_q, int32_t k, int32_t q_pos0,
                                            int32_t n_sink, int32_t n_window, int32_t* out, cudaStream_t stream) {
  if (n_q < 0 || k < 1 || n_sink < 0 || n_window < 0 || q_pos0 < 0) return SA_ERR_INVALID_ARGUMENT;
  if (n_q == 0) return SA_OK;
  if (idx == nullptr || out == nullptr) return SA_ERR_INVALID_ARGUMENT;
  expand_sinks_window_kernel<<<(n_q + 7) / 8, 256, 0, stream>>>(idx, n_q, k, q_pos0, n_sink, n_window, out);
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}
