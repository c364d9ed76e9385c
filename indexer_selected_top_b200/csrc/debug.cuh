// debug.cuh -- invariant checks of the debug build (compiled with
// -DSA_DEBUG_CHECKS; the release build compiles none of this).
//
// A failed check records an error in a word of device memory and the kernel
// carries on without the access the invariant guarded (it skips the key, or
// clamps the write): no trap, no assert, so the context stays usable and the
// host reads what went wrong after the call (sa_debug_errors). Each
// translation unit keeps its own word (device variables are not shared across
// units without relocatable device code); SA_DEBUG_UNIT(name) defines its host
// reader, and sa_debug_errors in sa_api.cu reads them all.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

// sites: which check failed (the record keeps the first site and its value)
#define SA_DBG_ATTN_INDEX 1          // attention index >= n_k (the key is skipped)
#define SA_DBG_GROUP_UNION 2         // a two-stage group's key union exceeds its list
#define SA_DBG_LSA_BUCKET 3          // an LSA top-p bucket the query cannot see
#define SA_DBG_LSA_KEY 4             // an LSA long-range key outside [0, position]
#define SA_DBG_LSA_FAR_UNION 5       // an LSA long-range union exceeds its list
#define SA_DBG_LSA_CLUSTER 6         // a bucket list entry outside its cluster block

#ifdef SA_DEBUG_CHECKS
namespace sa {
// [first site, its value, count of failed checks, 0]
static __device__ uint32_t sa_dbg_word[4];

static __device__ __noinline__ void sa_dbg_record(uint32_t site, uint32_t value) {
  if (atomicCAS(&sa_dbg_word[0], 0u, site) == 0u) sa_dbg_word[1] = value;
  atomicAdd(&sa_dbg_word[2], 1u);
}
}  // namespace sa
// records (site, value) when `ok` is false; the code around it already copes
// with the failure (skips the key, clamps the count), as in the release build
#define SA_DBG_CHECK(ok, site, value)                                   \
  do {                                                                  \
    if (!(ok)) sa::sa_dbg_record((site), (uint32_t)(value));            \
  } while (0)
// host reader of this unit's word (and reset when asked)
#define SA_DEBUG_UNIT(name)                                                                         \
  int name(uint32_t* out, int reset) {                                                              \
    if (cudaMemcpyFromSymbol(out, sa::sa_dbg_word, 4 * sizeof(uint32_t)) != cudaSuccess) return 1; \
    if (reset) {                                                                                    \
      const uint32_t z[4] = {0u, 0u, 0u, 0u};                                                       \
      if (cudaMemcpyToSymbol(sa::sa_dbg_word, z, sizeof(z)) != cudaSuccess) return 1;               \
    }                                                                                               \
    return 0;                                                                                       \
  }
#else
#define SA_DBG_CHECK(ok, site, value) \
  do {                                \
  } while (0)
#define SA_DEBUG_UNIT(name)
#endif
