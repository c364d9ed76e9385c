// sa_internal.h -- declarations shared by the library's translation units.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "sa.h"

namespace sa {

enum IdxMode { IDX_PREFILL = 0, IDX_DECODE = 1, IDX_GATHER = 2, IDX_GROUPED = 3 };

// Arguments of the indexer kernel (plain device pointers and sizes).
struct IdxArgs {
  int n_q;               // query rows (prefill / gather) or sequences (decode)
  int n_k;               // keys per sequence (table width for prefill)
  int q_pos0;            // absolute position of query row 0
  int div, off;          // key s visible to row t iff s <= (q_pos0 + t) / div - off
  const float* q_scale;  // [n_q, H] or null (bf16)
  const float* k_scale;  // [n_k] / [batch, n_k] or null
  const float* w;        // [n_q, H]
  float* out;            // score table (row stride ld)
  long long ld;
  const int* seq_lens;   // decode: [batch] or null (= n_k)
  int tiles_per_cta;     // decode: key tiles per CTA
  const int* kept;       // gather: [n_q, keep] kept block ids, ascending, -1 padded
  int keep;
  // grouped (two-stage stage 2 over groups of queries): the group's queries
  // (perm), and per group its union blocks (ascending) with every query's
  // slot of each (byte q of gb_slot; 0xFF: not kept), gb_cap entries per group
  const int* perm;
  const int* gb_n;
  const int* gb_blk;
  const unsigned long long* gb_slot;
  int gb_cap;
  int n_groups;
  uint32_t* status;      // device [error, site] or null
  long long budget;      // wait budget in clock cycles
  int hook;
  // prefill: absolute position of every query row (ascending), overriding
  // q_pos0 + t when non-null
  const int* row_pos;
  // prefill: query row t of this launch is row q_rows[t] of q (and of w,
  // q_scale) when non-null; rows t >= *row_count - row_base (a count on the
  // device) are skipped, so a launch sized for the worst case does only the
  // rows a previous kernel flagged
  const int* q_rows;
  const int* row_count;
  int row_base;
  // prefill: only the key tiles [tile_lo, tile_hi) of 128 keys are scored
  int tile_lo, tile_hi;
  // decode: keys per sequence the grid covers (<= n_k, the cache's row stride)
  int span;
  // candidate mode (prefill): instead of writing the table, append every
  // visible key with score >= theta[t] to row t's list as the packed key
  // (order-preserving score bits << 32 | ~key); counts may exceed cap
  const float* theta;
  unsigned long long* cand;
  int* cand_cnt;
  int cap;
};

// A kernel launch, with programmatic stream serialization when `pdl` is set
// (the kernel may then be launched before the previous one in the stream
// ends; it waits for it in pdl_wait()).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                     Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Host launchers (return cudaError_t of the launch). `pdl`: launched as a
// programmatic dependent of the previous kernel in the stream (decode chain).
cudaError_t launch_indexer(int mode, int heads, int d, sa_dtype dt, const void* q, const void* k, int q_rows,
                           long long k_rows, const IdxArgs& a, cudaStream_t st);

cudaError_t launch_topk_table(const float* scores, int n_rows, int n_cols, long long ld, int q_pos0, int k,
                              int32_t* idx, int vis_mode, const int* kept, int keep, const int* seq_lens,
                              cudaStream_t st, const int* row_pos = nullptr, const int* out_rows = nullptr,
                              const int* only_flagged = nullptr, const int* row_count = nullptr, int row_base = 0,
                              bool pdl = false);

// sel (gathered rows only, nullable): per row keep * 2 words, bit c of the
// row's bitmap set iff candidate column c was selected
cudaError_t launch_topk_fast(const float* scores, int n_rows, long long ld, int n_cols, int q_pos0, const int* row_pos,
                             const int* kept, int keep, int k, int32_t* idx, cudaStream_t st,
                             uint32_t* sel = nullptr);

// ---- streaming selector (stream.cu) ----
cudaError_t launch_gather_rows(const void* src, void* dst, const int* rows, int n_rows, long long src_stride,
                               int m_stride, int row_bytes, cudaStream_t st);
cudaError_t launch_theta(const float* stab, int n_rows, int n_s, long long ld, int q_pos0, int m, int n_k, int k,
                         int cap, float gamma, int hook, float* theta, cudaStream_t st, int decode = 0,
                         const int* seq_lens = nullptr, int* zero_cnt = nullptr, bool pdl = false);
cudaError_t launch_select_cand(const unsigned long long* cand, const int* cnt, const float* theta, int n_rows,
                               int cap, int q_pos0, int n_k, int k, int32_t* idx, int* miss_flag, uint32_t* status,
                               cudaStream_t st, int decode = 0, const int* seq_lens = nullptr, bool pdl = false);
cudaError_t launch_collect_cand(const float* rows, int batch, long long ld, int n_k, const int* seq_lens,
                                const float* theta, unsigned long long* cand, int* cnt, int cap, cudaStream_t st,
                                bool pdl = false);
// Running threshold between the key phases of the streaming scan: every
// row whose list holds more than k and at most cap entries keeps exactly its
// k best packed keys (compacted to the front, count = k), and its threshold
// rises to the score of the k-th.
cudaError_t launch_raise_theta(unsigned long long* cand, int* cnt, float* theta, int n_rows, int cap, int k,
                               cudaStream_t st);
cudaError_t launch_compact_rows(const int* flags, int n_rows, int* rows, int* count, int q_pos0, int* pos,
                                cudaStream_t st);

cudaError_t launch_block_select(const float* bscores, int n_q, int nb, long long ld, int q_pos0, int block,
                                int keep, int* kept, cudaStream_t st);

cudaError_t launch_block_keep_warp(const float* bscores, int n_q, long long ld, int q_pos0, int block, int keep,
                                   int* kept, cudaStream_t st);

cudaError_t launch_pool_blocks(const uint8_t* k, const float* k_scale, int n_blocks, int block,
                               uint8_t* blk, float* blk_scale, cudaStream_t st);

cudaError_t launch_attention(const void* q, const void* kc, const void* vc, const int32_t* idx, int n_q, int k,
                             int n_k, int hq, int dh, float scale, int batch, void* out, float* lse,
                             float* part_o, float* part_lse, int splits, cudaStream_t st,
                             uint32_t* status = nullptr, bool pdl = false);

// grouped prefill attention (group.cu): perm orders the queries so that runs
// of kGroupQueries share keys (nullptr: query order); n_perm = its length
constexpr int kGroupQueries = 8;
int group_perm_len(int n_q);
// sel (nullable): the top-k's selection bitmaps; with it only kept blocks
// holding at least min_sel selected keys enter the signature
// holding at least min_sel selected keys enter the signature; sig = [n_q] scratch
cudaError_t launch_group_queries(const int* kept, int keep, const uint32_t* sel, int min_sel, int n_q, int q_pos0,
                                 int block, unsigned long long* sig, int* perm, cudaStream_t st);
cudaError_t launch_attention_grouped(const void* q, const void* kc, const void* vc, const int32_t* idx,
                                     const int* perm, int n_perm, int n_q, int k, int n_k, int hq, int dh,
                                     float scale, void* out, float* lse, bool ungrouped, cudaStream_t st);

// union of the kept blocks of each group (ascending) with every query's slot
// of each union block; cap = entries per group (kGroupQueries * keep at most)
int group_blocks_cap();
cudaError_t launch_group_blocks(const int* kept, int keep, const int* perm, int n_perm, int n_q, int n_k, int* gb_n,
                                int* gb_blk, unsigned long long* gb_slot, cudaStream_t st);

// union of each group's index sets (two-stage rows: kept blocks + selection
// bitmaps) as ascending key lists padded (-1, mask 0) to whole chunks of
// kUnionChunk keys, with per-key masks of the group's queries; cap = list
// capacity per group (a multiple of kUnionChunk)
constexpr int kUnionChunk = 128;
int group_union_cap(int k);
cudaError_t launch_group_union(const int* kept, int keep, const uint32_t* sel, const int* perm, int n_perm, int n_q,
                               int n_k, int cap, int* list, uint8_t* lmask, int* n_list, cudaStream_t st);

// tcgen05 attention of the groups' union lists (attn_tc.cu), 16 heads x 128 dims
bool tc_attention_supported(int hq, int dh);
// perm[w * W + i] = the query of rank i in window w of W queries (W =
// group_window()) by the 64-bit key sig[t] (ascending), -1 past n_q
cudaError_t launch_group_sort(const unsigned long long* sig, int n_q, int* perm, cudaStream_t st);
int group_window();
cudaError_t launch_attention_tc(const void* q, const void* kc, const void* vc, const int* list, const uint8_t* lmask,
                                const int* n_list, const int* perm, int n_groups, int n_q, int cap, float scale,
                                void* out, float* lse, uint32_t* status, long long budget, cudaStream_t st);

cudaError_t launch_fill_upper(float* scores, int n_q, int n_k, long long ld, int q_pos0, cudaStream_t st);

// Encodes a 2-D TMA descriptor (rows x inner elements, row-major).
bool make_tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t rows,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw);

}  // namespace sa
