// sa_api.cu -- the C ABI (include/sa.h): validation, workspace layout and
// the launch sequences of the sparse-attention hot path.
#include <cmath>
#include <cstring>

#include "sa_internal.h"

namespace sa {

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;   // resolved once; read-only afterwards
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool make_tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t rows,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr || rows == 0) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------ validation
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool idx_supported(const sa_indexer_in* in) {
  if (in->dtype == SA_FP8_E4M3) return in->d_idx == 128 && (in->n_heads == 64 || in->n_heads == 32);
  if (in->dtype == SA_BF16) return in->batch == 0 && in->d_idx == 32 && (in->n_heads == 4 || in->n_heads == 8);
  return false;
}

static sa_status check_indexer(const sa_indexer_in* in, bool decode) {
  if (in == nullptr) return SA_ERR_INVALID_ARGUMENT;
  if (in->n_q < 0 || in->n_k <= 0 || in->n_heads <= 0 || in->d_idx <= 0 || in->q_pos0 < 0)
    return SA_ERR_INVALID_ARGUMENT;
  if (decode != (in->batch > 0)) return SA_ERR_INVALID_ARGUMENT;
  if (decode && in->n_q != in->batch) return SA_ERR_INVALID_ARGUMENT;
  if (in->n_q > 0 && (in->q == nullptr || in->k == nullptr || in->w == nullptr)) return SA_ERR_INVALID_ARGUMENT;
  if (in->dtype == SA_FP8_E4M3 && in->n_q > 0 && (in->q_scale == nullptr || in->k_scale == nullptr))
    return SA_ERR_INVALID_ARGUMENT;
  if (!aligned16(in->q) || !aligned16(in->k)) return SA_ERR_INVALID_ARGUMENT;
  if (in->d_idx % 32 != 0 || in->d_idx > 128) return SA_ERR_INVALID_ARGUMENT;
  if (!idx_supported(in)) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

static sa_status check_attn(const sa_attn_in* at, bool decode) {
  if (at == nullptr) return SA_ERR_INVALID_ARGUMENT;
  if (at->n_q < 0 || at->n_k <= 0) return SA_ERR_INVALID_ARGUMENT;
  if (decode != (at->batch > 0)) return SA_ERR_INVALID_ARGUMENT;
  if (decode && at->n_q != at->batch) return SA_ERR_INVALID_ARGUMENT;
  if (at->n_q > 0 && (at->q == nullptr || at->k_cache == nullptr || at->v_cache == nullptr))
    return SA_ERR_INVALID_ARGUMENT;
  if (!aligned16(at->q) || !aligned16(at->k_cache) || !aligned16(at->v_cache)) return SA_ERR_INVALID_ARGUMENT;
  if (!(at->head_dim == 64 || at->head_dim == 128)) return SA_ERR_UNSUPPORTED;
  if (!(at->n_q_heads == 16 || at->n_q_heads == 8)) return SA_ERR_UNSUPPORTED;
  if (!(at->softmax_scale >= 0.f) || std::isinf(at->softmax_scale)) return SA_ERR_INVALID_ARGUMENT;
  return SA_OK;
}

static float attn_scale(const sa_attn_in* at) {
  return at->softmax_scale > 0.f ? at->softmax_scale : 1.0f / std::sqrt((float)at->head_dim);
}

static sa_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SA_OK;
  if (e == cudaErrorNotSupported) return SA_ERR_UNSUPPORTED;
  return SA_ERR_CUDA;
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr long long kWaitBudget = 4000000000ll;     // ~2 s of SM clock
constexpr long long kHookBudget = 20000000ll;       // ~10 ms: the stall hook
#ifndef SA_DECODE_SPLIT_KEYS
#define SA_DECODE_SPLIT_KEYS 256
#endif
constexpr int kDecodeSplitKeys = SA_DECODE_SPLIT_KEYS;   // keys per decode attention split
constexpr int kDecodeTilesPerCta = 64;              // 8192 keys per decode indexer CTA
constexpr int kDecodeSamples = 8192;                // sampled scores per sequence for the decode threshold
constexpr int kMaxBlocks = 16384;                   // two-stage: blocks per sequence

static int decode_splits(int k) { return std::max(1, (k + kDecodeSplitKeys - 1) / kDecodeSplitKeys); }

// ------------------------------------------------------------ workspace plans
struct PrefillPlan {
  int R;           // rows per chunk
  int nb;          // two-stage: complete blocks
  bool stream;     // FLAT without a score table
  int m, n_s, cap, fb;   // stream: sample stride and count, list capacity, fallback rows per batch
  size_t off_table, off_idx, off_blk, off_blks, off_bsc, off_kept, off_cand, off_perm, total;
  size_t off_sel, off_ulist, off_umask, off_unl;   // two-stage: group union lists
  size_t off_gbn, off_gbblk, off_gbslot;            // two-stage: group unions of kept blocks
  size_t off_perm2;                                 // two-stage: attention groups (from the selections)
  size_t off_sig;                                   // two-stage: grouping signatures
  int n_groups, ucap;
  size_t off_ks, off_kss, off_stab, off_theta, off_cnt, off_list, off_miss, off_rows, off_count, off_pos;
  size_t off_ftab;
};

constexpr int kStreamSamples = 16384;      // sampled keys per row for the threshold (at most)
constexpr float kStreamGamma = 2.0f;       // target list length = gamma * k
constexpr int kTableMaxKeys = 65536;       // FLAT auto: table path up to this many keys
constexpr int kStreamPhases = 4;           // streaming scan: key phases (running threshold between them) ...
constexpr int kStreamPhaseTilesMin = 2048; // ... of at least this many 128-key tiles
constexpr int kUnionMaxKeys = 1 << 20;     // block bitmap of the group union kernel

static bool flat_streams(const sa_indexer_in* in, const sa_prefill_opts* o) {
  if (o->mode != SA_MODE_FLAT) return false;
  if (o->flat_path == SA_FLAT_STREAM) return true;
  if (o->flat_path == SA_FLAT_TABLE) return false;
  return in->n_k > kTableMaxKeys;
}

static bool plan_prefill(const sa_indexer_in* in, const sa_prefill_opts* o, PrefillPlan* p) {
  const long long nq = std::max(in->n_q, 1);
  int R = o->chunk_rows > 0 ? o->chunk_rows : 32768;
  R = (int)std::min<long long>(R, nq);
  std::memset(p, 0, sizeof(*p));
  size_t off = 0;
  if (o->mode == SA_MODE_FLAT && flat_streams(in, o)) {
    p->stream = true;
    p->m = std::max(1, (in->n_k + kStreamSamples - 1) / kStreamSamples);
    p->n_s = (in->n_k + p->m - 1) / p->m;
    p->cap = (4 * o->k + 63) / 64 * 64;
    if (o->chunk_rows <= 0) R = std::min(R, 16384);
    while (R > 1 && ((long long)R * p->n_s * 4ll > (2ll << 30) || (long long)R * p->cap * 8ll > (2ll << 30)))
      R = (R + 1) / 2;
    p->fb = (int)std::max<long long>(1, std::min<long long>(R, (1ll << 30) / ((long long)in->n_k * 4)));
    p->off_ks = off;
    off += align256((size_t)p->n_s * in->d_idx * (in->dtype == SA_FP8_E4M3 ? 1 : 2));
    p->off_kss = off;
    off += align256((size_t)p->n_s * 4);
    p->off_stab = off;
    off += align256((size_t)R * p->n_s * 4);
    p->off_theta = off;
    off += align256((size_t)R * 4);
    p->off_cnt = off;
    off += align256((size_t)R * 4);
    p->off_list = off;
    off += align256((size_t)R * p->cap * 8);
    p->off_miss = off;
    off += align256((size_t)R * 4);
    p->off_rows = off;
    off += align256((size_t)R * 4);
    p->off_count = off;
    off += 256;
    p->off_pos = off;
    off += align256((size_t)R * 4);
    p->off_ftab = off;
    off += align256((size_t)p->fb * in->n_k * 4);
  } else if (o->mode == SA_MODE_FLAT) {
    // score table of one chunk; shrink the chunk so the table stays <= 4 GiB
    while (R > 1 && (long long)R * in->n_k * 4ll > (4ll << 30)) R = (R + 1) / 2;
    p->off_table = off;
    off += align256((size_t)R * in->n_k * 4);
  } else {
    const int nb = in->n_k / o->block_size;
    p->nb = nb;
    p->off_blk = off;
    off += align256((size_t)std::max(nb, 1) * in->d_idx);
    p->off_blks = off;
    off += align256((size_t)std::max(nb, 1) * 4);
    p->off_bsc = off;
    off += align256((size_t)R * std::max(nb, 1) * 4);
    p->off_kept = off;
    off += align256((size_t)R * o->keep_blocks * 4);
    p->off_cand = off;
    off += align256((size_t)R * o->keep_blocks * o->block_size * 4);
    p->off_perm = off;
    off += align256((size_t)group_perm_len(R) * 4);
    p->off_perm2 = off;
    off += align256((size_t)group_perm_len(R) * 4);
    p->off_sig = off;
    off += align256((size_t)R * 8);
    // tensor-core attention of the groups' union lists
    p->n_groups = group_perm_len(R) / kGroupQueries;
    p->ucap = group_union_cap(o->k);
    p->off_sel = off;
    off += align256((size_t)R * o->keep_blocks * 2 * 4);
    p->off_ulist = off;
    off += align256((size_t)p->n_groups * p->ucap * 4);
    p->off_umask = off;
    off += align256((size_t)p->n_groups * p->ucap);
    p->off_gbn = off;
    off += align256((size_t)p->n_groups * 4);
    p->off_gbblk = off;
    off += align256((size_t)p->n_groups * group_blocks_cap() * 4);
    p->off_gbslot = off;
    off += align256((size_t)p->n_groups * group_blocks_cap() * 8);
    p->off_unl = off;
    off += align256((size_t)p->n_groups * 4);
  }
  p->off_idx = off;
  off += align256((size_t)R * o->k * 4);
  p->R = R;
  p->total = off;
  return true;
}

struct DecodePlan {
  size_t off_scores, off_idx, off_po, off_pl, total;
  size_t off_theta, off_cnt, off_list, off_miss;
  int splits, cap, m;
};

static void plan_decode(const sa_indexer_in* in, const sa_attn_in* at, int k, DecodePlan* p) {
  size_t off = 0;
  p->splits = decode_splits(k);
  p->cap = (4 * k + 63) / 64 * 64;
  p->m = std::max(1, (in->n_k + kDecodeSamples - 1) / kDecodeSamples);
  p->off_scores = off;
  off += align256((size_t)in->batch * in->n_k * 4);
  p->off_idx = off;
  off += align256((size_t)in->batch * k * 4);
  p->off_theta = off;
  off += align256((size_t)in->batch * 4);
  p->off_cnt = off;
  off += align256((size_t)in->batch * 4);
  p->off_list = off;
  off += align256((size_t)in->batch * p->cap * 8);
  p->off_miss = off;
  off += align256((size_t)in->batch * 4);
  p->off_po = off;
  off += align256((size_t)in->batch * p->splits * at->n_q_heads * at->head_dim * 4);
  p->off_pl = off;
  off += align256((size_t)in->batch * p->splits * at->n_q_heads * 4);
  p->total = off;
}

static size_t attn_ws(const sa_attn_in* at, int k) {
  if (at->batch == 0) return 0;
  const int sp = decode_splits(k);
  return align256((size_t)at->batch * sp * at->n_q_heads * at->head_dim * 4) +
         align256((size_t)at->batch * sp * at->n_q_heads * 4);
}

static IdxArgs base_args(const sa_indexer_in* in, uint32_t* status, int hook) {
  IdxArgs a;
  std::memset(&a, 0, sizeof(a));
  a.n_q = in->n_q;
  a.n_k = in->n_k;
  a.q_pos0 = in->q_pos0;
  a.div = 1;
  a.off = 0;
  a.q_scale = in->q_scale;
  a.k_scale = in->k_scale;
  a.w = in->w;
  a.seq_lens = in->seq_lens;
  a.status = status;
  a.budget = hook == SA_HOOK_STALL_WAIT ? kHookBudget : kWaitBudget;
  a.hook = hook;
  a.tile_lo = 0;
  a.tile_hi = 1 << 30;
  a.span = in->n_k;
  return a;
}

static size_t esize(sa_dtype d) { return d == SA_FP8_E4M3 ? 1 : 2; }

// Records stage_events[base + i] when the caller asked for them; base is the
// first event of the current chunk (chunk * (stages + 1)).
struct StageMarks {
  cudaEvent_t* ev;
  int n;
  int base = 0;
  bool ok = true;
  void mark(int i, cudaStream_t st) {
    if (ev != nullptr && base + i < n && cudaEventRecord(ev[base + i], st) != cudaSuccess) {
      (void)cudaGetLastError();   // do not let a bad event handle surface as a launch error
      ok = false;
    }
  }
};

// Streaming FLAT selection of one chunk (rows ci->q_pos0 ...): sampled
// thresholds, the appending scan, the exact list select, then the whole-row
// fallback for the rows whose list missed (queued on the device; no host
// synchronisation).
static sa_status stream_select_chunk(const sa_indexer_in* in, const sa_indexer_in* ci, const sa_prefill_opts* o,
                                     const PrefillPlan& p, char* w, bool first, int32_t* idx, uint32_t* status,
                                     cudaStream_t stream) {
  const int R = ci->n_q;
  const size_t esz = esize(in->dtype);
  const int krow = in->d_idx * (int)esz;
  uint8_t* ks = reinterpret_cast<uint8_t*>(w + p.off_ks);
  float* kss = reinterpret_cast<float*>(w + p.off_kss);
  float* stab = reinterpret_cast<float*>(w + p.off_stab);
  float* theta = reinterpret_cast<float*>(w + p.off_theta);
  int* cnt = reinterpret_cast<int*>(w + p.off_cnt);
  auto* list = reinterpret_cast<unsigned long long*>(w + p.off_list);
  int* miss = reinterpret_cast<int*>(w + p.off_miss);
  int* rows = reinterpret_cast<int*>(w + p.off_rows);
  int* count = reinterpret_cast<int*>(w + p.off_count);
  int* pos = reinterpret_cast<int*>(w + p.off_pos);
  cudaError_t e = cudaSuccess;
  if (first) {   // the sample: every m-th key (and its scale)
    e = launch_gather_rows(in->k, ks, nullptr, p.n_s, krow, p.m, krow, stream);
    if (e == cudaSuccess && in->k_scale)
      e = launch_gather_rows(in->k_scale, kss, nullptr, p.n_s, 4, p.m, 4, stream);
    if (e != cudaSuccess) return cuda_status(e);
  }
  // 1. sample scores: sample i (key m*i) is visible to row t iff m*i <= p
  {
    sa_indexer_in si = *ci;
    si.n_k = p.n_s;
    si.k = ks;
    si.k_scale = in->k_scale ? kss : nullptr;
    IdxArgs a = base_args(&si, status, o->test_hook);
    a.div = p.m;
    a.off = 0;
    a.out = stab;
    a.ld = p.n_s;
    e = launch_indexer(IDX_PREFILL, in->n_heads, in->d_idx, in->dtype, ci->q, ks, R, p.n_s, a, stream);
    if (e != cudaSuccess) return cuda_status(e);
  }
  // 2. thresholds
  e = launch_theta(stab, R, p.n_s, p.n_s, ci->q_pos0, p.m, in->n_k, o->k, p.cap, kStreamGamma, o->test_hook, theta,
                   stream);
  if (e != cudaSuccess) return cuda_status(e);
  // 3. the scan appends candidates, in key phases; between phases each list
  // holding more than k keys is cut to its k best and its threshold raised
  // to the k-th (a running threshold: later phases list fewer keys)
  if (cudaMemsetAsync(cnt, 0, (size_t)R * 4, stream) != cudaSuccess) return SA_ERR_CUDA;
  {
    const int n_tiles = (ci->q_pos0 + R - 1) / 128 + 1;            // key tiles the chunk's last row sees
    int per = (n_tiles + kStreamPhases - 1) / kStreamPhases;
    per = std::max(per, std::min(n_tiles, kStreamPhaseTilesMin));
    if (o->test_hook == SA_HOOK_THETA_RUNNING) per = std::max(1, (p.cap - o->k) / 128);
    for (int lo = 0; lo < n_tiles; lo += per) {
      IdxArgs a = base_args(ci, status, o->test_hook);
      a.theta = theta;
      a.cand = list;
      a.cand_cnt = cnt;
      a.cap = p.cap;
      a.tile_lo = lo;
      a.tile_hi = std::min(n_tiles, lo + per);
      e = launch_indexer(IDX_PREFILL, in->n_heads, in->d_idx, in->dtype, ci->q, in->k, R, in->n_k, a, stream);
      if (e == cudaSuccess && lo + per < n_tiles) e = launch_raise_theta(list, cnt, theta, R, p.cap, o->k, stream);
      if (e != cudaSuccess) return cuda_status(e);
    }
  }
  // 4. exact select of each list; flag the misses and queue them (ascending)
  e = launch_select_cand(list, cnt, theta, R, p.cap, ci->q_pos0, in->n_k, o->k, idx, miss, status, stream);
  if (e == cudaSuccess) e = launch_compact_rows(miss, R, rows, count, ci->q_pos0, pos, stream);
  if (e != cudaSuccess) return cuda_status(e);
  // 5. whole-row fallback of the queued rows, in batches of p.fb sized for
  // the worst case (every row of the chunk); the kernels read the queue's
  // length on the device and skip the rows past it, so the host never waits
  // for the count (the call stays stream-ordered and can be captured)
  float* ftab = reinterpret_cast<float*>(w + p.off_ftab);
  for (int b0 = 0; b0 < R; b0 += p.fb) {
    const int nb = std::min(p.fb, R - b0);
    sa_indexer_in fi = *ci;
    fi.n_q = nb;
    IdxArgs a = base_args(&fi, status, o->test_hook);
    a.row_pos = pos + b0;
    a.q_rows = rows + b0;
    a.row_count = count;
    a.row_base = b0;
    a.out = ftab;
    a.ld = in->n_k;
    e = launch_indexer(IDX_PREFILL, in->n_heads, in->d_idx, in->dtype, ci->q, in->k, R, in->n_k, a, stream);
    if (e == cudaSuccess)
      e = launch_topk_table(ftab, nb, in->n_k, in->n_k, 0, o->k, idx, 0, nullptr, 0, nullptr, stream, pos + b0,
                            rows + b0, nullptr, count, b0);
    if (e != cudaSuccess) return cuda_status(e);
  }
  return SA_OK;
}

}  // namespace sa

using namespace sa;

extern "C" {

const char* sa_status_string(sa_status s) {
  switch (s) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARGUMENT: return "SA_ERR_INVALID_ARGUMENT";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
    case SA_ERR_WORKSPACE_TOO_SMALL: return "SA_ERR_WORKSPACE_TOO_SMALL";
    case SA_ERR_CUDA: return "SA_ERR_CUDA";
    case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT";
    case SA_ERR_INTERNAL: return "SA_ERR_INTERNAL";
  }
  return "SA_ERR_UNKNOWN";
}

sa_status sa_workspace_size(sa_op op, const sa_indexer_in* in, const sa_attn_in* at, const void* opts,
                            size_t* bytes) {
  if (bytes == nullptr) return SA_ERR_INVALID_ARGUMENT;
  *bytes = 0;
  switch (op) {
    case SA_OP_INDEX_SCORES:
    case SA_OP_TOPK:
      return SA_OK;
    case SA_OP_SPARSE_ATTN: {
      if (at == nullptr || opts == nullptr) return SA_ERR_INVALID_ARGUMENT;
      *bytes = attn_ws(at, *static_cast<const int32_t*>(opts));
      return SA_OK;
    }
    case SA_OP_PREFILL: {
      if (in == nullptr || opts == nullptr) return SA_ERR_INVALID_ARGUMENT;
      const sa_prefill_opts* o = static_cast<const sa_prefill_opts*>(opts);
      if (o->k <= 0 || o->block_size <= 0 || o->keep_blocks <= 0) return SA_ERR_INVALID_ARGUMENT;
      PrefillPlan p;
      plan_prefill(in, o, &p);
      *bytes = p.total;
      return SA_OK;
    }
    case SA_OP_DECODE: {
      if (in == nullptr || at == nullptr || opts == nullptr) return SA_ERR_INVALID_ARGUMENT;
      const sa_decode_opts* o = static_cast<const sa_decode_opts*>(opts);
      if (o->k <= 0 || in->batch <= 0) return SA_ERR_INVALID_ARGUMENT;
      DecodePlan p;
      plan_decode(in, at, o->k, &p);
      *bytes = p.total;
      return SA_OK;
    }
  }
  return SA_ERR_INVALID_ARGUMENT;
}

sa_status sa_prefill_chunk_rows(const sa_indexer_in* in, const sa_prefill_opts* o, int32_t* rows) {
  if (in == nullptr || o == nullptr || rows == nullptr) return SA_ERR_INVALID_ARGUMENT;
  if (o->k <= 0 || o->block_size <= 0 || o->keep_blocks <= 0 || in->n_q < 0 || in->n_k <= 0)
    return SA_ERR_INVALID_ARGUMENT;
  PrefillPlan p;
  plan_prefill(in, o, &p);
  *rows = p.R;
  return SA_OK;
}

sa_status sa_index_scores(const sa_indexer_in* in, float* scores, int64_t ld, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
  (void)ws;
  (void)ws_bytes;
  sa_status s = check_indexer(in, false);
  if (s != SA_OK) return s;
  if (scores == nullptr || ld < in->n_k) return SA_ERR_INVALID_ARGUMENT;
  if (in->n_q == 0) return SA_OK;
  if ((long long)in->n_q * ld > (1ll << 34)) return SA_ERR_UNSUPPORTED;
  IdxArgs a = base_args(in, nullptr, 0);
  a.out = scores;
  a.ld = ld;
  cudaError_t e = launch_indexer(IDX_PREFILL, in->n_heads, in->d_idx, in->dtype, in->q, in->k, in->n_q, in->n_k, a,
                                 stream);
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(launch_fill_upper(scores, in->n_q, in->n_k, ld, in->q_pos0, stream));
}

sa_status sa_topk(const float* scores, int32_t n_q, int32_t n_k, int64_t ld, int32_t q_pos0, int32_t k,
                  int32_t* idx, void* ws, size_t ws_bytes, cudaStream_t stream) {
  (void)ws;
  (void)ws_bytes;
  if (n_q < 0 || n_k <= 0 || ld < n_k || q_pos0 < 0 || k <= 0) return SA_ERR_INVALID_ARGUMENT;
  if (n_q == 0) return SA_OK;
  if (scores == nullptr || idx == nullptr) return SA_ERR_INVALID_ARGUMENT;
  cudaError_t e = launch_topk_fast(scores, n_q, ld, n_k, q_pos0, nullptr, nullptr, 0, k, idx, stream);
  if (e == cudaErrorNotSupported)   // rows longer than one CTA holds in registers
    e = launch_topk_table(scores, n_q, n_k, ld, q_pos0, k, idx, 0, nullptr, 0, nullptr, stream);
  return cuda_status(e);
}

sa_status sa_sparse_attn(const sa_attn_in* at, const int32_t* idx, int32_t k, void* out, float* lse, void* ws,
                         size_t ws_bytes, cudaStream_t stream) {
  sa_status s = check_attn(at, at != nullptr && at->batch > 0);
  if (s != SA_OK) return s;
  if (k <= 0 || (at->n_q > 0 && (idx == nullptr || out == nullptr))) return SA_ERR_INVALID_ARGUMENT;
  if (at->n_q == 0) return SA_OK;
  const size_t need = attn_ws(at, k);
  if (ws_bytes < need || (need > 0 && ws == nullptr)) return SA_ERR_WORKSPACE_TOO_SMALL;
  int splits = 1;
  float *po = nullptr, *pl = nullptr;
  if (at->batch > 0) {
    splits = decode_splits(k);
    po = static_cast<float*>(ws);
    pl = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                  align256((size_t)at->batch * splits * at->n_q_heads * at->head_dim * 4));
  }
  return cuda_status(launch_attention(at->q, at->k_cache, at->v_cache, idx, at->n_q, k, at->n_k, at->n_q_heads,
                                      at->head_dim, attn_scale(at), at->batch, out, lse, po, pl, splits, stream));
}

sa_status sa_prefill(const sa_indexer_in* in, const sa_attn_in* at, const sa_prefill_opts* o, int32_t* idx_out,
                     void* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
  sa_status s = check_indexer(in, false);
  if (s != SA_OK) return s;
  s = check_attn(at, false);
  if (s != SA_OK) return s;
  if (o == nullptr || o->k <= 0 || o->k > 4096) return SA_ERR_INVALID_ARGUMENT;
  if (at->n_q != in->n_q || at->n_k != in->n_k || in->q_pos0 + (long long)in->n_q > in->n_k)
    return SA_ERR_INVALID_ARGUMENT;
  if (in->n_q > 0 && out == nullptr) return SA_ERR_INVALID_ARGUMENT;
  if (o->mode != SA_MODE_FLAT && o->mode != SA_MODE_TWO_STAGE) return SA_ERR_INVALID_ARGUMENT;
  if (o->mode == SA_MODE_TWO_STAGE) {
    if (o->block_size != 64) return SA_ERR_UNSUPPORTED;
    if (o->keep_blocks < 2 || o->keep_blocks > 64) return SA_ERR_INVALID_ARGUMENT;
    if (in->dtype != SA_FP8_E4M3) return SA_ERR_UNSUPPORTED;
    if ((in->q_pos0 + in->n_q - 1) / o->block_size >= kMaxBlocks) return SA_ERR_UNSUPPORTED;
  }
  const int n_stages = o->mode == SA_MODE_FLAT ? SA_PREFILL_FLAT_STAGES : SA_PREFILL_TWO_STAGE_STAGES;
  if (o->stage_events != nullptr && o->n_stage_events < n_stages + 1) return SA_ERR_INVALID_ARGUMENT;
  if (in->n_q == 0) return SA_OK;
  PrefillPlan p;
  plan_prefill(in, o, &p);
  if (ws == nullptr || ws_bytes < p.total) return SA_ERR_WORKSPACE_TOO_SMALL;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return SA_ERR_INVALID_ARGUMENT;
  char* w = static_cast<char*>(ws);
  uint32_t* status = o->status ? reinterpret_cast<uint32_t*>(o->status) : nullptr;
  if (status && cudaMemsetAsync(status, 0, sizeof(sa_device_status), stream) != cudaSuccess) return SA_ERR_CUDA;
  const float scale = attn_scale(at);
  const size_t qrow = (size_t)in->n_heads * in->d_idx * esize(in->dtype);
  cudaError_t e = cudaSuccess;
  StageMarks sm{o->stage_events, o->n_stage_events};

  if (o->mode == SA_MODE_TWO_STAGE) {
    uint8_t* blk = reinterpret_cast<uint8_t*>(w + p.off_blk);
    float* blks = reinterpret_cast<float*>(w + p.off_blks);
    sm.mark(0, stream);
    e = launch_pool_blocks(static_cast<const uint8_t*>(in->k), in->k_scale, p.nb, o->block_size, blk, blks, stream);
    if (e != cudaSuccess) return cuda_status(e);
  }

  for (int r0 = 0; r0 < in->n_q; r0 += p.R) {
    const int R = std::min(p.R, in->n_q - r0);
    sa_indexer_in ci = *in;
    ci.n_q = R;
    ci.q_pos0 = in->q_pos0 + r0;
    ci.q = static_cast<const char*>(in->q) + (size_t)r0 * qrow;
    ci.q_scale = in->q_scale ? in->q_scale + (size_t)r0 * in->n_heads : nullptr;
    ci.w = in->w + (size_t)r0 * in->n_heads;
    int32_t* idx = idx_out ? idx_out + (size_t)r0 * o->k : reinterpret_cast<int32_t*>(w + p.off_idx);
    sm.base = (r0 / p.R) * (n_stages + 1);
    if (o->mode == SA_MODE_TWO_STAGE && r0 > 0) sm.mark(0, stream);   // pooling ran in the first chunk
    if (o->mode == SA_MODE_FLAT && p.stream) {
      sm.mark(0, stream);
      sa_status fs = stream_select_chunk(in, &ci, o, p, w, r0 == 0, idx, status, stream);
      if (fs != SA_OK) return fs;
      sm.mark(1, stream);
    } else if (o->mode == SA_MODE_FLAT) {
      float* table = reinterpret_cast<float*>(w + p.off_table);
      IdxArgs a = base_args(&ci, status, o->test_hook);
      a.out = table;
      a.ld = in->n_k;
      sm.mark(0, stream);
      e = launch_indexer(IDX_PREFILL, in->n_heads, in->d_idx, in->dtype, ci.q, in->k, R, in->n_k, a, stream);
      if (e != cudaSuccess) return cuda_status(e);
      sm.mark(1, stream);
      e = launch_topk_fast(table, R, in->n_k, in->n_k, ci.q_pos0, nullptr, nullptr, 0, o->k, idx, stream);
      if (e == cudaErrorNotSupported)
        e = launch_topk_table(table, R, in->n_k, in->n_k, ci.q_pos0, o->k, idx, 0, nullptr, 0, nullptr, stream);
      if (e != cudaSuccess) return cuda_status(e);
    } else {
      const uint8_t* blk = reinterpret_cast<const uint8_t*>(w + p.off_blk);
      const float* blks = reinterpret_cast<const float*>(w + p.off_blks);
      float* bsc = reinterpret_cast<float*>(w + p.off_bsc);
      int* kept = reinterpret_cast<int*>(w + p.off_kept);
      float* cand = reinterpret_cast<float*>(w + p.off_cand);
      const int ncand = o->keep_blocks * o->block_size;
      // stage 1: complete blocks b < floor(p / block) (the current block is forced)
      sm.mark(1, stream);
      if (p.nb > 0) {
        sa_indexer_in bi = ci;
        bi.n_k = p.nb;
        bi.k = blk;
        bi.k_scale = blks;
        IdxArgs a = base_args(&bi, status, o->test_hook);
        a.div = o->block_size;
        a.off = 1;
        a.out = bsc;
        a.ld = p.nb;
        e = launch_indexer(IDX_PREFILL, in->n_heads, in->d_idx, in->dtype, ci.q, blk, R, p.nb, a, stream);
        if (e != cudaSuccess) return cuda_status(e);
      }
      sm.mark(2, stream);
      e = launch_block_keep_warp(bsc, R, std::max(p.nb, 1), ci.q_pos0, o->block_size, o->keep_blocks, kept, stream);
      if (e == cudaErrorNotSupported)   // more blocks than a warp keeps in shared memory
        e = launch_block_select(bsc, R, p.nb, std::max(p.nb, 1), ci.q_pos0, o->block_size, o->keep_blocks, kept,
                                stream);
      if (e != cudaSuccess) return cuda_status(e);
      // groups of queries that keep the same blocks, and each group's union
      // of kept blocks (stage 2 scores a union block once for the group)
      int* perm = reinterpret_cast<int*>(w + p.off_perm);
      int* gbn = reinterpret_cast<int*>(w + p.off_gbn);
      int* gbblk = reinterpret_cast<int*>(w + p.off_gbblk);
      unsigned long long* gbslot = reinterpret_cast<unsigned long long*>(w + p.off_gbslot);
      unsigned long long* sig = reinterpret_cast<unsigned long long*>(w + p.off_sig);
      e = launch_group_queries(kept, o->keep_blocks, nullptr, 0, R, ci.q_pos0, o->block_size, sig, perm, stream);
      if (e != cudaSuccess) return cuda_status(e);
      const bool grouped = o->test_hook != SA_HOOK_ATTN_UNGROUPED && in->n_k <= kUnionMaxKeys;
      if (grouped) {
        e = launch_group_blocks(kept, o->keep_blocks, perm, group_perm_len(R), R, in->n_k, gbn, gbblk, gbslot,
                                stream);
        if (e != cudaSuccess) return cuda_status(e);
      }
      // stage 2: the visible keys of the kept blocks
      sm.mark(3, stream);
      IdxArgs a = base_args(&ci, status, o->test_hook);
      a.out = cand;
      a.ld = ncand;
      a.kept = kept;
      a.keep = o->keep_blocks;
      a.perm = perm;
      a.gb_n = gbn;
      a.gb_blk = gbblk;
      a.gb_slot = gbslot;
      a.gb_cap = group_blocks_cap();
      a.n_groups = p.n_groups;
      e = launch_indexer(grouped ? IDX_GROUPED : IDX_GATHER, in->n_heads, in->d_idx, in->dtype, ci.q, in->k, R,
                         in->n_k, a, stream);
      if (e != cudaSuccess) return cuda_status(e);
      sm.mark(4, stream);
      uint32_t* sel = reinterpret_cast<uint32_t*>(w + p.off_sel);
      e = launch_topk_fast(cand, R, ncand, ncand, 0, nullptr, kept, o->keep_blocks, o->k, idx, stream, sel);
      if (e != cudaSuccess) return cuda_status(e);   // keep_blocks <= 64: at most 4096 candidates
    }
    const void* qa = static_cast<const char*>(at->q) + (size_t)r0 * at->n_q_heads * at->head_dim * 2;
    void* oa = static_cast<char*>(out) + (size_t)r0 * at->n_q_heads * at->head_dim * 2;
    float* la = lse ? lse + (size_t)r0 * at->n_q_heads : nullptr;
    sm.mark(n_stages - 1, stream);
    // grouped attention: two-stage groups by kept blocks (tensor cores over
    // each group's union of keys), FLAT groups by query order
    const int* perm = o->mode == SA_MODE_TWO_STAGE ? reinterpret_cast<const int*>(w + p.off_perm) : nullptr;
    const bool ungrouped = o->test_hook == SA_HOOK_ATTN_UNGROUPED;
    if (o->mode == SA_MODE_TWO_STAGE && !ungrouped && tc_attention_supported(at->n_q_heads, at->head_dim) &&
        in->n_k <= kUnionMaxKeys) {
      int* list = reinterpret_cast<int*>(w + p.off_ulist);
      uint8_t* lmask = reinterpret_cast<uint8_t*>(w + p.off_umask);
      int* nlist = reinterpret_cast<int*>(w + p.off_unl);
      const int* kept = reinterpret_cast<const int*>(w + p.off_kept);
      const uint32_t* sel = reinterpret_cast<const uint32_t*>(w + p.off_sel);
      // attention groups: queries that draw most of their keys from the same
      // blocks (a block counts when at least half of its keys were selected)
      int* perm2 = reinterpret_cast<int*>(w + p.off_perm2);
      e = launch_group_queries(kept, o->keep_blocks, sel, o->block_size / 2, R, ci.q_pos0, o->block_size,
                               reinterpret_cast<unsigned long long*>(w + p.off_sig), perm2, stream);
      if (e != cudaSuccess) return cuda_status(e);
      e = launch_group_union(kept, o->keep_blocks, sel, perm2, group_perm_len(R), R, in->n_k, p.ucap, list, lmask,
                             nlist, stream);
      if (e != cudaSuccess) return cuda_status(e);
      e = launch_attention_tc(qa, at->k_cache, at->v_cache, list, lmask, nlist, perm2, p.n_groups, R, p.ucap, scale,
                              oa, la, status, o->test_hook == SA_HOOK_STALL_WAIT ? kHookBudget : kWaitBudget,
                              stream);
    } else {
      e = launch_attention_grouped(qa, at->k_cache, at->v_cache, idx, perm, group_perm_len(R), R, o->k, at->n_k,
                                   at->n_q_heads, at->head_dim, scale, oa, la, ungrouped, stream);
    }
    if (e != cudaSuccess) return cuda_status(e);
    sm.mark(n_stages, stream);
  }
  return sm.ok ? SA_OK : SA_ERR_INVALID_ARGUMENT;
}

sa_status sa_decode(const sa_indexer_in* in, const sa_attn_in* at, const sa_decode_opts* o, int32_t* idx_out,
                    void* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
  sa_status s = check_indexer(in, true);
  if (s != SA_OK) return s;
  s = check_attn(at, true);
  if (s != SA_OK) return s;
  if (o == nullptr || o->k <= 0 || o->k > 4096) return SA_ERR_INVALID_ARGUMENT;
  if (at->batch != in->batch || at->n_k != in->n_k || out == nullptr) return SA_ERR_INVALID_ARGUMENT;
  DecodePlan p;
  plan_decode(in, at, o->k, &p);
  if (ws == nullptr || ws_bytes < p.total) return SA_ERR_WORKSPACE_TOO_SMALL;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return SA_ERR_INVALID_ARGUMENT;
  if (o->stage_events != nullptr && o->n_stage_events < SA_DECODE_STAGES + 1) return SA_ERR_INVALID_ARGUMENT;
  if (o->max_len < 0) return SA_ERR_INVALID_ARGUMENT;
  const int span = o->max_len > 0 ? std::min(o->max_len, in->n_k) : in->n_k;   // keys per sequence the grids cover
  char* w = static_cast<char*>(ws);
  uint32_t* status = o->status ? reinterpret_cast<uint32_t*>(o->status) : nullptr;
  if (status && cudaMemsetAsync(status, 0, sizeof(sa_device_status), stream) != cudaSuccess) return SA_ERR_CUDA;
  StageMarks sm{o->stage_events, o->n_stage_events};
  float* rows = reinterpret_cast<float*>(w + p.off_scores);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(w + p.off_idx);
  IdxArgs a = base_args(in, status, o->test_hook);
  a.out = rows;
  a.ld = in->n_k;
  a.tiles_per_cta = kDecodeTilesPerCta;
  a.span = span;
  sm.mark(0, stream);
  cudaError_t e = launch_indexer(IDX_DECODE, in->n_heads, in->d_idx, in->dtype, in->q, in->k, in->batch,
                                 (long long)in->batch * in->n_k, a, stream);
  if (e != cudaSuccess) return cuda_status(e);
  // selection from the written rows (LSA appendix F.1, "Flat decode"): a
  // threshold from every m-th score, the scores at or above it listed, the
  // lists ranked exactly; a sequence whose list missed is re-selected from
  // its whole written row (device-side, no host synchronisation)
  sm.mark(1, stream);
  {
    float* theta = reinterpret_cast<float*>(w + p.off_theta);
    int* cnt = reinterpret_cast<int*>(w + p.off_cnt);
    auto* list = reinterpret_cast<unsigned long long*>(w + p.off_list);
    int* miss = reinterpret_cast<int*>(w + p.off_miss);
    // the selection kernels and the attention run as a chain of programmatic
    // dependent launches: each is launched while its predecessor runs and
    // waits for it on the device (the threshold kernel also empties the lists)
    e = launch_theta(rows, in->batch, 0, in->n_k, 0, p.m, span, o->k, p.cap, kStreamGamma, o->test_hook, theta,
                     stream, 1, in->seq_lens, cnt, true);
    if (e == cudaSuccess)
      e = launch_collect_cand(rows, in->batch, in->n_k, span, in->seq_lens, theta, list, cnt, p.cap, stream, true);
    if (e == cudaSuccess)
      e = launch_select_cand(list, cnt, theta, in->batch, p.cap, 0, span, o->k, idx, miss, status, stream, 1,
                             in->seq_lens, true);
    if (e == cudaSuccess)
      e = launch_topk_table(rows, in->batch, span, in->n_k, 0, o->k, idx, 1, nullptr, 0, in->seq_lens, stream,
                            nullptr, nullptr, miss, nullptr, 0, true);
    if (e != cudaSuccess) return cuda_status(e);
  }
  sm.mark(2, stream);
  e = launch_attention(at->q, at->k_cache, at->v_cache, idx, in->batch, o->k, at->n_k, at->n_q_heads, at->head_dim,
                       attn_scale(at), in->batch, out, lse, reinterpret_cast<float*>(w + p.off_po),
                       reinterpret_cast<float*>(w + p.off_pl), p.splits, stream, status, true);
  if (e != cudaSuccess) return cuda_status(e);
  sm.mark(3, stream);
  return sm.ok ? SA_OK : SA_ERR_INVALID_ARGUMENT;
}

}  // extern "C"

// ------------------------------------------------------------ debug build
#ifdef SA_DEBUG_CHECKS
namespace sa {
int dbg_read_attn(uint32_t* out, int reset);
int dbg_read_group(uint32_t* out, int reset);
int dbg_read_lsa(uint32_t* out, int reset);
int dbg_read_lsa_attn(uint32_t* out, int reset);
}  // namespace sa
#endif

extern "C" sa_status sa_debug_errors(uint32_t* out, int32_t reset) {
#ifdef SA_DEBUG_CHECKS
  if (out == nullptr) return SA_ERR_INVALID_ARGUMENT;
  int (*const readers[])(uint32_t*, int) = {sa::dbg_read_attn, sa::dbg_read_group, sa::dbg_read_lsa,
                                            sa::dbg_read_lsa_attn};
  uint32_t acc[4] = {0u, 0u, 0u, 0u};
  for (auto rd : readers) {
    uint32_t w[4];
    if (rd(w, reset) != 0) return SA_ERR_CUDA;
    if (acc[0] == 0u && w[0] != 0u) {
      acc[0] = w[0];
      acc[1] = w[1];
    }
    acc[2] += w[2];
  }
  std::memcpy(out, acc, sizeof(acc));
  return SA_OK;
#else
  (void)out;
  (void)reset;
  return SA_ERR_UNSUPPORTED;
#endif
}
