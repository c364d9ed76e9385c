/*
 * sa.h -- C ABI of libsa: learned top-k sparse attention on B200 (sm_100a).
 *
 * The hot path has three stages (token sparse attention, "Latent Sparse
 * Attention", paperpeel 2610.42147, section 2 and 2.1):
 *   (1) indexer:   score(t,s) = sum_h w[t,h] * ReLU(q_idx[t,h] . k_idx[s]), s <= t
 *   (2) top-k:     the k visible keys of largest score (ties: lower key index)
 *   (3) attention: softmax attention over the selected keys of one shared KV
 *                  head, one index set shared by every query head (section 3.2)
 * plus an optional two-stage indexer that first keeps the best mean-pooled key
 * blocks and runs (1)-(2) only inside them (HISA, theflow "related" page;
 * block score by the mean of its keys, LSA section 2.2).
 *
 * Conventions (all calls):
 *  - Every pointer argument is DEVICE memory unless marked "host". The caller
 *    owns every buffer; the library never allocates, and never synchronises
 *    the host except where a call says so.
 *  - Tensors are row-major and contiguous; the innermost row of every index
 *    tensor (q_idx, k_idx) must start on a 16-byte boundary (TMA operand).
 *  - Calls are ordered on `stream` and reentrant; there is no global mutable
 *    state. Argument validation is synchronous and happens before any launch;
 *    a failed validation launches nothing.
 *  - Index rows ("J", appendix F.1 "Attention kernels") are int32 key
 *    positions (KV-cache slots) in UNSPECIFIED order, padded with -1 at the
 *    tail when fewer than k keys are visible. The attention does not depend on
 *    their order (appendix F.1, "Selection by threshold").
 *  - Errors: SA_ERR_INVALID_ARGUMENT (bad sizes, null pointers, misaligned
 *    rows), SA_ERR_UNSUPPORTED (a valid shape this build does not implement),
 *    SA_ERR_WORKSPACE_TOO_SMALL, SA_ERR_CUDA (a launch failed; the stream
 *    state is whatever CUDA reports), SA_ERR_TIMEOUT is reported only through
 *    the device status word (a bounded wait inside a kernel gave up).
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARGUMENT = 1,
  SA_ERR_UNSUPPORTED = 2,
  SA_ERR_WORKSPACE_TOO_SMALL = 3,
  SA_ERR_CUDA = 4,
  SA_ERR_TIMEOUT = 5,
  SA_ERR_INTERNAL = 6
} sa_status;

typedef enum {
  SA_BF16 = 0,      /* bfloat16 */
  SA_FP8_E4M3 = 1,  /* OCP e4m3 ("fn": no inf, 0x7F/0xFF NaN), one fp32 scale per row */
  SA_F32 = 2
} sa_dtype;

typedef enum { SA_MODE_FLAT = 0, SA_MODE_TWO_STAGE = 1 } sa_mode;

typedef enum {
  SA_OP_INDEX_SCORES = 0,
  SA_OP_TOPK = 1,
  SA_OP_SPARSE_ATTN = 2,
  SA_OP_PREFILL = 3,
  SA_OP_DECODE = 4
} sa_op;

/*
 * Indexer operands (stage 1 of the path; the lightweight indexer "with fewer
 * heads, smaller dimension, lower precision", LSA section 2.1).
 *
 * Prefill (batch == 0): query row i sits at absolute position q_pos0 + i and
 *   sees keys s <= q_pos0 + i, s < n_k.
 *     q        [n_q, n_heads, d_idx]  (fp8 bytes or bf16)
 *     q_scale  [n_q, n_heads] fp32    (fp8 only; NULL for bf16)
 *     k        [n_k, d_idx]
 *     k_scale  [n_k] fp32             (fp8 only; NULL for bf16)
 *     w        [n_q, n_heads] fp32    head weights, expected >= 0
 *   FP8 values are q_scale * e4m3(q) and k_scale * e4m3(k).
 * Decode (batch > 0): sequence b has ONE query (n_q must equal batch) and its
 *   own cache of capacity n_k keys; the query sees keys s < seq_lens[b]
 *   (its own key is the cache's last row).
 *     q [batch, n_heads, d_idx], q_scale [batch, n_heads], w [batch, n_heads]
 *     k [batch, n_k, d_idx], k_scale [batch, n_k]
 *     seq_lens [batch] int32 device, each in [1, n_k]; NULL means n_k for all.
 * Supported (else SA_ERR_UNSUPPORTED): fp8 with d_idx = 128 and n_heads in
 *            {32, 64}; bf16 with d_idx = 32 and n_heads in {4, 8} (prefill only).
 */
typedef struct {
  int32_t n_q;
  int32_t n_k;
  int32_t q_pos0;
  int32_t n_heads;
  int32_t d_idx;
  sa_dtype dtype;
  const void* q;
  const float* q_scale;
  const void* k;
  const float* k_scale;
  const float* w;
  int32_t batch;
  const int32_t* seq_lens;
} sa_indexer_in;

/*
 * Attention operands (stage 3): one shared KV head (MQA).
 *   q       [n_q, n_q_heads, head_dim] bf16
 *   k_cache [n_k, head_dim] bf16 (decode: [batch, n_k, head_dim])
 *   v_cache [n_k, head_dim] bf16 (decode: [batch, n_k, head_dim])
 *   head_dim in {64, 128}; n_q_heads in {8, 16}.
 *   softmax_scale: logits are scale * q . k; 0 means 1/sqrt(head_dim).
 */
typedef struct {
  int32_t n_q;
  int32_t n_k;
  int32_t n_q_heads;
  int32_t head_dim;
  float softmax_scale;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  int32_t batch;
} sa_attn_in;

/* Device-side status word, written by sa_prefill / sa_decode when non-NULL.
 * Read it after synchronising the stream. */
typedef struct {
  uint32_t error;          /* 0 = ok; SA_ERR_TIMEOUT if a bounded wait gave up */
  uint32_t timeout_site;   /* which wait gave up (diagnostic) */
  uint32_t fallback_rows;  /* rows re-selected from their whole score row */
  uint32_t overflow_rows;  /* rows whose candidate list overflowed */
} sa_device_status;

/* Optional stage timing: when stage_events is non-NULL the call records,
 * for every chunk c of its rows (sa_prefill_chunk_rows gives the chunk
 * size; decode has one chunk), stage_events[c * (n + 1) + i] on `stream`
 * before stage i of that chunk and stage_events[c * (n + 1) + n] after its
 * last stage. n_stage_events must be >= n + 1; chunks whose events lie past
 * n_stage_events are not recorded. The time of stage i summed over the
 * recorded chunks is then the sum of the elapsed times between events
 * c * (n + 1) + i and c * (n + 1) + i + 1.
 * Stages (n): FLAT = indexer, top-k, attention (3); TWO_STAGE = pooling,
 * stage-1 indexer, block keep, stage-2 indexer, top-k, attention (6);
 * decode = indexer, top-k, attention (3). The two-stage pooling runs once,
 * in the first chunk (later chunks record an empty pooling stage); the FLAT
 * path without a score table (SA_FLAT_STREAM) scores and selects inside its
 * indexer stage (its top-k stage is empty). Events are created by the
 * caller; an event that cannot be recorded makes the call return
 * SA_ERR_INVALID_ARGUMENT after its work has been queued. */
#define SA_PREFILL_FLAT_STAGES 3
#define SA_PREFILL_TWO_STAGE_STAGES 6
#define SA_DECODE_STAGES 3

typedef struct {
  int32_t k;             /* top-k budget, 1..4096 */
  sa_mode mode;          /* FLAT or TWO_STAGE */
  int32_t block_size;    /* two-stage key block (64) */
  int32_t keep_blocks;   /* two-stage kept blocks per query (>= 2, <= 64) */
  int32_t chunk_rows;    /* query rows per chunk (0 = library default) */
  sa_device_status* status;  /* device, nullable; zeroed by the call */
  int32_t test_hook;     /* 0 in production; see SA_HOOK_* */
  cudaEvent_t* stage_events;  /* host array, nullable (see above) */
  int32_t n_stage_events;
  int32_t flat_path;     /* FLAT mode: SA_FLAT_AUTO, SA_FLAT_TABLE or SA_FLAT_STREAM */
} sa_prefill_opts;

/* FLAT prefill paths. TABLE writes each chunk's score table and selects its
 * rows; STREAM never writes the table: a sampled threshold per row, the
 * indexer's epilogue appends the keys at or above it to the row's candidate
 * list (capacity 4k), an exact select ranks the list, and rows whose list
 * missed are re-selected from their whole row. AUTO takes TABLE while the
 * keys number at most 65536, STREAM beyond. */
#define SA_FLAT_AUTO 0
#define SA_FLAT_TABLE 1
#define SA_FLAT_STREAM 2

typedef struct {
  int32_t k;
  sa_device_status* status;  /* device, nullable; zeroed by the call */
  int32_t test_hook;
  cudaEvent_t* stage_events;  /* host array, nullable (see above) */
  int32_t n_stage_events;
  int32_t max_len;       /* 0, or the longest context this call serves (<= n_k): the kernels' grids cover
                            max_len keys per sequence instead of the cache's n_k, so a CUDA graph captured
                            for a context-length bucket does only that bucket's work; a sequence longer
                            than max_len sets status->error = SA_ERR_INVALID_ARGUMENT and is read up to
                            max_len only */
} sa_decode_opts;

/* test hooks: force the threshold of the streaming selector, a stalled wait,
 * or the per-query schedule of the grouped prefill attention */
#define SA_HOOK_NONE 0
#define SA_HOOK_THETA_POS_INF 1   /* every row misses low -> whole-row fallback */
#define SA_HOOK_THETA_NEG_INF 2   /* every key is a candidate -> overflow path */
#define SA_HOOK_STALL_WAIT 3      /* a device wait that never completes -> SA_ERR_TIMEOUT */
#define SA_HOOK_THETA_RUNNING 5    /* every threshold starts at -inf and the streaming scan runs in key phases of
                                     cap - k keys, so only the running threshold keeps the lists in bounds */
#define SA_HOOK_ATTN_UNGROUPED 4  /* no query groups: the two-stage stage 2 scores each query's kept blocks on
                                     its own and the prefill attention takes one query at a time, as for a
                                     group whose union of selected keys does not fit the kernel's tables */

/* Human-readable name of a status code (host, static storage). */
const char* sa_status_string(sa_status s);

/*
 * sa_index_scores: writes the causal indexer score table (stage 1).
 *   scores[i * ld + s] = score(q_pos0 + i, s) for s <= q_pos0 + i, -inf for
 *   the other s < n_k; columns >= n_k are not touched. ld >= n_k.
 * Prefill only (batch == 0). Needs no workspace (ws may be NULL, ws_bytes 0).
 * This is the pages' short-context path that writes S with one matrix product
 * (LSA appendix F.1, "Flat prefill": below 32,768 buckets S is written).
 * Returns SA_ERR_UNSUPPORTED if n_q * ld exceeds 2^34 entries.
 */
sa_status sa_index_scores(const sa_indexer_in* in, float* scores, int64_t ld,
                          void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * sa_topk: exact top-k of each row of a score table (stage 2).
 *   Row i considers columns s < min(n_k, q_pos0 + i + 1) and writes to
 *   idx[i * k ...] the min(k, that count) columns of largest score, ties to
 *   the lower column, in unspecified order, then -1 padding. Selection is the
 *   radix select over packed keys of LSA appendix F.1 (score bits above the
 *   inverted id). NaN scores order above +inf (by sign) and are not expected.
 * Workspace: none (ws may be NULL).
 */
sa_status sa_topk(const float* scores, int32_t n_q, int32_t n_k, int64_t ld, int32_t q_pos0,
                  int32_t k, int32_t* idx, void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * sa_sparse_attn: softmax attention over given index rows (stage 3).
 *   idx [n_q, k] int32 (decode: [batch, k], positions in that sequence's
 *   cache); entries < 0 are skipped, entries must be < n_k.
 *   out [n_q, n_q_heads, head_dim] bf16; lse [n_q, n_q_heads] fp32 (natural
 *   log, nullable). A row with no valid index gets out = 0, lse = -inf.
 * Workspace: sa_workspace_size(SA_OP_SPARSE_ATTN, ...) bytes (decode splits).
 */
sa_status sa_sparse_attn(const sa_attn_in* in, const int32_t* idx, int32_t k, void* out, float* lse,
                         void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * sa_prefill: the fused prefill path (indexer -> top-k -> attention).
 *   idx_out [n_q, k] int32 (nullable: then held in the workspace),
 *   out [n_q, n_q_heads, head_dim] bf16, lse [n_q, n_q_heads] fp32 (nullable).
 * FLAT: the token indexer over all visible keys. With a small table it writes
 *   S and selects rows (LSA appendix F.1, "Flat prefill", short context);
 *   above that it never writes S: each query keeps a threshold and a
 *   candidate list filled in the indexer's epilogue, then selects exactly
 *   (LSA appendix F.1, "Selection by threshold"; HyTopK's on-the-fly exact
 *   top-k). Rows whose list misses are re-selected from their whole row.
 * TWO_STAGE: block keys = mean of each block's dequantised keys (stored as
 *   e4m3 with one scale per block); stage 1 scores complete blocks b <
 *   floor(p / block_size) and keeps block 0, the current block and the best
 *   keep_blocks - 2 others; stage 2 scores the visible keys of the kept
 *   blocks; then top-k and attention. The two-stage path schedules its
 *   queries in groups of 8 that keep (stage 2) or select (attention) mostly
 *   the same keys, so a group's keys are loaded once; every query's scores,
 *   selection and attention are its own, whatever its group.
 * Requires in->n_k == n_k of attn, q_pos0 + n_q <= n_k.
 * No host synchronisation and no allocation in any mode: the rows whose
 * candidate list missed are queued on the device and re-selected from their
 * whole rows by kernels sized for the chunk's worst case that skip the rows
 * past the queue's length, so the call is stream-ordered throughout and can
 * be captured in a CUDA graph.
 */
sa_status sa_prefill(const sa_indexer_in* in, const sa_attn_in* attn, const sa_prefill_opts* opts,
                     int32_t* idx_out, void* out, float* lse, void* ws, size_t ws_bytes,
                     cudaStream_t stream);

/*
 * sa_decode: one decode step for `batch` sequences (one new query each).
 *   in->batch == attn->batch > 0. Keys visible to sequence b: s < seq_lens[b].
 *   idx_out [batch, k] int32 (nullable), out [batch, n_q_heads, head_dim]
 *   bf16, lse [batch, n_q_heads] (nullable).
 * No host synchronisation and no allocation: the call can be captured in a
 * CUDA graph (shapes are fixed by n_k; seq_lens are read on the device).
 */
sa_status sa_decode(const sa_indexer_in* in, const sa_attn_in* attn, const sa_decode_opts* opts,
                    int32_t* idx_out, void* out, float* lse, void* ws, size_t ws_bytes,
                    cudaStream_t stream);

/*
 * sa_sparse_attn_decode_noalloc: the decode form of sa_sparse_attn (batch >
 * 0) for callers that cannot provide device workspace -- for example a plugin
 * in a serving engine that owns all device memory and passes only inputs and
 * outputs, or a decode loop whose memory is fixed after start-up and which
 * must not call the CUDA allocator (cudaMalloc / cudaFree may synchronise the
 * device). The pages have no counterpart; this is a deployment convenience.
 *   Arguments and results as sa_sparse_attn with batch > 0, without ws.
 *   The per-split partial results live in one fixed array inside the library
 *   (8 MiB + 512 KiB of device memory on every GPU that loads it, held until
 *   the process exits): batch * ceil(k / 256) * n_q_heads * head_dim must be
 *   <= 2^21 and batch * ceil(k / 256) * n_q_heads <= 2^17, otherwise the call
 *   returns SA_ERR_WORKSPACE_TOO_SMALL and launches nothing (64 sequences x
 *   k = 2048 x 16 heads x 128 fits).
 *   The first call on a device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   Every call uses the same array, so calls that overlap on the GPU (other
 *   streams, other host threads) race: order them. Calls allocate nothing.
 */
sa_status sa_sparse_attn_decode_noalloc(const sa_attn_in* in, const int32_t* idx, int32_t k, void* out,
                                        float* lse, cudaStream_t stream);

/*
 * sa_quantize_rows_e4m3: the indexer's FP8 input encoding, on the device
 * (Latent Sparse Attention section 2.1: the indexer runs in lower precision;
 * the format is OCP FP8 e4m3, one fp32 scale per row), for example for the
 * index key of each token a decode step appends.
 *   x: device [n_rows, d] row-major, dtype SA_F32 or SA_BF16.
 *   Per row: amax = max |x|; scale = amax / 448 in fp32 (1 for an all-zero
 *   row); bytes = e4m3(x / scale) with the division in fp32 (IEEE round to
 *   nearest) and the encoding rounding to nearest, ties to even, saturating
 *   at +-448.
 *   out: device [n_rows, d] uint8; scale: device [n_rows] fp32 (both
 *   caller-owned). d in [1, 4096]; n_rows >= 0 (0 is a no-op). A negative
 *   value that rounds to zero may encode as 0x80 (-0). NaN or infinite
 *   inputs are not supported (their rows' results are unspecified).
 *   SA_ERR_INVALID_ARGUMENT for null pointers or d out of range,
 *   SA_ERR_UNSUPPORTED for other dtypes, SA_ERR_CUDA on a launch error.
 */
sa_status sa_quantize_rows_e4m3(const void* x, sa_dtype dtype, int64_t n_rows, int32_t d, uint8_t* out,
                                float* scale, cudaStream_t stream);

/*
 * sa_expand_sinks_window: the index rows attention serves around the k
 * selected long-range keys (Latent Sparse Attention section 3.2 with its
 * attention-sink and local-window keys: J_t = sinks + window + the selected
 * keys those do not already cover).
 *   idx: device [n_q, k] int32 selected keys (any order, -1 padded); row t
 *   sits at position p = q_pos0 + t.
 *   out: device [n_q, n_sink + n_window + k] int32, caller-owned. Row t lists
 *   the sinks s < min(n_sink, p + 1) ascending, then the window keys
 *   max(n_sink, p - n_window + 1) <= s <= p ascending, then the entries of
 *   idx row t that are neither (in their order, -1 entries dropped), then -1.
 *   n_sink >= 0, n_window >= 0, k >= 1, n_q >= 0 (0 is a no-op).
 *   SA_ERR_INVALID_ARGUMENT for null pointers or negative sizes, SA_ERR_CUDA
 *   on a launch error.
 */
sa_status sa_expand_sinks_window(const int32_t* idx, int32_t n_q, int32_t k, int32_t q_pos0, int32_t n_sink,
                                 int32_t n_window, int32_t* out, cudaStream_t stream);

/*
 * LSA flat semantic search (Latent Sparse Attention section 3.1 "Semantic
 * Clustering", section 3.2 "Semantic Search", appendix F.1 "Kernels"): index
 * keys are clustered by content into buckets, once per cluster block of
 * n_cluster consecutive keys, and each query expands its best buckets into
 * its index row. Index keys and queries are bf16 rows of d_idx = 64.
 *
 *   n_pool           consecutive unit keys summed into one pool key (>= 1)
 *   n_cluster        keys per cluster block, a multiple of n_pool, with
 *                    n_cluster / n_pool <= 256 pool keys
 *   n_buckets        m, buckets per cluster block (1 .. n_cluster / n_pool)
 *   max_bucket_keys  n_b^max, a multiple of n_pool. With n_b^max >= 2
 *                    n_cluster / m every block reaches m buckets; a smaller
 *                    cap can leave no pair that fits before m buckets remain
 *                    (sa_lsa_build_buckets then reports it, see there)
 * Violations are SA_ERR_INVALID_ARGUMENT; d_idx != 64 or more than 256 pool
 * keys per block are SA_ERR_UNSUPPORTED.
 */
typedef struct {
  int32_t d_idx;
  int32_t n_pool;
  int32_t n_cluster;
  int32_t n_buckets;
  int32_t max_bucket_keys;
} sa_lsa_params;

/*
 * sa_lsa_build_buckets: the bucket cache of cluster blocks [block0, block0 +
 *   n_blocks) of the index keys k_idx (device bf16 [n_k, 64]; block c holds
 *   keys c * n_cluster .. (c + 1) * n_cluster - 1, so (block0 + n_blocks) *
 *   n_cluster <= n_k). Per block (section 3.1): keys are L2 normalised,
 *   summed n_pool at a time into pool keys, and clustered bottom up with
 *   Ward's method -- every round, all pairs of buckets that are each other's
 *   cheapest merge (among the merges that keep a bucket within n_b^max keys)
 *   merge, until m buckets remain; a round that would overshoot merges its
 *   cheapest pairs. The merge cost is n_a n_b / (n_a + n_b) |mu_a - mu_b|^2
 *   over bucket means mu (counts in pool keys), computed in fp32 with one
 *   rounding per operation and dimensions summed from 0 upward; cost ties go
 *   to the lower index. Buckets of a block are numbered by their lowest pool
 *   key; bucket b = c * m + r.
 *   Outputs (device, caller-owned, indexed by absolute block so that later
 *   blocks can be added by later calls):
 *     centroids    bf16 [(block0 + n_blocks) * m, 64]: the bucket's key sum
 *                  L2 normalised (fp32) and rounded to bf16 (nearest even)
 *     bucket_off   int32 [(block0 + n_blocks) * m]: start of the bucket's key
 *                  list in bucket_keys; the list ends at bucket_off[b + 1],
 *                  or at (c + 1) * n_cluster for the block's last bucket
 *     bucket_keys  int32 [(block0 + n_blocks) * n_cluster]: key positions,
 *                  ascending within each bucket; block c fills [c * n_cluster,
 *                  (c + 1) * n_cluster)
 *   status (device, nullable) is zeroed by the call; error = SA_ERR_INTERNAL
 *   if a block could not reach m buckets because no remaining pair fits the
 *   cap (only possible with n_b^max < 2 n_cluster / m); that block's outputs
 *   are then left unwritten.
 *   k_idx and centroids must be 16-byte aligned. No workspace, no host
 *   synchronisation. n_blocks = 0 is a no-op.
 */
sa_status sa_lsa_build_buckets(const sa_lsa_params* prm, const void* k_idx, int32_t n_k, int32_t block0,
                               int32_t n_blocks, void* centroids, int32_t* bucket_off, int32_t* bucket_keys,
                               sa_device_status* status, cudaStream_t stream);

/* Search regimes (appendix F.1 "Flat prefill"): TABLE writes each query's
 * bucket scores and selects its top p from them; STREAM never writes them:
 * a threshold per query from about 8192 sampled centroids, a scan that lists
 * the buckets at or above it (room for 3p), the top p of the list, and a
 * whole-row rescoring for the rows whose list missed (fewer than p listed, or
 * more than its room; their count is read back to the host once per chunk of
 * 8192 queries). Both select the same buckets from the same scores. AUTO
 * takes TABLE up to 32,768 buckets and STREAM beyond. */
#define SA_LSA_AUTO 0
#define SA_LSA_TABLE 1
#define SA_LSA_STREAM 2

typedef struct {
  int32_t p;          /* buckets kept per query, 1 .. 2048 */
  int32_t k;          /* long-range keys per query, >= 1 */
  int32_t n_sink;     /* attention-sink keys 0 .. n_sink - 1, >= 0 */
  int32_t n_window;   /* most recent keys, >= 0 */
  sa_device_status* status;   /* device, nullable; zeroed by the call (STREAM counts its fallback and
                                 overflowed rows there) */
  int32_t regime;     /* SA_LSA_AUTO, SA_LSA_TABLE or SA_LSA_STREAM (sa_lsa_search only) */
  int32_t test_hook;  /* 0; SA_HOOK_THETA_POS_INF / _NEG_INF force every STREAM row to its fallback */
} sa_lsa_search_opts;

/*
 * sa_lsa_search: index rows of queries over a bucket cache (section 3.2).
 *   q_idx: device bf16 [n_q, 64] index queries (not yet normalised); row i
 *   sits at position pos = q_pos0 + i. The cache holds blocks 0 .. n_blocks
 *   - 1 (from sa_lsa_build_buckets); the query scores the unit centroids of
 *   blocks c < min(n_blocks, pos / n_cluster), s_b = c_b . q (q L2
 *   normalised in fp32, rounded to bf16; products on the tensor cores with
 *   fp32 accumulation), keeps the top p (ties: lower bucket id), and takes
 *   their keys best first (score, then lower id; a bucket's keys in list
 *   order) until k long-range keys are held, skipping keys among the sinks
 *   (s < n_sink) or in the window (s >= max(n_sink, pos - n_window + 1)).
 *   J: device int32 [n_q, n_sink + n_window + k], caller-owned. Row i: the
 *   sinks ascending, the window ascending, the long-range keys (best bucket
 *   first), then -1. Fewer than k long-range keys when the p buckets hold
 *   fewer uncovered keys.
 *   Regimes: see SA_LSA_*. TABLE needs n_blocks * m <= 32768 and STREAM
 *   n_blocks * m <= 2^21 (else SA_ERR_UNSUPPORTED). Workspace:
 *   sa_lsa_search_workspace_size bytes (for the same opts), 256-byte
 *   aligned. TABLE does not synchronise the host; STREAM synchronises the
 *   stream once per chunk of 8192 queries. status error = SA_ERR_TIMEOUT if
 *   a bounded wait gave up.
 */
sa_status sa_lsa_search(const sa_lsa_params* prm, const sa_lsa_search_opts* opts, const void* q_idx, int32_t n_q,
                        int32_t q_pos0, const void* centroids, const int32_t* bucket_off,
                        const int32_t* bucket_keys, int32_t n_blocks, int32_t* J, void* ws, size_t ws_bytes,
                        cudaStream_t stream);

/* Workspace bytes of sa_lsa_search for these sizes (host call). */
sa_status sa_lsa_search_workspace_size(const sa_lsa_params* prm, const sa_lsa_search_opts* opts, int32_t n_q,
                                       int32_t q_pos0, int32_t n_blocks, size_t* bytes);

/*
 * sa_lsa_decode: one LSA decode step for `batch` sequences, each with its own
 *   bucket cache (appendix F.1 "Flat decode": every request adds one query
 *   per step, which scores the centroids of its request once, on the CUDA
 *   cores -- at one flop per byte the scan is bound by HBM).
 *   q_idx: device bf16 [batch, 64], the new index query of each sequence; it
 *   sits at position seq_lens[b] - 1 (seq_lens: device int32 [batch], >= 1).
 *   The caches are per-sequence slabs of what sa_lsa_build_buckets writes
 *   for that sequence's keys: centroids bf16 [batch, max_blocks * m, 64],
 *   bucket_off int32 [batch, max_blocks * m], bucket_keys int32 [batch,
 *   max_blocks * n_cluster], positions within the sequence. n_blocks: device
 *   int32 [batch], the cluster blocks each cache holds; the query scores the
 *   buckets of blocks c < min(n_blocks[b], max_blocks, (seq_lens[b] - 1) /
 *   n_cluster). Selection and the row layout are those of sa_lsa_search.
 *   J: device int32 [batch, n_sink + n_window + k].
 *   max_blocks * m <= 32768 (else SA_ERR_UNSUPPORTED). Workspace:
 *   sa_lsa_decode_workspace_size bytes, 256-byte aligned. No host
 *   synchronisation and no allocation, and every size is fixed by max_blocks
 *   and batch (lengths are read on the device): the call can be captured in a
 *   CUDA graph.
 */
sa_status sa_lsa_decode(const sa_lsa_params* prm, const sa_lsa_search_opts* opts, const void* q_idx, int32_t batch,
                        const void* centroids, const int32_t* bucket_off, const int32_t* bucket_keys,
                        int32_t max_blocks, const int32_t* n_blocks, const int32_t* seq_lens, int32_t* J, void* ws,
                        size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes of sa_lsa_decode for these sizes (host call). */
sa_status sa_lsa_decode_workspace_size(const sa_lsa_params* prm, const sa_lsa_search_opts* opts, int32_t batch,
                                       int32_t max_blocks, size_t* bytes);

/*
 * sa_lsa_attention: softmax attention over LSA index rows (section 3.2: one
 *   row J_i per query, shared by all heads), on the tensor cores in two passes
 *   whose results are merged by their log-sum-exp: the sinks and windows of
 *   groups of 8 consecutive queries, and the long-range keys of groups of 8
 *   queries whose long-range keys overlap (MinHash grouping). The result is
 *   attention over the whole row, as sa_sparse_attn computes it.
 *   J: device int32 [n_q, width] as sa_lsa_search writes it for these q_pos0,
 *   n_sink and n_window (width = n_sink + n_window + k): row i holds the
 *   sinks and window of position q_pos0 + i, then long-range keys, then -1.
 *   attn: prefill operands (batch 0), with q_pos0 + n_q <= n_k (the local part
 *   reads the keys up to each query's own position); out bf16 [n_q, n_q_heads, head_dim],
 *   lse fp32 [n_q, n_q_heads] (nullable). Supported: 16 heads x 128 and
 *   n_k <= 196608 (else SA_ERR_UNSUPPORTED: use sa_sparse_attn). status
 *   (nullable) is zeroed by the call and reports a bounded wait that gave up.
 *   Workspace: sa_lsa_attention_workspace_size bytes, 256-byte aligned. No
 *   host synchronisation.
 */
sa_status sa_lsa_attention(const sa_attn_in* attn, const int32_t* J, int32_t width, int32_t q_pos0, int32_t n_sink,
                           int32_t n_window, void* out, float* lse, sa_device_status* status, void* ws,
                           size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes of sa_lsa_attention (host call). */
sa_status sa_lsa_attention_workspace_size(const sa_attn_in* attn, int32_t width, int32_t q_pos0, int32_t n_sink,
                                          int32_t n_window, size_t* bytes);

/*
 * sa_debug_errors: invariant checks of the debug build (compiled with
 *   -DSA_DEBUG_CHECKS: `build.py --debug-checks` writes libsa_debug.so). A
 *   failed check records its site and value in device memory and the kernel
 *   carries on without the guarded access (an attention index beyond the
 *   cache is skipped, as in the release build); nothing traps. This call
 *   reads the record: out (host uint32 [4]) = {first failed site
 *   (SA_DBG_* in the library's debug.cuh), its value, number of failed
 *   checks, 0}; reset != 0 clears it. Synchronous (device -> host copies);
 *   call it after the stream's work has finished. The record is global to the
 *   process: concurrent calls share it. Release builds return
 *   SA_ERR_UNSUPPORTED and check nothing.
 */
sa_status sa_debug_errors(uint32_t* out, int32_t reset);

/*
 * sa_workspace_size: bytes of device workspace `op` needs for these operands
 * (host call, no device work). opts points to sa_prefill_opts (PREFILL),
 * sa_decode_opts (DECODE), an int32_t k (TOPK, SPARSE_ATTN) or NULL.
 * Workspace must be 256-byte aligned.
 */
sa_status sa_workspace_size(sa_op op, const sa_indexer_in* in, const sa_attn_in* attn,
                            const void* opts, size_t* bytes);

/*
 * sa_prefill_chunk_rows: the number of query rows sa_prefill processes per
 * chunk for these operands and options (host call, no device work): the
 * call's rows are taken in ceil(n_q / rows) consecutive chunks, each with
 * its own stage events (see stage_events above). It follows the same plan as
 * sa_workspace_size (SA_OP_PREFILL). SA_ERR_INVALID_ARGUMENT for a NULL
 * argument or invalid options.
 */
sa_status sa_prefill_chunk_rows(const sa_indexer_in* in, const sa_prefill_opts* opts, int32_t* rows);

#ifdef __cplusplus
}
#endif
#endif /* SA_H_ */
