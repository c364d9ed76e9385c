"""CPU oracle for learned top-k sparse attention -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct numpy code (fp64 unless a step fixes another
precision) that states what the hot path computes:

  (1) indexer   score(t, s) = sum_h w[t,h] * ReLU(q_idx[t,h] . k_idx[s]), s <= t
  (2) top-k     the k visible keys of largest score, ties to the lower index
  (3) attention softmax attention over the selected keys of one shared KV head
  (+) two-stage mean-pooled key blocks filter the keys before (1)-(2)
  (+) LSA flat semantic search (``oracle.lsa``): unit keys pooled and
      Ward-clustered into buckets per cluster block, queries score the
      bucket centroids, and the top-p buckets expand into the index row

Only tests/, the smoke check and the CPU-baseline leg of the benchmark may
import this package; the product path (the CUDA library and its binding) never
does, and this package imports nothing from it. The oracle and the CUDA path
share no code; they share only the seeded input generator (``workloads``),
which holds none of the method's arithmetic.

Sources: "Latent Sparse Attention" (paperpeel 2610.42147) section 2 (token
sparse attention: an indexer selects k keys per query, attention runs over
only those), section 2.1 (the lightweight indexer), section 3.2 (one index
set shared by all query heads), appendix F.1 "Selection by threshold" (packed
64-bit key: higher score first, lower id on ties; output order irrelevant) and
"Attention kernels" (index rows of KV slots padded with -1); the HISA summary
on the theflow "related" page (block-level coarse filter, then the token
indexer inside the kept blocks) and LSA section 2.2 (a block scored by the mean
of its keys, as in MoBA).
"""
from .fp8 import e4m3_decode_table, e4m3_decode, e4m3_quantize_rne, quantize_rows  # noqa: F401
from .indexer import scores_row, scores_rows  # noqa: F401
from .topk import topk_row, topk_row_bruteforce  # noqa: F401
from .attention import sparse_attention_row, dense_causal_attention_row  # noqa: F401
from .two_stage import pool_block_keys, keep_blocks_row, two_stage_candidates  # noqa: F401
from .pipeline import prefill_rows, decode_rows  # noqa: F401
