"""Oracle two-stage (hierarchical) indexer.

HISA (theflow "related" page): a block-level coarse filter first discards
irrelevant regions, then the original token-level indexer runs only inside the
retained blocks, feeding the same top-k pattern to the attention. A block is
scored by the mean of its keys (MoBA, as summarised in Latent Sparse
Attention section 2.2), with the token indexer's own formula.

Readings where the pages leave a step open (each listed in the design notes):
  * block keys: K_b = mean over the block_size keys of block b of the
    dequantised index keys sk[s] * e4m3(k[s]); the sum runs in fp64 in key
    order, is divided by block_size and rounded to fp32. K_b is then stored
    like every index key: e4m3 bytes with one fp32 scale per block, scale =
    amax/448 (1 for a zero block), bytes = RNE(K_b / scale) (fp32 division)
    saturated to +-448. Stage 1 therefore runs the same low-precision
    indexer arithmetic as stage 2.
  * eligible blocks of query t (absolute position p = pos0 + t): the complete
    blocks b < cur = floor(p / block_size). Block 0 and the current block cur
    are always kept (the pages' block-sparse baselines always keep the first
    and the current blocks, Latent Sparse Attention section 4.1 / Table 2);
    the best keep-2 of the others b in [1, cur-1] by (score desc, b asc) join
    them (all of them when there are fewer).
  * stage 2 candidates: the keys s <= p of the kept blocks; top-k over them in
    the order of the token-level top-k.
"""
import numpy as np

from .fp8 import e4m3_decode, e4m3_quantize_rne
from .indexer import scores_row


def pool_block_keys(k_bytes, k_scale, block: int = 64):
    """Block keys of the complete blocks: (uint8 [nb, d], fp32 scale [nb])."""
    kv = e4m3_decode(np.asarray(k_bytes, dtype=np.uint8))            # [n, d] fp64
    sk = np.asarray(k_scale, dtype=np.float32).astype(np.float64)
    n, d = kv.shape
    nb = n // block
    out_b = np.zeros((nb, d), dtype=np.uint8)
    out_s = np.ones(nb, dtype=np.float32)
    for b in range(nb):
        acc = np.zeros(d, dtype=np.float64)
        for s in range(b * block, (b + 1) * block):         # key order
            acc = acc + kv[s] * sk[s]
        mean = (acc / block).astype(np.float32)
        amax = np.float32(np.abs(mean).max())
        scale = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
        out_b[b] = e4m3_quantize_rne((mean / scale).astype(np.float32))
        out_s[b] = scale
    return out_b, out_s


def keep_blocks_row(block_scores, p: int, block: int = 64, keep: int = 64) -> np.ndarray:
    """Kept blocks (ascending) of a query at absolute position p, given the
    fp32 scores of blocks [0, cur) (entries at index >= cur are ignored)."""
    cur = p // block
    if cur == 0:
        return np.array([0], dtype=np.int64)
    others = np.arange(1, cur)
    if len(others) > keep - 2:
        sc = np.asarray(block_scores, dtype=np.float32)[1:cur].astype(np.float64)
        order = np.lexsort((others, -sc))
        others = others[order[:keep - 2]]
    return np.array(sorted({0, cur} | set(int(b) for b in others)), dtype=np.int64)


def two_stage_candidates(kept, p: int, block: int = 64) -> np.ndarray:
    """Visible keys (ascending) of the kept blocks."""
    out = []
    for b in kept:
        lo, hi = int(b) * block, min(int(b) * block + block, p + 1)
        out.extend(range(lo, hi))
    return np.array(out, dtype=np.int64)


def block_scores_row(q_t, sq_t, blk_vals, blk_scale, w_t, cur: int) -> np.ndarray:
    """Scores of blocks [0, cur) for one query (token-indexer formula)."""
    return scores_row(q_t, sq_t, blk_vals[:cur], blk_scale[:cur], w_t)
