"""Oracle for whole rows of the hot path: indexer -> exact top-k -> sparse
attention (flat or two-stage prefill, and one decode step).

Prefill rows: query t sits at absolute position pos0 + t and sees keys
s <= pos0 + t (causal, Latent Sparse Attention section 2). Decode: each
sequence adds one query whose own key is the last cache row, so it sees keys
s < seq_len (a reading: the new token's key is appended before it attends).
Index rows have k entries padded with -1 when fewer keys are visible.
"""
import numpy as np

from .attention import sparse_attention_row
from .fp8 import e4m3_decode
from .indexer import IndexerInputs, as_numpy, dequant, scores_row
from .topk import pad_row, topk_row
from .two_stage import block_scores_row, keep_blocks_row, pool_block_keys, two_stage_candidates


def prefill_rows(host, rows, k: int, mode: str = "flat", block: int = 64, keep: int = 64,
                 pos0: int = 0, scale=None, attention: bool = True, blocks=None, positions=None):
    """Oracle results for the given query rows of a prefill input.

    Per row: idx (int64 [k], -1 padded), cand (candidate key indices), scores
    (fp32 scores of the candidates, same order), and for two-stage kept
    (kept blocks) and bscores (block scores of blocks [0, cur)); O / lse
    (fp64 attention over idx) unless attention=False. ``blocks`` may carry
    precomputed (bytes, scale) block keys. ``positions`` (same length as
    rows) gives each row's absolute position when the host tensors hold only
    the sampled query rows (default pos0 + t)."""
    ii = IndexerInputs(host)
    n_k = ii.kv.shape[0]
    K = as_numpy(host["K"]) if attention else None
    V = as_numpy(host["V"]) if attention else None
    if mode == "two_stage":
        if blocks is None:
            blocks = pool_block_keys(host["k_idx"].numpy(), host["k_scale"].numpy(), block)
        blk_vals = e4m3_decode(blocks[0])
        blk_scale = blocks[1].astype(np.float64)
    out = {}
    for i, t in enumerate(rows):
        t = int(t)
        p = pos0 + t if positions is None else int(positions[i])
        n_vis = min(n_k, p + 1)
        r = {}
        q_t = dequant(ii.q[t])
        sq_t = None if ii.sq is None else ii.sq[t]
        if mode == "flat":
            cand = np.arange(n_vis)
            sc = scores_row(q_t, sq_t, ii.kv[:n_vis], None if ii.sk is None else ii.sk[:n_vis], ii.w[t])
        else:
            cur = p // block
            bs = block_scores_row(q_t, sq_t, blk_vals, blk_scale, ii.w[t], cur)
            kept = keep_blocks_row(bs, p, block, keep)
            cand = two_stage_candidates(kept, min(p, n_k - 1), block)
            sc = scores_row(q_t, sq_t, ii.kv[cand], None if ii.sk is None else ii.sk[cand], ii.w[t])
            r["kept"], r["bscores"] = kept, bs
        r["cand"], r["scores"] = cand, sc
        r["idx"] = pad_row(cand[topk_row(sc, k)], k)
        if attention:
            r["O"], r["lse"] = sparse_attention_row(as_numpy(host["Q"][t]), K, V, r["idx"], scale)
        out[t] = r
    return out


def attention_rows(host, idx_rows: dict, scale=None):
    """Prefill attention of the given rows over supplied index rows {t: idx}."""
    K, V = as_numpy(host["K"]), as_numpy(host["V"])
    return {t: sparse_attention_row(as_numpy(host["Q"][t]), K, V, np.asarray(idx), scale)
            for t, idx in idx_rows.items()}


def decode_rows(host, seqs, k: int, scale=None, attention: bool = True):
    """Oracle for one decode step of the given sequences."""
    out = {}
    lens = as_numpy(host["seq_lens"])
    for b in seqs:
        b = int(b)
        L = int(lens[b])
        kv = e4m3_decode(host["k_idx"][b, :L].numpy())
        sk = host["k_scale"][b, :L].numpy().astype(np.float64)
        q_t = e4m3_decode(host["q_idx"][b].numpy())
        sq_t = host["q_scale"][b].numpy().astype(np.float64)
        w_t = host["w"][b].numpy().astype(np.float64)
        sc = scores_row(q_t, sq_t, kv, sk, w_t)
        r = {"scores": sc, "cand": np.arange(L), "idx": pad_row(topk_row(sc, k), k)}
        if attention:
            r["O"], r["lse"] = decode_attention_row(host, b, r["idx"], scale)
        out[b] = r
    return out


def decode_attention_row(host, b: int, idx, scale=None):
    """Attention of sequence b's query over its own cache rows idx."""
    L = int(as_numpy(host["seq_lens"])[b])
    return sparse_attention_row(as_numpy(host["Q"][b]), as_numpy(host["K"][b, :L]),
                                as_numpy(host["V"][b, :L]), np.asarray(idx), scale)


def expand_sinks_window_row(idx, p: int, n_sink: int, n_window: int):
    """The served index row of the query at position p (Latent Sparse
    Attention section 3.2 with attention sinks and a local window): the sinks
    0 .. min(n_sink, p + 1) - 1, then the window max(n_sink, p - n_window + 1)
    .. p, then the selected keys (in their order) that neither covers, then -1
    up to n_sink + n_window + len(idx)."""
    idx = [int(s) for s in np.asarray(idx).tolist()]
    sinks = list(range(min(n_sink, p + 1)))
    w_lo = max(n_sink, p - n_window + 1)
    window = list(range(w_lo, p + 1))
    rest = [s for s in idx if s >= 0 and not (s < n_sink or s >= w_lo)]
    row = sinks + window + rest
    return np.array(row + [-1] * (n_sink + n_window + len(idx) - len(row)), dtype=np.int64)
