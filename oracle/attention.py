"""Oracle softmax attention over the selected keys of one shared KV head.

O[h] = sum_{s in J} softmax_s(scale * Q[h] . K[s]) V[s], with one index set J
shared by every query head (Latent Sparse Attention section 3.2: "a single J_i
is shared across all query heads"; attention is computed only over the keys
indexed by J_i). J rows hold KV-cache slots padded with -1 (appendix F.1,
"Attention kernels"); the order of J does not matter. scale defaults to
1/sqrt(head_dim) (the pages give none; the usual softmax scaling). fp64
throughout; lse is the natural-log sum of exponentials of the scaled logits.
"""
import math

import numpy as np


def sparse_attention_row(Q_t, K, V, idx, scale=None):
    """Q_t [Hq, dh], K/V [n, dh] (fp64), idx [k] with -1 padding.
    Returns (O [Hq, dh] fp64, lse [Hq] fp64). No selected key -> zeros, -inf."""
    Q_t = np.asarray(Q_t, dtype=np.float64)
    dh = Q_t.shape[1]
    scale = 1.0 / math.sqrt(dh) if not scale else scale
    sel = np.asarray(idx)
    sel = sel[sel >= 0]
    if sel.size == 0:
        return np.zeros_like(Q_t), np.full(Q_t.shape[0], -np.inf)
    logits = (Q_t @ np.asarray(K, dtype=np.float64)[sel].T) * scale
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    l = p.sum(axis=1, keepdims=True)
    O = (p @ np.asarray(V, dtype=np.float64)[sel]) / l
    return O, (m + np.log(l))[:, 0]


def dense_causal_attention_row(Q_t, K, V, t, scale=None):
    """Full causal attention of query t over keys 0..t, written independently
    of the function above (explicit per-key loop, two passes) for the
    k >= t+1 self-check."""
    Q_t = np.asarray(Q_t, dtype=np.float64)
    Hq, dh = Q_t.shape
    scale = 1.0 / math.sqrt(dh) if not scale else scale
    O = np.zeros((Hq, dh))
    lse = np.zeros(Hq)
    for h in range(Hq):
        logits = [float(np.dot(Q_t[h], np.asarray(K[s], dtype=np.float64))) * scale
                  for s in range(t + 1)]
        mx = max(logits)
        den = 0.0
        acc = np.zeros(dh)
        for s in range(t + 1):
            e = math.exp(logits[s] - mx)
            den += e
            acc += e * np.asarray(V[s], dtype=np.float64)
        O[h] = acc / den
        lse[h] = mx + math.log(den)
    return O, lse
