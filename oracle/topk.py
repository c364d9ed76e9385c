"""Oracle exact top-k.

Order of keys: higher fp32 score first; at equal scores the lower key index
first. This is the order of the packed 64-bit key of Latent Sparse Attention
appendix F.1 ("Selection by threshold": score bits in the upper half, the
inverted id in the lower half, a larger packed key is a better score or, at
equal scores, a lower id). The selected set is the first min(k, n) keys of a
full sort in that order; rows with fewer than k visible keys are padded with
-1 by the caller.
"""
import numpy as np


def topk_row(scores, k: int) -> np.ndarray:
    """Indices (int64) of the top-k of a fp32 score row by full sort on
    (score descending, index ascending). -0.0 and +0.0 compare equal."""
    s = np.asarray(scores, dtype=np.float32).astype(np.float64)
    n = s.shape[0]
    idx = np.arange(n)
    order = np.lexsort((idx, -s))          # last key is the primary one
    return order[:min(k, n)]


def topk_row_bruteforce(scores, k: int) -> np.ndarray:
    """The same set by explicit ranks: rank(s) = #{s': score[s'] > score[s] or
    (score[s'] == score[s] and s' < s)}; selected iff rank < k. O(n^2), for
    self-checks on tiny rows."""
    s = [float(x) for x in np.asarray(scores, dtype=np.float32)]
    n = len(s)
    sel = []
    for i in range(n):
        rank = 0
        for j in range(n):
            if s[j] > s[i] or (s[j] == s[i] and j < i):
                rank += 1
        if rank < k:
            sel.append(i)
    return np.array(sel, dtype=np.int64)


def pad_row(sel, k: int) -> np.ndarray:
    out = np.full(k, -1, dtype=np.int64)
    out[:len(sel)] = sel
    return out
