"""Oracle indexer scores.

score(t, s) = sum_h w[t,h] * ReLU(q_idx[t,h] . k_idx[s]) for the causal keys
s <= t: the lightweight token-level indexer ("fewer heads, smaller dimension,
lower precision", Latent Sparse Attention section 2.1), here with per-head
query weights w >= 0 and no further normalisation.

With FP8 inputs, q_idx[t,h] = sq[t,h] * e4m3(bytes) and k_idx[s] = sk[s] *
e4m3(bytes). Every e4m3 value is a multiple of 2^-9 with at most 4 significant
bits, so each product is a multiple of 2^-18 below 2^17.7 and a sum of 128 of
them stays below 2^24.7: the dot product of the decoded values is EXACT in
fp64 whatever the summation order (42.6 < 53 bits). The oracle then forms
a_h = dot * sq * sk and sum_h w * max(a_h, 0) in fp64 and rounds once to fp32.
bf16 inputs: products are exact in fp64, the sum is fp64.
"""
import numpy as np

from .fp8 import e4m3_decode


def as_numpy(t):
    """Host tensor -> numpy: uint8 (e4m3 bytes) stays uint8, int stays int,
    floating point (bf16 / fp32) is widened exactly to fp64. None -> None."""
    if t is None:
        return None
    import torch
    if t.dtype in (torch.uint8, torch.int32, torch.int64):
        return t.numpy()
    return t.to(torch.float64).numpy()


def dequant(x) -> np.ndarray:
    """Index vectors as fp64 values without their scale: e4m3 bytes are
    decoded, anything else is already fp64."""
    if x.dtype == np.uint8:
        return e4m3_decode(x)
    return np.asarray(x, dtype=np.float64)


def scores_row(q_t, sq_t, k_vals, sk, w_t) -> np.ndarray:
    """Scores of one query against the key rows given.

    q_t    [H, d] fp64 decoded index query (scale not applied)
    sq_t   [H]    per-head query scale, or None (bf16 inputs: scale 1)
    k_vals [n, d] fp64 decoded index keys (scale not applied)
    sk     [n]    per-key scale, or None
    w_t    [H]    head weights (>= 0)
    returns fp32 [n]
    """
    a = k_vals @ q_t.T                                     # [n, H] dot products
    if sq_t is not None:
        a = a * np.asarray(sq_t, dtype=np.float64)[None, :]
    if sk is not None:
        a = a * np.asarray(sk, dtype=np.float64)[:, None]
    s = (np.maximum(a, 0.0) * np.asarray(w_t, dtype=np.float64)[None, :]).sum(axis=1)
    return s.astype(np.float32)


class IndexerInputs:
    """numpy view of one indexer problem: decoded keys are computed once."""

    def __init__(self, host, keys_from=0, keys_to=None):
        self.q = as_numpy(host["q_idx"])
        self.sq = as_numpy(host.get("q_scale"))
        k = as_numpy(host["k_idx"])
        self.kv = dequant(k if keys_to is None else k[keys_from:keys_to])
        sk = as_numpy(host.get("k_scale"))
        self.sk = None if sk is None else (sk if keys_to is None else sk[keys_from:keys_to])
        self.w = as_numpy(host["w"])

    def row(self, t, n_vis):
        """fp32 scores of query row t against keys [0, n_vis)."""
        return scores_row(dequant(self.q[t]), None if self.sq is None else self.sq[t],
                          self.kv[:n_vis], None if self.sk is None else self.sk[:n_vis],
                          self.w[t])


def scores_rows(host, rows, pos0: int = 0) -> dict:
    """Causal score rows {t: fp32 [min(n_k, pos0 + t + 1)]} of a prefill input."""
    ii = IndexerInputs(host)
    n_k = ii.kv.shape[0]
    return {int(t): ii.row(int(t), min(n_k, pos0 + int(t) + 1)) for t in rows}
