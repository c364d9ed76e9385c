"""Comparison rules shared by the parity tests (CUDA path vs oracle).

Top-k ("tie band"): theta = the oracle's k-th score of the row, M = the row
max, band = 1e-4 * M. The GPU set passes iff every key scoring > theta + band
is in it, no key scoring < theta - band is, it has min(k, visible) distinct
visible keys, and -1 appears only after them. Sets are compared, not orders
(the order of an index row is unspecified).

Scores: normwise per row, max_s |g - o| <= tol * max_s |o| over visible keys,
with the contract tolerance (2e-2 FP8, 2e-3 bf16) and an internal gate of
1e-5 (fp32 accumulation only; it has to stay well inside the 1e-4 band).

Attention: max |g - o| <= 1e-2 against fp64 over the same indices (the
contract) and the internal gate max |g - o| <= 1e-2 * max |o| + 1e-6.
"""
import numpy as np

BAND = 1e-4
SCORE_GATE = 1e-5


def check_topk_row(gpu_row, cand, scores, k, where=""):
    """gpu_row: int array [k] (-1 padded); cand: candidate key ids; scores:
    their fp32 oracle scores (same order)."""
    g = np.asarray(gpu_row, dtype=np.int64)
    n_vis = len(cand)
    want = min(k, n_vis)
    valid = g[g >= 0]
    assert len(valid) == want, f"{where}: {len(valid)} valid entries, want {want}"
    assert (g[:want] >= 0).all() and (g[want:] == -1).all(), f"{where}: -1 not at the tail"
    assert len(set(valid.tolist())) == want, f"{where}: duplicate indices"
    pos = {int(c): i for i, c in enumerate(cand)}
    missing = [int(x) for x in valid if int(x) not in pos]
    assert not missing, f"{where}: invisible keys {missing[:5]}"
    if want == n_vis:
        return
    s = np.asarray(scores, dtype=np.float64)
    order = np.lexsort((np.arange(n_vis), -s))
    theta = s[order[want - 1]]
    band = BAND * max(np.abs(s).max(), 1e-30)
    sel = np.zeros(n_vis, dtype=bool)
    sel[[pos[int(x)] for x in valid]] = True
    must = s > theta + band
    never = s < theta - band
    assert not (must & ~sel).any(), f"{where}: {int((must & ~sel).sum())} keys above the band missing"
    assert not (never & sel).any(), f"{where}: {int((never & sel).sum())} keys below the band selected"


def check_scores_row(gpu, ref, tol, where=""):
    g = np.asarray(gpu, dtype=np.float64)
    o = np.asarray(ref, dtype=np.float64)
    m = np.abs(o).max() if o.size else 0.0
    err = np.abs(g - o).max() if o.size else 0.0
    assert err <= tol * max(m, 1e-30), f"{where}: normwise err {err / max(m, 1e-30):.3e} > {tol}"
    return err / max(m, 1e-30)


def check_attention_row(o_gpu, o_ref, lse_gpu=None, lse_ref=None, where=""):
    g = np.asarray(o_gpu, dtype=np.float64)
    r = np.asarray(o_ref, dtype=np.float64)
    err = np.abs(g - r).max()
    assert err <= 1e-2, f"{where}: max-abs err {err}"
    assert err <= 1e-2 * np.abs(r).max() + 1e-6, f"{where}: err {err} vs max|o| {np.abs(r).max()}"
    if lse_gpu is not None:
        lg, lr = np.asarray(lse_gpu, dtype=np.float64), np.asarray(lse_ref, dtype=np.float64)
        fin = np.isfinite(lr)
        assert np.array_equal(np.isfinite(lg), fin), f"{where}: lse finiteness"
        if fin.any():
            assert np.abs(lg[fin] - lr[fin]).max() <= 1e-4, f"{where}: lse err {np.abs(lg[fin] - lr[fin]).max()}"
    return err


# LSA index rows: the device ranks buckets by fp32 tensor-core sums, the oracle
# by fp64 sums over the same bf16 operands (a few 1e-7 apart at d_idx = 64).
LSA_TIE = 1e-5


def _bucket_end(b, off, m, n_cluster):
    c, r = divmod(b, m)
    return (c + 1) * n_cluster if r == m - 1 else int(off[b + 1])


def check_lsa_row(got, want, qn, pos, cache, n_blocks, n_cluster, m, p, n_sink, n_window, where=""):
    """An LSA index row against the oracle's. Sinks and window must be exact.
    The long-range part must equal the oracle's, or else differ only by the
    order of buckets whose fp64 scores lie within LSA_TIE (the device ranks by
    fp32 tensor-core sums): the device's bucket sequence is recovered from its
    keys, and then (a) every bucket's keys come as one run, in list order,
    skipping the keys the sinks or the window hold, all of them except in the
    last bucket when the row is full; (b) consecutive buckets are in score
    order up to LSA_TIE; (c) every bucket used could be among the top p (its
    score at least the p-th best minus LSA_TIE); (d) no bucket scoring more
    than LSA_TIE above the last one used, with a key to give, was skipped, and
    a row with room left used every bucket above the p-th best plus LSA_TIE.
    Returns True when the row needed the tie exception."""
    from oracle import lsa
    cent, off, keys = cache
    got = np.asarray(got)
    head = min(n_sink, pos + 1) + max(0, pos - max(n_sink, pos - n_window + 1) + 1)
    assert np.array_equal(got[:head], want[:head]), f"{where}: sinks / window"
    if np.array_equal(got, want):
        return False
    k = len(got) - n_sink - n_window
    w_lo = max(n_sink, pos - n_window + 1)
    far = got[head:]
    assert (far[(far >= 0).sum():] == -1).all(), f"{where}: -1 not at the tail"
    far = far[far >= 0].tolist()
    n_vis = min(n_blocks, pos // n_cluster) * m
    s = lsa.bucket_scores(qn, cent, n_vis)
    order = np.lexsort((np.arange(n_vis), -s))
    theta_p = s[order[min(p, n_vis) - 1]] if n_vis else np.inf
    uncovered = {}
    def free_keys(b):
        if b not in uncovered:
            lst = keys[off[b]:_bucket_end(b, off, m, n_cluster)]
            uncovered[b] = [int(x) for x in lst if not (int(x) < n_sink or int(x) >= w_lo)]
        return uncovered[b]
    key2b = {}
    for c in sorted({x // n_cluster for x in far}):
        assert c < min(n_blocks, pos // n_cluster), f"{where}: key of an invisible block"
        for b in range(c * m, c * m + m):
            for x in keys[off[b]:_bucket_end(b, off, m, n_cluster)]:
                key2b[int(x)] = b
    seq, i = [], 0
    while i < len(far):
        b = key2b[far[i]]
        assert b not in seq, f"{where}: bucket {b} in two runs"
        run = free_keys(b)
        n = min(len(run), len(far) - i)
        assert far[i:i + n] == run[:n], f"{where}: bucket {b} keys out of list order"
        last_partial = n < len(run)
        i += n
        assert not last_partial or i == k, f"{where}: bucket {b} cut short before the row is full"
        seq.append(b)
    assert len(far) == len(set(far)), f"{where}: duplicate keys"
    for a, b in zip(seq, seq[1:]):
        assert s[a] >= s[b] - LSA_TIE, f"{where}: bucket {b} ({s[b]:.7f}) after {a} ({s[a]:.7f})"
    for b in seq:
        assert s[b] >= theta_p - LSA_TIE, f"{where}: bucket {b} is not among the top {p}"
    used = set(seq)
    floor = s[seq[-1]] + LSA_TIE if seq else -np.inf
    if len(far) < k:
        floor = min(floor, theta_p + LSA_TIE)
    skipped = [int(b) for b in order[:p] if b not in used and s[b] > floor and free_keys(int(b))]
    assert not skipped, f"{where}: better buckets {skipped[:4]} skipped"
    return True
