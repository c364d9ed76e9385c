"""Oracle for the LSA flat semantic search -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check and the benchmark's CPU legs use this module; the
CUDA library never does, and it imports nothing from the library.

Follows "Latent Sparse Attention" (paperpeel 2610.42147):
  section 3.1  key normalisation, pooling of n_pool consecutive keys, Ward
               clustering of each cluster block of n_cluster keys into m
               buckets (mutually cheapest pairs merge in parallel rounds; a
               bucket never holds more than n_b^max keys), the bucket cache
               (unit-norm centroid of each bucket's key sum, and the
               positions of its keys);
  section 3.2  query normalisation, scores s_{i,b} = c_b . q_i over the
               buckets of the cluster blocks before the query's own, the
               top-p buckets, and their expansion best first into k
               long-range keys that skip the n_sink sinks and the n_w most
               recent keys, which the query attends to anyway;
  appendix F.1 "Selection by threshold" (buckets ranked by score, ties to
               the lower bucket id) and "Attention kernels" (index rows of
               n_sink + n_w + k key slots padded with -1).

Precision. Clustering turns floating-point costs into integer decisions
(which buckets merge), so the oracle takes them in the precision the device
takes them in: every operation on clustering data below is one IEEE fp32
operation (a product and a sum are two roundings, never one fused step), and
every sum over the d_idx dimensions runs from dimension 0 upward. Centroids
and normalised queries are rounded to bf16 (nearest, ties to even), the
operand type of the scan (appendix F.1: both operands bf16, fp32
accumulation). Scores here are exact products of those bf16 values summed in
fp64.

Readings of steps the pages leave open:
  - Ward's cost of merging buckets a and b is the increase of the squared
    distances of their members from their mean: n_a n_b / (n_a + n_b) *
    |mu_a - mu_b|^2 with mu = sum / n. Members are pool keys (every pool key
    stands for n_pool keys, so counting keys instead scales every cost alike).
  - A pair whose merged bucket would exceed n_b^max is never a partner: a
    bucket's cheapest partner is taken among the pairs that fit.
  - A bucket's cheapest partner breaks cost ties to the lower index. All
    mutually cheapest pairs merge in one round; when fewer merges are needed
    to reach m buckets, the cheapest pairs merge (cost, then lower index).
  - A merged bucket keeps the lower index; buckets are numbered within their
    cluster block by their lowest pool key, and bucket b of block c has id
    c * m + b. A bucket lists its key positions in ascending order.
  - The expansion walks the top-p buckets by (score descending, id
    ascending) and each bucket's keys in list order.
  - Sinks are positions 0 .. n_sink - 1; the window is positions
    max(n_sink, i - n_w + 1) .. i for the query at position i.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32


# ------------------------------------------------------------- number formats
def bf16_round(x) -> np.ndarray:
    """fp32 values rounded to the nearest bf16 (ties to even), returned as
    fp32. Finite inputs only."""
    u = np.ascontiguousarray(np.asarray(x, dtype=F32)).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(F32)


def normalize_rows(x) -> np.ndarray:
    """Section 3.1 / 3.2: x / |x| per row in fp32: |x|^2 summed from dimension
    0 up, its correctly rounded square root, one division per element. An
    all-zero row stays zero."""
    x = np.asarray(x, dtype=F32)
    ss = np.zeros(x.shape[0], dtype=F32)
    for j in range(x.shape[1]):
        ss = ss + x[:, j] * x[:, j]
    nrm = np.sqrt(ss)
    out = np.zeros_like(x)
    nz = nrm > 0
    out[nz] = x[nz] / nrm[nz, None]
    return out


def pool_keys(kn, n_pool: int) -> np.ndarray:
    """Section 3.1 "Pooling": every n_pool consecutive unit keys summed (fp32,
    in position order) into one pool key. len(kn) must divide by n_pool."""
    kn = np.asarray(kn, dtype=F32)
    g = kn.shape[0] // n_pool
    acc = kn[0::n_pool][:g].copy()
    for r in range(1, n_pool):
        acc = acc + kn[r::n_pool][:g]
    return acc


# ------------------------------------------------------------------- Ward
def ward_cost(s_a, n_a: int, s_b, n_b: int) -> np.float32:
    """Ward's criterion for merging two buckets with member sums s_a, s_b and
    member counts n_a, n_b: n_a n_b / (n_a + n_b) |s_a/n_a - s_b/n_b|^2, each
    step one fp32 operation, the squared distance summed from dimension 0."""
    mu_a = np.asarray(s_a, dtype=F32) / F32(n_a)
    mu_b = np.asarray(s_b, dtype=F32) / F32(n_b)
    dist = F32(0.0)
    for j in range(mu_a.shape[0]):
        diff = F32(mu_a[j] - mu_b[j])
        dist = F32(dist + F32(diff * diff))
    w = F32(F32(n_a * n_b) / F32(n_a + n_b))
    return F32(w * dist)


def _ward_cost_matrix(S, n):
    """ward_cost for every pair of rows (the same fp32 steps, vectorised)."""
    mu = S / n.astype(F32)[:, None]
    A = S.shape[0]
    dist = np.zeros((A, A), dtype=F32)
    for j in range(S.shape[1]):
        diff = mu[:, None, j] - mu[None, :, j]
        dist = dist + diff * diff
    w = (n[:, None] * n[None, :]).astype(F32) / (n[:, None] + n[None, :]).astype(F32)
    return w * dist


def ward_block(pool, m: int, cap: int, record: bool = False):
    """Section 3.1 "Clustering": bottom-up Ward clustering of one cluster
    block's pool keys into m buckets.

    pool: fp32 [P, d] pool keys; cap: the most pool keys a bucket may hold
    (n_b^max / n_pool). Every round, each bucket finds its cheapest partner
    among the buckets it may merge with; every pair of buckets that are each
    other's cheapest partner merges (the lower index keeps the merged sums);
    rounds repeat until m buckets remain, merging only the cheapest pairs in a
    round that would overshoot.

    Returns (bucket [P] int64: the bucket number 0..m-1 of every pool key,
    sums fp32 [m, d], counts [m] in pool keys), plus the list of rounds, each a
    list of merged (a, b, cost), when record is set."""
    S = np.array(pool, dtype=F32, copy=True)
    P = S.shape[0]
    n = np.ones(P, dtype=np.int64)
    parent = np.arange(P)
    alive = np.ones(P, dtype=bool)
    rounds = []
    while alive.sum() > m:
        ids = np.flatnonzero(alive)
        A = ids.size
        cost = _ward_cost_matrix(S[ids], n[ids])
        fits = (n[ids][:, None] + n[ids][None, :]) <= cap
        np.fill_diagonal(fits, False)
        best = np.full(A, -1)
        for a in range(A):
            cand = np.flatnonzero(fits[a])
            if cand.size:
                best[a] = cand[np.argmin(cost[a, cand])]      # first minimum: the lower index
        pairs = [(float(cost[a, best[a]]), a, int(best[a])) for a in range(A)
                 if best[a] > a and best[best[a]] == a]
        if not pairs:
            raise RuntimeError("no bucket pair fits n_b^max; need n_b^max >= 2 n_cluster / m")
        pairs.sort()
        pairs = pairs[:A - m]
        done = []
        for c, a, b in pairs:
            ga, gb = ids[a], ids[b]
            S[ga] = S[ga] + S[gb]
            n[ga] += n[gb]
            alive[gb] = False
            parent[gb] = ga
            done.append((int(ga), int(gb), c))
        rounds.append(done)
    root = np.arange(P)
    for g in range(P):
        r = g
        while parent[r] != r:
            r = parent[r]
        root[g] = r
    ids = np.flatnonzero(alive)
    number = np.full(P, -1)
    number[ids] = np.arange(ids.size)
    out = (number[root], S[ids].copy(), n[ids].copy())
    return out + (rounds,) if record else out


# ------------------------------------------------------------- bucket cache
def build_buckets(k, n_pool: int, n_cluster: int, m: int, max_bucket_keys: int, n_blocks: int | None = None):
    """Section 3.1: the bucket cache of the complete cluster blocks of index
    keys k ([n_k, d], the bf16 values as fp32).

    Returns (centroids fp32 [n_blocks * m, d] holding bf16 values, bucket_off
    int64 [n_blocks * m], bucket_keys int64 [n_blocks * n_cluster]): bucket b
    = c * m + r lists its key positions at bucket_keys[bucket_off[b] :
    bucket_end(b)], ascending; block c's lists fill [c * n_cluster, (c + 1) *
    n_cluster)."""
    k = np.asarray(k, dtype=F32)
    if n_blocks is None:
        n_blocks = k.shape[0] // n_cluster
    d = k.shape[1]
    P = n_cluster // n_pool
    cap = max_bucket_keys // n_pool
    cent = np.zeros((n_blocks * m, d), dtype=F32)
    off = np.zeros(n_blocks * m, dtype=np.int64)
    keys = np.zeros(n_blocks * n_cluster, dtype=np.int64)
    for c in range(n_blocks):
        kn = normalize_rows(k[c * n_cluster:(c + 1) * n_cluster])
        bucket, sums, _ = ward_block(pool_keys(kn, n_pool), m, cap)
        cent[c * m:(c + 1) * m] = bf16_round(normalize_rows(sums))
        w = c * n_cluster
        for r in range(m):
            off[c * m + r] = w
            for g in np.flatnonzero(bucket == r):
                for e in range(n_pool):
                    keys[w] = c * n_cluster + g * n_pool + e
                    w += 1
    return cent, off, keys


def bucket_end(b: int, bucket_off, m: int, n_cluster: int) -> int:
    """End of bucket b's key list: the next bucket's start, or the end of its
    cluster block's lists for the block's last bucket."""
    c, r = divmod(b, m)
    return (c + 1) * n_cluster if r == m - 1 else int(bucket_off[b + 1])


# ------------------------------------------------------------------ search
def normalized_queries(q) -> np.ndarray:
    """Section 3.2 "Query normalisation", rounded to the bf16 scan operand."""
    return bf16_round(normalize_rows(q))


def bucket_scores(qn, cent, n_vis: int) -> np.ndarray:
    """Section 3.2 "Scoring": s_b = c_b . q for the first n_vis buckets, fp64
    over the bf16 operands."""
    return np.asarray(cent[:n_vis], dtype=np.float64) @ np.asarray(qn, dtype=np.float64)


def search_row(qn, pos: int, cent, bucket_off, bucket_keys, n_blocks: int, n_cluster: int, m: int,
               p: int, k: int, n_sink: int, n_window: int, return_buckets: bool = False):
    """Section 3.2 for the normalised query qn at position pos: the index row
    J (int64 [n_sink + n_window + k]) = the sinks, the window, then the k
    long-range keys the top-p buckets yield best first (keys the sinks or the
    window hold are skipped), then -1. With return_buckets, also the top-p
    bucket ids in expansion order."""
    n_vis = min(n_blocks, pos // n_cluster) * m
    s = bucket_scores(qn, cent, n_vis)
    order = np.lexsort((np.arange(n_vis), -s))[:p]
    sinks = list(range(min(n_sink, pos + 1)))
    w_lo = max(n_sink, pos - n_window + 1)
    window = list(range(w_lo, pos + 1))
    far = []
    for b in order:
        for key in bucket_keys[bucket_off[b]:bucket_end(int(b), bucket_off, m, n_cluster)]:
            key = int(key)
            if key < n_sink or key >= w_lo:
                continue
            if len(far) == k:
                break
            far.append(key)
        if len(far) == k:
            break
    row = sinks + window + far
    J = np.array(row + [-1] * (n_sink + n_window + k - len(row)), dtype=np.int64)
    return (J, order) if return_buckets else J
