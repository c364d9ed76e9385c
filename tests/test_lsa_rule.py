"""The LSA row comparison rule (tests/helpers.py: check_lsa_row) pinned on
the CPU with the oracle: a row that reorders two buckets of equal score is
accepted, and rows with the mistakes a device could make (buckets out of
score order, a skipped bucket, keys out of list order, a duplicate) are
rejected."""
import numpy as np
import pytest

from helpers import check_lsa_row
from oracle import lsa

N_POOL, N_CLUSTER, M, CAP = 4, 64, 8, 16
P, K, N_SINK, N_WINDOW = 10, 40, 4, 32


def _expand(order, pos, off, keys):
    """The expansion of the pages' flat search for an explicit bucket order
    (the oracle's own loop, with the order given instead of sorted)."""
    w_lo = max(N_SINK, pos - N_WINDOW + 1)
    far = []
    for b in order:
        end = (b // M + 1) * N_CLUSTER if b % M == M - 1 else int(off[b + 1])
        for key in keys[off[b]:end]:
            if int(key) < N_SINK or int(key) >= w_lo:
                continue
            if len(far) == K:
                break
            far.append(int(key))
        if len(far) == K:
            break
    row = list(range(min(N_SINK, pos + 1))) + list(range(w_lo, pos + 1)) + far
    return np.array(row + [-1] * (N_SINK + N_WINDOW + K - len(row)), dtype=np.int64)


@pytest.fixture(scope="module")
def case():
    rng = np.random.default_rng(3)
    T = 512
    k_idx = rng.standard_normal((T, 64)).astype(np.float32)
    cent, off, keys = lsa.build_buckets(k_idx, N_POOL, N_CLUSTER, M, CAP)
    qn = lsa.normalized_queries(rng.standard_normal((1, 64)).astype(np.float32))[0]
    pos, nb = 500, T // N_CLUSTER
    n_vis = min(nb, pos // N_CLUSTER) * M
    s = lsa.bucket_scores(qn, cent, n_vis)
    order = list(np.lexsort((np.arange(n_vis), -s))[:P])
    return cent, off, keys, qn, pos, nb, order


def _check(row, want, qn, pos, cache, nb):
    return check_lsa_row(row, want, qn, pos, cache, nb, N_CLUSTER, M, P, N_SINK, N_WINDOW, "row")


def test_exact_row_passes(case):
    cent, off, keys, qn, pos, nb, order = case
    want = lsa.search_row(qn, pos, cent, off, keys, nb, N_CLUSTER, M, P, K, N_SINK, N_WINDOW)
    assert np.array_equal(_expand(order, pos, off, keys), want)      # the test's expansion is the oracle's
    assert _check(want, want, qn, pos, (cent, off, keys), nb) is False


def test_tied_buckets_may_come_in_either_order(case):
    cent, off, keys, qn, pos, nb, order = case
    c2 = cent.copy()
    c2[order[2]] = c2[order[1]]                                       # two buckets of exactly equal score
    want = lsa.search_row(qn, pos, c2, off, keys, nb, N_CLUSTER, M, P, K, N_SINK, N_WINDOW)
    n_vis = min(nb, pos // N_CLUSTER) * M
    s = lsa.bucket_scores(qn, c2, n_vis)
    o2 = list(np.lexsort((np.arange(n_vis), -s))[:P])
    i, j = o2.index(order[1]), o2.index(order[2])
    o2[i], o2[j] = o2[j], o2[i]
    swapped = _expand(o2, pos, off, keys)
    assert not np.array_equal(swapped, want)
    assert _check(swapped, want, qn, pos, (c2, off, keys), nb) is True


@pytest.mark.parametrize("mistake", ["order", "skip", "keys", "duplicate"])
def test_device_mistakes_are_rejected(case, mistake):
    cent, off, keys, qn, pos, nb, order = case
    want = lsa.search_row(qn, pos, cent, off, keys, nb, N_CLUSTER, M, P, K, N_SINK, N_WINDOW)
    head = N_SINK + N_WINDOW
    if mistake == "order":                                            # two buckets of distinct scores swapped
        o = list(order)
        o[0], o[1] = o[1], o[0]
        bad = _expand(o, pos, off, keys)
    elif mistake == "skip":                                           # the second best bucket left out
        bad = _expand(order[:1] + order[2:], pos, off, keys)
    elif mistake == "keys":                                           # two keys of one bucket exchanged
        bad = want.copy()
        bad[head], bad[head + 1] = bad[head + 1], bad[head]
    else:                                                             # a key listed twice
        bad = want.copy()
        bad[head + 3] = bad[head + 2]
    assert not np.array_equal(bad, want)
    with pytest.raises(AssertionError):
        _check(bad, want, qn, pos, (cent, off, keys), nb)
