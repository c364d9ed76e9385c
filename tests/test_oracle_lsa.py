"""Pins of the LSA semantic-search oracle (CPU only).

Each test ties the oracle to something other than itself: values worked by
hand (tests/golden/lsa_hand.json), an independent library (torch's bf16
rounding, scipy's Ward linkage), the definition of Ward's criterion as a
change of squared distances computed from the member points, or a special
case that reduces the search to a plain top-k.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

from oracle import lsa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "lsa_hand.json")


def _hand_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(4096).astype(np.float32),
                        # exact ties between two bf16 values, both parities
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 0.0, -0.0],
                                 dtype=np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    got = lsa.bf16_round(x)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_normalize_rows_unit_direction_and_zero_row():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 64)).astype(np.float32) * 3
    x[5] = 0
    y = lsa.normalize_rows(x)
    n = np.linalg.norm(y.astype(np.float64), axis=1)
    assert np.all(y[5] == 0)
    ok = np.arange(64) != 5
    assert np.allclose(n[ok], 1.0, atol=1e-6)
    ref = x[ok].astype(np.float64) / np.linalg.norm(x[ok].astype(np.float64), axis=1, keepdims=True)
    assert np.allclose(y[ok], ref, atol=1e-7)


def test_pool_keys_sums_consecutive_keys():
    rng = np.random.default_rng(3)
    kn = rng.standard_normal((24, 8)).astype(np.float32)
    for n_pool in (1, 2, 4, 8):
        got = lsa.pool_keys(kn, n_pool)
        ref = kn.astype(np.float64).reshape(24 // n_pool, n_pool, 8).sum(axis=1)
        assert got.shape == ref.shape
        assert np.allclose(got, ref, atol=1e-5)


def _sse(points):
    p = np.asarray(points, dtype=np.float64)
    return float(((p - p.mean(axis=0)) ** 2).sum())


def test_ward_cost_is_the_increase_of_squared_distances():
    """Ward's criterion by definition: SSE(a u b) - SSE(a) - SSE(b), each SSE
    the squared distances of the member points from their mean."""
    rng = np.random.default_rng(4)
    for na, nb in [(1, 1), (1, 3), (2, 5), (7, 4)]:
        a = rng.standard_normal((na, 16))
        b = rng.standard_normal((nb, 16)) + 0.5
        want = _sse(np.vstack([a, b])) - _sse(a) - _sse(b)
        got = float(lsa.ward_cost(a.sum(0).astype(np.float32), na, b.sum(0).astype(np.float32), nb))
        assert got == pytest.approx(want, rel=1e-5)


def _clusters_from_rounds(P, rounds):
    """Every cluster (as a frozenset of pool keys) formed by the merges."""
    members = {g: frozenset([g]) for g in range(P)}
    formed = set()
    heights = {}
    for rnd in rounds:
        for a, b, c in rnd:
            members[a] = members[a] | members[b]
            formed.add(members[a])
            heights[members[a]] = c
    return formed, heights


def test_ward_rounds_build_scipy_ward_hierarchy():
    """Ward's linkage is reducible, so merging mutually cheapest pairs in
    parallel rounds builds the same hierarchy as the textbook one-merge-at-a-
    time Ward linkage (scipy). Merge heights: scipy reports sqrt(2 cost)."""
    from scipy.cluster.hierarchy import linkage
    rng = np.random.default_rng(5)
    for trial in range(6):
        P = 12 + 4 * trial
        pts = (rng.standard_normal((P, 3)) + rng.integers(0, 4, size=(P, 1)) * 3.0).astype(np.float32)
        _, _, _, rounds = lsa.ward_block(pts, 1, P, record=True)
        formed, heights = _clusters_from_rounds(P, rounds)
        Z = linkage(pts.astype(np.float64), method="ward")
        members = {g: frozenset([g]) for g in range(P)}
        ref = {}
        for i, (u, v, h, _) in enumerate(Z):
            members[P + i] = members[int(u)] | members[int(v)]
            ref[members[P + i]] = h
        assert formed == set(ref)
        for cl, c in heights.items():
            assert np.sqrt(2.0 * c) == pytest.approx(ref[cl], rel=1e-4, abs=1e-5)


def _fp64_best(buckets, pts, cap):
    """Brute force: the cheapest fitting partner of every bucket, with the
    cost gap to the runner-up (fp64, from the member points)."""
    out = {}
    for a in buckets:
        costs = []
        for b in buckets:
            if b == a or len(buckets[a]) + len(buckets[b]) > cap:
                continue
            A, B = pts[sorted(buckets[a])], pts[sorted(buckets[b])]
            costs.append((_sse(np.vstack([A, B])) - _sse(A) - _sse(B), b))
        costs.sort()
        if costs:
            gap = costs[1][0] - costs[0][0] if len(costs) > 1 else np.inf
            out[a] = (costs[0][1], costs[0][0], gap)
    return out


@pytest.mark.parametrize("P,m,cap", [(32, 8, 8), (64, 16, 8), (40, 5, 16), (48, 12, 10)])
def test_ward_rounds_merge_mutually_cheapest_pairs_within_the_cap(P, m, cap):
    """Replays each round against a brute-force fp64 search over the current
    buckets: a merged pair is each other's cheapest fitting partner, a pair
    that is mutually cheapest (by a clear margin) merges unless the round
    merged enough cheaper pairs, and a last round takes the cheapest pairs."""
    rng = np.random.default_rng(P + m)
    pts = rng.standard_normal((P, 6)).astype(np.float32)
    bucket, sums, counts, rounds = lsa.ward_block(pts, m, cap, record=True)
    buckets = {g: {g} for g in range(P)}
    for rnd in rounds:
        best = _fp64_best(buckets, pts.astype(np.float64), cap)
        mutual = sorted((best[a][1], a, b) for a, (b, c, gap) in best.items()
                        if a < b and best.get(b, (None,))[0] == a)
        merged = {(a, b) for a, b, _ in rnd}
        for a, b, c in rnd:
            tight = min(best[a][2], best[b][2]) < 1e-4 * (1 + best[a][1])
            assert tight or (best[a][0] == b and best[b][0] == a)
        need = len(buckets) - m
        clear = all(min(best[a][2], best[b][2]) > 1e-4 * (1 + c) for c, a, b in mutual)
        if clear:
            assert merged == {(a, b) for _, a, b in mutual[:need]}
        for a, b, _ in rnd:
            buckets[a] |= buckets.pop(b)
    assert len(buckets) == m
    assert counts.max() <= cap
    assert sorted(np.bincount(bucket, minlength=m).tolist()) == sorted(counts.tolist())
    # bucket numbers follow the lowest pool key of each bucket
    lows = [min(np.flatnonzero(bucket == r)) for r in range(m)]
    assert lows == sorted(lows)
    assert np.allclose(sums, np.stack([pts[bucket == r].astype(np.float64).sum(0) for r in range(m)]),
                       atol=1e-4)


def test_ward_last_round_merges_only_the_cheapest_pairs():
    """Four tight pairs at spreads 0.01 < 0.02 < 0.03 < 0.04, far apart:
    all four are mutually cheapest in round 1, but m = 6 of 8 needs only two
    merges, the two tightest."""
    pts = []
    for i, s in enumerate([0.03, 0.01, 0.04, 0.02]):
        c = np.zeros(4, dtype=np.float32)
        c[i] = 10.0
        pts += [c, c + np.array([s, 0, 0, 0], dtype=np.float32)]
    bucket, _, _, rounds = lsa.ward_block(np.array(pts), 6, 8, record=True)
    assert len(rounds) == 1
    assert sorted((a, b) for a, b, _ in rounds[0]) == [(2, 3), (6, 7)]
    assert bucket.tolist() == [0, 1, 2, 2, 3, 4, 5, 5]


def test_ward_reaches_m_whenever_the_cap_allows_it():
    rng = np.random.default_rng(7)
    for P, m in [(128, 64), (128, 32), (64, 8)]:
        cap = 2 * P // m
        pts = rng.standard_normal((P, 8)).astype(np.float32)
        bucket, _, counts = lsa.ward_block(pts, m, cap)
        assert len(counts) == m and counts.max() <= cap and counts.sum() == P


@pytest.mark.parametrize("case", range(3))
def test_bucket_cache_and_search_hand_fixture(case):
    c = _hand_cases()[case]
    k = np.array(c["keys"], dtype=np.float32)
    cent, off, keys = lsa.build_buckets(k, c["n_pool"], c["n_cluster"], c["m"], c["max_bucket_keys"],
                                        c["n_blocks"])
    if "centroids" in c:
        assert cent.tolist() == c["centroids"]
    assert off.tolist() == c["bucket_off"]
    assert keys.tolist() == c["bucket_keys"]
    if "uncapped_bucket_off" in c:
        _, off2, keys2 = lsa.build_buckets(k, c["n_pool"], c["n_cluster"], c["m"], c["n_cluster"],
                                           c["n_blocks"])
        assert off2.tolist() == c["uncapped_bucket_off"]
        assert keys2.tolist() == c["uncapped_bucket_keys"]
    for q in c["queries"]:
        qn = lsa.normalized_queries(np.array([q["q"]], dtype=np.float32))[0]
        J = lsa.search_row(qn, q["pos"], cent, off, keys, c["n_blocks"], c["n_cluster"], c["m"], q["p"], q["k"],
                           c["n_sink"], c["n_window"])
        assert J.tolist() == q["J"]


def test_centroids_point_along_the_mean_of_their_unit_keys():
    rng = np.random.default_rng(8)
    k = rng.standard_normal((1024, 64)).astype(np.float32)
    n_pool, nc, m, cap = 4, 512, 64, 32
    cent, off, keys = lsa.build_buckets(k, n_pool, nc, m, cap)
    kn = k.astype(np.float64) / np.linalg.norm(k.astype(np.float64), axis=1, keepdims=True)
    for b in range(2 * m):
        mem = keys[off[b]:lsa.bucket_end(b, off, m, nc)]
        assert n_pool <= len(mem) <= cap and len(mem) % n_pool == 0
        mean = kn[mem].mean(0)
        cos = cent[b] @ mean / (np.linalg.norm(cent[b]) * np.linalg.norm(mean))
        assert cos > 1 - 1e-4
    # every key of every complete block is listed exactly once, blocks kept apart
    assert sorted(keys.tolist()) == list(range(1024))
    assert set(keys[:nc].tolist()) == set(range(nc))


def test_search_with_single_key_buckets_is_a_plain_top_k():
    """n_pool = 1 and m = n_cluster: no merges, each bucket is one key and its
    centroid the bf16 unit key, so the long-range part of J is the top-k of
    q . bf16(k / |k|) over the keys of earlier cluster blocks that neither a
    sink nor the window holds (ties to the lower position)."""
    rng = np.random.default_rng(9)
    d, nc, n_k = 16, 32, 160
    k = rng.standard_normal((n_k, d)).astype(np.float32)
    cent, off, keys = lsa.build_buckets(k, 1, nc, nc, 1)
    assert keys.tolist() == list(range(n_k // nc * nc))
    ku = k.astype(np.float64) / np.linalg.norm(k.astype(np.float64), axis=1, keepdims=True)
    kb = torch.from_numpy(ku.astype(np.float32)).to(torch.bfloat16).double().numpy()
    n_sink, n_w, kk = 3, 20, 12
    for pos in [40, 70, 100, 159]:
        q = rng.standard_normal(d).astype(np.float32)
        qn = lsa.normalized_queries(q[None])[0]
        J = lsa.search_row(qn, pos, cent, off, keys, n_k // nc, nc, nc, 10 ** 6, kk, n_sink, n_w)
        w_lo = max(n_sink, pos - n_w + 1)
        elig = [s for s in range((pos // nc) * nc) if not (s < n_sink or s >= w_lo)]
        sc = kb[elig] @ qn.astype(np.float64)
        ranked = sorted(range(len(elig)), key=lambda i: (-sc[i], elig[i]))[:kk]
        far = [elig[i] for i in ranked]
        head = list(range(n_sink)) + list(range(w_lo, pos + 1))
        assert J.tolist() == head + far + [-1] * (n_sink + n_w + kk - len(head) - len(far))


def test_search_rows_are_valid_best_first_expansions():
    """Invariants of any row: sinks then window, no repeats, only keys of
    earlier cluster blocks, only keys of the top-p buckets, and best first:
    every bucket ranked above the last one used gives all its uncovered keys."""
    rng = np.random.default_rng(10)
    d, n_pool, nc, m, cap = 32, 2, 64, 8, 16
    n_k = 640
    k = rng.standard_normal((n_k, d)).astype(np.float32)
    cent, off, keys = lsa.build_buckets(k, n_pool, nc, m, cap)
    nb = n_k // nc
    n_sink, n_w, p, kk = 4, 64, 12, 40
    for pos in rng.integers(0, n_k, size=40).tolist() + [nc - 1, nc, n_k - 1]:
        qn = lsa.normalized_queries(rng.standard_normal((1, d)).astype(np.float32))[0]
        J, order = lsa.search_row(qn, pos, cent, off, keys, nb, nc, m, p, kk, n_sink, n_w, return_buckets=True)
        assert len(J) == n_sink + n_w + kk
        w_lo = max(n_sink, pos - n_w + 1)
        head = list(range(min(n_sink, pos + 1))) + list(range(w_lo, pos + 1))
        assert J[:len(head)].tolist() == head
        far = [s for s in J[len(head):].tolist() if s >= 0]
        assert all(s < 0 for s in J[len(head) + len(far):])
        assert len(set(far)) == len(far) and not set(far) & set(head)
        assert all(s < (pos // nc) * nc for s in far)
        owner = {}
        for b in range(nb * m):
            for s in keys[off[b]:lsa.bucket_end(b, off, m, nc)]:
                owner[int(s)] = b
        used = [owner[s] for s in far]
        assert set(used) <= set(order.tolist())
        # buckets appear in rank order, each used one completely before the next
        rank = {b: i for i, b in enumerate(order.tolist())}
        assert [rank[b] for b in used] == sorted(rank[b] for b in used)
        avail = lambda b: [int(s) for s in keys[off[b]:lsa.bucket_end(b, off, m, nc)]
                           if not (s < n_sink or s >= w_lo)]
        for b in order.tolist():
            got = [s for s in far if owner[s] == b]
            if len(far) < kk or (used and rank[b] < rank[used[-1]]):
                assert got == avail(b)
        assert len(far) == min(kk, sum(len(avail(b)) for b in order.tolist()))


def test_ward_refuses_a_cap_below_twice_the_mean_bucket():
    """Below n_b^max = 2 n_cluster / m the cap can leave no pair that fits
    before m buckets remain (here 32 pool keys, m = 8, at most 4 per bucket
    would need a perfect split); the oracle says so instead of looping."""
    pts = np.random.default_rng(11).standard_normal((32, 4)).astype(np.float32)
    with pytest.raises(RuntimeError):
        lsa.ward_block(pts, 8, 4)


def test_ward_partner_ties_go_to_the_lower_index():
    """Three points 0, 1, 2 on a line: the middle one is equally cheap to
    merge with either neighbour (cost 0.5 exactly); its partner is the lower
    index, so with m = 2 the buckets are {0, 1} and {2}."""
    pts = np.array([[0, 0], [1, 0], [2, 0]], dtype=np.float32)
    assert lsa.ward_cost(pts[0], 1, pts[1], 1) == lsa.ward_cost(pts[1], 1, pts[2], 1) == np.float32(0.5)
    bucket, _, counts = lsa.ward_block(pts, 2, 3)
    assert bucket.tolist() == [0, 0, 1] and counts.tolist() == [2, 1]


def test_ward_properties_on_random_blocks():
    """Many random small blocks: exactly m buckets, none above the cap, every
    pool key in one bucket, buckets numbered by their lowest pool key, sums
    equal to their members' sums; with no cap and m = 1, the clusters formed
    are those of scipy's Ward linkage."""
    from hypothesis import given, settings, strategies as st
    from scipy.cluster.hierarchy import linkage

    @settings(max_examples=60, deadline=None, derandomize=True, database=None)
    @given(P=st.integers(2, 24), dim=st.integers(1, 5), m_frac=st.floats(0.05, 1.0), extra=st.integers(0, 4),
           seed=st.integers(0, 2 ** 31 - 1))
    def check(P, dim, m_frac, extra, seed):
        pts = np.random.default_rng(seed).standard_normal((P, dim)).astype(np.float32)
        m = max(1, min(P, int(round(m_frac * P))))
        cap = -(-2 * P // m) + extra
        bucket, sums, counts = lsa.ward_block(pts, m, cap)
        assert len(counts) == m and counts.max() <= max(cap, 1) and counts.sum() == P
        assert sorted(set(bucket.tolist())) == list(range(m))
        lows = [int(np.flatnonzero(bucket == r)[0]) for r in range(m)]
        assert lows == sorted(lows)
        assert np.allclose(sums, np.stack([pts[bucket == r].astype(np.float64).sum(0) for r in range(m)]),
                           atol=1e-4)
        if P >= 3:
            _, _, _, rounds = lsa.ward_block(pts, 1, P, record=True)
            formed, _ = _clusters_from_rounds(P, rounds)
            Z = linkage(pts.astype(np.float64), method="ward")
            members = {g: frozenset([g]) for g in range(P)}
            ref = set()
            for i, (u, v, _, _) in enumerate(Z):
                members[P + i] = members[int(u)] | members[int(v)]
                ref.add(members[P + i])
            assert formed == ref

    check()
