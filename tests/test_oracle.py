"""Pins of the CPU oracle against things other than itself: values worked by
hand (tests/golden), exact integer arithmetic, torch's own e4m3 decoder,
brute force on tiny rows, and closed forms of attention. CPU only."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle.fp8 import e4m3_decode, e4m3_decode_table, e4m3_quantize_rne
from oracle.indexer import scores_row
from oracle.topk import topk_row, topk_row_bruteforce
from oracle.attention import sparse_attention_row, dense_causal_attention_row
from oracle.two_stage import pool_block_keys, keep_blocks_row
from workloads import WORKLOADS, PrefillInputs, DecodeInputs, sample_rows

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------- fp8
def test_e4m3_table_matches_torch_decoder():
    tab = e4m3_decode_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(tab)
    assert list(np.flatnonzero(nan)) == [0x7F, 0xFF]
    assert np.array_equal(tab[~nan], ref[~nan])


def test_e4m3_hand_values():
    assert e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9
    assert e4m3_decode(np.array([0x08]))[0] == 2.0 ** -6
    assert e4m3_decode(np.array([0x38]))[0] == 1.0
    assert e4m3_decode(np.array([0xB8]))[0] == -1.0
    assert e4m3_decode(np.array([0x3F]))[0] == 1.875


def test_e4m3_quantize_roundtrip_ties_and_saturation():
    tab = e4m3_decode_table()
    codes = np.array([c for c in range(256) if not np.isnan(tab[c]) and c != 0x80], dtype=np.uint8)
    assert np.array_equal(e4m3_quantize_rne(tab[codes]), codes)
    # ties go to the even code: 1.0625 between 1.0 (0x38) and 1.125 (0x39)
    assert e4m3_quantize_rne(np.array([1.0625]))[0] == 0x38
    assert e4m3_quantize_rne(np.array([1.1875]))[0] == 0x3A
    assert e4m3_quantize_rne(np.array([-1.1875]))[0] == 0xBA
    assert e4m3_quantize_rne(np.array([500.0, -1e9]))[0] == 0x7E
    assert e4m3_quantize_rne(np.array([-1e9]))[0] == 0xFE
    # random values: nearest representable (torch's cast rounds to nearest even)
    x = np.random.default_rng(0).standard_normal(20000).astype(np.float32) * 60
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(e4m3_quantize_rne(x), ref)


# ----------------------------------------------------------------- indexer
def test_indexer_hand_worked_example():
    g = json.load(open(os.path.join(GOLD, "indexer_hand.json")))
    s = scores_row(np.array(g["q"], float), None, np.array(g["keys"], float), None, np.array(g["w"]))
    assert s.tolist() == g["scores"]
    assert topk_row(s, 2).tolist() == g["top2"]


def _int_dot_e4m3(qb, kb):
    """Exact dot of two e4m3 byte vectors with Python integers (values * 2^9)."""
    tab = e4m3_decode_table()
    return sum(int(tab[a] * 512) * int(tab[b] * 512) for a, b in zip(qb, kb))


def test_indexer_fp8_dot_is_exact_integer_arithmetic():
    rng = np.random.default_rng(1)
    good = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    qb = rng.choice(good, size=(3, 128))
    kb = rng.choice(good, size=(5, 128))
    # one head, weight 1, unit scales: score = ReLU(dot); dot exact in fp64
    for h in range(3):
        s = scores_row(e4m3_decode(qb[h:h + 1]), None, e4m3_decode(kb), None, np.array([1.0]))
        for j in range(5):
            exact = Fraction(_int_dot_e4m3(qb[h], kb[j]), 2 ** 18)
            want = np.float32(float(max(exact, 0)))
            assert s[j] == want
    # extreme magnitudes: 128 products of 448*448 stay exact
    big = np.full((1, 128), 0x7E, dtype=np.uint8)
    s = scores_row(e4m3_decode(big), None, e4m3_decode(big), None, np.array([1.0]))
    assert s[0] == np.float32(448.0 * 448.0 * 128)


def test_indexer_scales_applied_per_head_and_per_key():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((4, 16))
    k = rng.standard_normal((9, 16))
    sq = 2.0 ** rng.uniform(-6, 6, 4)        # scales far apart: a mixed-up scale fails
    sk = 2.0 ** rng.uniform(-6, 6, 9)
    w = rng.uniform(0, 1, 4)
    got = scores_row(q, sq, k, sk, w)
    # explicit loops over heads and keys
    for j in range(9):
        tot = 0.0
        for h in range(4):
            a = sum(q[h, i] * k[j, i] for i in range(16)) * sq[h] * sk[j]
            tot += w[h] * max(a, 0.0)
        assert abs(float(got[j]) - tot) <= 1e-6 * max(1.0, abs(tot))


def test_indexer_invariants():
    rng = np.random.default_rng(3)
    q, k, w = rng.standard_normal((6, 32)), rng.standard_normal((50, 32)), rng.uniform(0, 1, 6)
    s = scores_row(q, None, k, None, w)
    assert (s >= 0).all()
    assert np.array_equal(scores_row(q, None, k, None, 2 * w), 2 * s)      # exact (power of 2)
    perm = rng.permutation(6)
    assert np.allclose(scores_row(q[perm], None, k, None, w[perm]), s, rtol=1e-6)
    # ReLU: a head contributes only where its dot is positive
    only0 = scores_row(q[:1], None, k, None, w[:1])
    dots = k @ q[0]
    assert np.allclose(only0, np.where(dots > 0, w[0] * dots, 0.0), rtol=1e-6)


def test_indexer_fp8_contract_tolerance_against_prequant_rows():
    """Scores from the encoded rows (bytes + scales) stay within 2e-2 of the
    row max against the fp32 rows before encoding, on rows with >= 64 keys.
    (With 3 mantissa bits the encoding itself moves a single score by up to
    ~5% when a row holds only a few keys; the contract tolerance therefore
    applies to the GPU against the oracle on the same bytes.)"""
    wl = WORKLOADS["prefill_t16k"].with_(T=600)
    inp = PrefillInputs(wl, "cpu", seed=5)
    host = inp.to_host()
    rows = [63, 64, 299, 599]
    got = oracle.scores_rows(host, rows)
    kf = inp.k_f32.double().numpy()
    for t in rows:
        qf = inp.q_f32_rows(t, t + 1)[0].double().numpy()
        ref = scores_row(qf, None, kf[:t + 1], None, host["w"][t].double().numpy())
        err = np.abs(got[t].astype(np.float64) - ref.astype(np.float64)).max()
        assert err <= 2e-2 * np.abs(ref).max()


# -------------------------------------------------------------------- top-k
def test_topk_ties_golden():
    g = json.load(open(os.path.join(GOLD, "topk_ties.json")))
    for c in g["cases"]:
        s = np.array(c["scores"], dtype=np.float32)
        assert topk_row(s, c["k"]).tolist() == c["expect"], c["why"]


@pytest.mark.parametrize("k", [1, 8, 63, 64])
def test_topk_sort_equals_bruteforce_tiny(k):
    wl = WORKLOADS["tiny_t512"].with_(T=64)
    host = PrefillInputs(wl, "cpu", seed=7).to_host()
    rows = oracle.scores_rows(host, range(64))
    for t, s in rows.items():
        a = set(topk_row(s, k).tolist())
        b = set(topk_row_bruteforce(s, k).tolist())
        assert a == b
        assert len(a) == min(k, t + 1)


def test_topk_bruteforce_with_duplicates():
    rng = np.random.default_rng(4)
    for _ in range(50):
        s = rng.integers(0, 4, size=rng.integers(1, 40)).astype(np.float32)
        k = int(rng.integers(1, 45))
        assert topk_row(s, k).tolist() == sorted(topk_row_bruteforce(s, k).tolist(),
                                                 key=lambda i: (-s[i], i))


# ---------------------------------------------------------------- attention
def test_attention_k_covers_all_visible_equals_dense_causal():
    wl = WORKLOADS["tiny_t512"].with_(T=96)
    inp = PrefillInputs(wl, "cpu", seed=11)
    host = inp.to_host()
    res = oracle.prefill_rows(host, [0, 1, 37, 95], k=512)
    for t, r in res.items():
        assert (r["idx"] >= 0).sum() == t + 1
        O_d, lse_d = dense_causal_attention_row(host["Q"][t].double().numpy(),
                                                host["K"].double().numpy(), host["V"].double().numpy(), t)
        assert np.abs(r["O"] - O_d).max() <= 1e-12
        assert np.abs(r["lse"] - lse_d).max() <= 1e-12


def test_attention_closed_forms():
    rng = np.random.default_rng(5)
    K, V = rng.standard_normal((40, 8)), rng.standard_normal((40, 8))
    idx = np.array([3, 17, 5, -1, 22, -1])
    # all-equal logits (Q = 0): output is the mean of the selected V rows
    O, lse = sparse_attention_row(np.zeros((2, 8)), K, V, idx)
    assert np.allclose(O, V[[3, 17, 5, 22]].mean(0)[None, :], atol=1e-15)
    assert np.allclose(lse, math.log(4))
    # a single selected key: output is its V row, lse its scaled logit
    Q = rng.standard_normal((3, 8))
    O, lse = sparse_attention_row(Q, K, V, np.array([-1, 9, -1]))
    assert np.allclose(O, V[9][None, :], atol=1e-15)
    assert np.allclose(lse, Q @ K[9] / math.sqrt(8))
    # order of J does not matter
    O1, _ = sparse_attention_row(Q, K, V, idx)
    O2, _ = sparse_attention_row(Q, K, V, idx[::-1].copy())
    assert np.allclose(O1, O2, atol=1e-14)


# ------------------------------------------------------------ planted keys
def test_planted_keys_land_in_topk_tiny():
    wl = WORKLOADS["tiny_t512"]
    inp = PrefillInputs(wl, "cpu", seed=0)
    host = inp.to_host()
    rows = range(wl.k + 1, wl.T, 3)           # queries with more than k visible keys
    res = oracle.prefill_rows(host, rows, k=wl.k, attention=False)
    hit = tot = 0
    for t, r in res.items():
        pl = inp.planted_for_row(t)
        sel = set(r["idx"].tolist())
        hit += sum(int(p) in sel for p in pl)
        tot += len(pl)
    assert tot > 500
    # random keys would land with probability k/(t+1) < 0.5
    assert hit / tot >= 0.97, hit / tot


def test_planted_keys_land_in_topk_fp8():
    wl = WORKLOADS["prefill_t16k"].with_(T=2600, k=256)
    inp = PrefillInputs(wl, "cpu", seed=1)
    host = inp.to_host()
    rows = sample_rows(wl.T, 24, seed=1, k=wl.k)
    res = oracle.prefill_rows(host, [t for t in rows if t > wl.k], k=wl.k, attention=False)
    hit = tot = 0
    for t, r in res.items():
        pl = inp.planted_for_row(t)
        sel = set(r["idx"].tolist())
        hit += sum(int(p) in sel for p in pl)
        tot += len(pl)
    assert tot > 100 and hit == tot


# ---------------------------------------------------------------- two-stage
def test_pool_block_keys_exact_mean():
    rng = np.random.default_rng(6)
    good = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    kb = rng.choice(good[(good & 0x78) < 0x50], size=(128, 8))   # moderate magnitudes
    sk = rng.uniform(0.01, 0.02, 128).astype(np.float32)
    blk, bsc = pool_block_keys(kb, sk, block=64)
    tab = e4m3_decode_table()
    for b in range(2):
        for j in range(8):
            # exact rational mean, rounded once to fp32
            tot = sum(Fraction(tab[kb[s, j]]) * Fraction(float(sk[s])) for s in range(64 * b, 64 * b + 64))
            m = np.float32(float(tot / 64))
            mean_all = [np.float32(float(sum(Fraction(tab[kb[s, jj]]) * Fraction(float(sk[s]))
                                             for s in range(64 * b, 64 * b + 64)) / 64)) for jj in range(8)]
            scale = np.float32(np.float32(max(abs(v) for v in mean_all)) / np.float32(448.0))
            assert bsc[b] == scale
            assert blk[b, j] == e4m3_quantize_rne(np.array([np.float32(m / scale)]))[0]


def test_keep_blocks_rule():
    assert keep_blocks_row(np.zeros(0), 10, 64, 64).tolist() == [0]
    assert keep_blocks_row(np.zeros(1), 64, 64, 64).tolist() == [0, 1]
    sc = np.arange(100, dtype=np.float32)            # higher block id -> higher score
    kept = keep_blocks_row(sc, 100 * 64 + 5, 64, 4)
    assert kept.tolist() == [0, 98, 99, 100]           # 2 forced + best 2 of 1..99
    kept = keep_blocks_row(sc, 99 * 64, 64, 4)        # cur=99: others 1..98, best 2 = 97, 98
    assert kept.tolist() == [0, 97, 98, 99]
    eq = np.ones(50, dtype=np.float32)                # ties -> lower block ids
    assert keep_blocks_row(eq, 50 * 64, 64, 5).tolist() == [0, 1, 2, 3, 50]


def test_two_stage_equals_flat_when_all_blocks_kept():
    wl = WORKLOADS["two_stage_t64k"].with_(T=1500, k=128, topics=4, topic_run=256)
    host = PrefillInputs(wl, "cpu", seed=2).to_host()
    rows = [0, 63, 64, 700, 1499]
    flat = oracle.prefill_rows(host, rows, k=wl.k, attention=False)
    # fewer than 64 blocks exist below t < 4096: two-stage keeps them all
    two = oracle.prefill_rows(host, rows, k=wl.k, mode="two_stage", attention=False)
    for t in rows:
        assert np.array_equal(flat[t]["idx"], two[t]["idx"])
    # and with keep = all blocks at a larger T
    two_all = oracle.prefill_rows(host, rows, k=wl.k, mode="two_stage", keep=10 ** 6, attention=False)
    for t in rows:
        assert np.array_equal(flat[t]["idx"], two_all[t]["idx"])


def test_two_stage_filters_by_topic():
    wl = WORKLOADS["two_stage_t64k"].with_(T=12288, k=512, keep_blocks=16)
    inp = PrefillInputs(wl, "cpu", seed=3)
    host = inp.to_host()
    res = oracle.prefill_rows(host, [12287, 9000, 6000], k=wl.k, mode="two_stage", keep=16,
                              attention=False)
    for t, r in res.items():
        topic = inp.query_topic[t]
        kept_topics = [inp.run_topic[(b * 64) // wl.topic_run] for b in r["kept"][1:-1]]
        # every non-forced kept block comes from the query's own topic
        assert all(x == topic for x in kept_topics), (t, topic, kept_topics)


# ------------------------------------------------------------------ decode
def test_decode_equals_last_prefill_row():
    wl = WORKLOADS["prefill_t16k"].with_(T=700, k=64)
    pin = PrefillInputs(wl, "cpu", seed=9)
    host = pin.to_host()
    T = wl.T
    pre = oracle.prefill_rows(host, [T - 1], k=wl.k)[T - 1]
    dec_host = {
        "q_idx": host["q_idx"][T - 1:T], "q_scale": host["q_scale"][T - 1:T], "w": host["w"][T - 1:T],
        "k_idx": host["k_idx"][None], "k_scale": host["k_scale"][None],
        "Q": host["Q"][T - 1:T], "K": host["K"][None], "V": host["V"][None],
        "seq_lens": torch.tensor([T], dtype=torch.int32),
    }
    dec = oracle.decode_rows(dec_host, [0], k=wl.k)[0]
    assert np.array_equal(dec["idx"], pre["idx"])
    assert np.abs(dec["O"] - pre["O"]).max() == 0.0


# -------------------------------------------------------------- generator
def test_generator_is_seeded_and_shaped():
    wl = WORKLOADS["tiny_t512"]
    a, b = PrefillInputs(wl, "cpu", seed=3), PrefillInputs(wl, "cpu", seed=3)
    assert torch.equal(a.q_idx, b.q_idx) and torch.equal(a.V, b.V)
    c = PrefillInputs(wl, "cpu", seed=4)
    assert not torch.equal(a.q_idx, c.q_idx)
    assert a.q_idx.shape == (512, 4, 32) and a.q_idx.dtype == torch.bfloat16
    d = DecodeInputs(WORKLOADS["decode_b64_l128k"].with_(batch=2, L=300), "cpu", seed=1)
    assert d.k_idx.shape == (2, 300, 128) and d.k_idx.dtype == torch.uint8
    rows = sample_rows(5000, 40, seed=0, k=256)
    for must in (0, 1, 255, 256, 257, 4999):
        assert must in rows


def test_quantize_rows_hand_values():
    """Per-row e4m3 encoding, values worked out from the format's definition
    (bias 7, 3 mantissa bits): 448 = 0x7E, 224 = 1.75 * 2^7 = 0x76, 1 = 0x38,
    0.75 = 1.5 * 2^-1 = 0x34; 1.0625 lies halfway between 1 (0x38) and 1.125
    (0x39) and 1.1875 halfway between 1.125 and 1.25 (0x3A): ties go to the
    even byte."""
    b, s = oracle.quantize_rows(np.array([[448.0, -224.0, 1.0, 0.0],
                                          [896.0, 1.5, 0.0, -896.0],
                                          [0.0, 0.0, 0.0, 0.0],
                                          [448.0, 1.0625, 1.1875, -1.0625]], dtype=np.float32))
    assert s.tolist() == [1.0, 2.0, 1.0, 1.0]
    assert b.tolist() == [[0x7E, 0xF6, 0x38, 0x00],
                          [0x7E, 0x34, 0x00, 0xFE],
                          [0x00, 0x00, 0x00, 0x00],
                          [0x7E, 0x38, 0x3A, 0xB8]]


def test_expand_sinks_window_hand_rows():
    """Position 10, two sinks, a window of three: sinks 0 1, window 8 9 10,
    then the selected keys neither covers (5 and 7; 9, 0, 1 and 10 are
    covered, -1 is dropped), then -1. Position 1: only the two sinks."""
    from oracle.pipeline import expand_sinks_window_row
    r = expand_sinks_window_row([9, 0, 5, -1, 7, 1, 10], 10, 2, 3)
    assert r.tolist() == [0, 1, 8, 9, 10, 5, 7, -1, -1, -1, -1, -1]
    r = expand_sinks_window_row([0, 1, -1], 1, 2, 3)
    assert r.tolist() == [0, 1, -1, -1, -1, -1, -1, -1]
    r = expand_sinks_window_row([3, 40, 2], 50, 0, 0)     # no sinks, no window: the selection unchanged
    assert r.tolist() == [3, 40, 2]
