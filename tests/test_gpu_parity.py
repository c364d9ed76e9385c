"""Parity of the CUDA path (through the C ABI) with the CPU oracle on the
same seeded inputs. Needs a B200."""
import numpy as np
import pytest
import torch

import oracle
from oracle.topk import topk_row
from oracle.pipeline import attention_rows, decode_attention_row
from workloads import WORKLOADS, PrefillInputs, DecodeInputs, sample_rows
from helpers import check_topk_row, check_scores_row, check_attention_row, SCORE_GATE

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import ensure_built
    ensure_built()
    import indexer_selected_top_b200 as m
    return m


def _gpu(t):
    return None if t is None else t.cuda()


# ------------------------------------------------------------------ indexer
def _check_table(sa, wl, seed, rows=None, q_pos0=0, n_q=None, tol=2e-2):
    inp = PrefillInputs(wl, "cuda", seed=seed)
    host = inp.to_host()
    T = wl.T
    n_q = T - q_pos0 if n_q is None else n_q
    q = inp.q_idx[q_pos0:q_pos0 + n_q]
    qs = None if inp.q_scale is None else inp.q_scale[q_pos0:q_pos0 + n_q]
    w = inp.w[q_pos0:q_pos0 + n_q]
    table = sa.index_scores(q, qs, inp.k_idx, inp.k_scale, w, q_pos0=q_pos0)
    torch.cuda.synchronize()
    tab = table.cpu().numpy()
    rows = range(n_q) if rows is None else rows
    ref = oracle.scores_rows(host, [q_pos0 + r for r in rows])
    worst = 0.0
    for r in rows:
        p = q_pos0 + r
        o = ref[p]
        g = tab[r, :p + 1]
        worst = max(worst, check_scores_row(g, o, tol, f"row {p}"))
        check_scores_row(g, o, SCORE_GATE, f"row {p} (gate)")
        assert np.isneginf(tab[r, p + 1:]).all(), f"row {p}: invisible entries not -inf"
    return tab, ref, worst


def test_index_scores_bf16_tiny(sa):
    _check_table(sa, WORKLOADS["tiny_t512"], seed=0, tol=2e-3)


def test_index_scores_fp8_ragged(sa):
    wl = WORKLOADS["prefill_t16k"].with_(T=1000)
    _check_table(sa, wl, seed=1, tol=2e-2)


def test_index_scores_fp8_offset_rows(sa):
    wl = WORKLOADS["prefill_t16k"].with_(T=1000)
    _check_table(sa, wl, seed=2, q_pos0=700, n_q=300, tol=2e-2)


# -------------------------------------------------------------------- top-k
def _topk_exact(sa, table, k, q_pos0=0):
    t = torch.from_numpy(table).cuda()
    idx = sa.topk(t, k, q_pos0=q_pos0).cpu().numpy()
    for r in range(table.shape[0]):
        n = min(table.shape[1], q_pos0 + r + 1)
        want = topk_row(table[r, :n], k)
        got = idx[r][idx[r] >= 0]
        assert sorted(got.tolist()) == sorted(want.tolist()), f"row {r}"
        assert (idx[r][len(got):] == -1).all()


def test_topk_exact_with_ties(sa):
    rng = np.random.default_rng(0)
    tab = rng.integers(0, 50, size=(37, 1000)).astype(np.float32)
    _topk_exact(sa, tab, 100)
    _topk_exact(sa, tab, 1)
    _topk_exact(sa, tab, 999, q_pos0=500)


def test_topk_large_rows_bucket_paths(sa):
    rng = np.random.default_rng(1)
    n = 131072
    rows = [
        rng.standard_normal(n).astype(np.float32),                     # distinct values
        rng.integers(0, 4, size=n).astype(np.float32),                 # huge ties at the cut
        np.full(n, 7.0, dtype=np.float32),                             # all equal
        np.where(rng.random(n) < 0.5, 0.0, -0.0).astype(np.float32),   # +0 / -0 equal
        (rng.standard_normal(n) * 1e-3 + 5).astype(np.float32),        # narrow band
    ]
    tab = np.stack(rows)
    _topk_exact(sa, tab, 2048, q_pos0=n)
    _topk_exact(sa, tab, 20000, q_pos0=n)


# ---------------------------------------------------------------- attention
def _attn_case(sa, n_q, n_k, hq, dh, k, seed, std=None, decode=False):
    g = torch.Generator(device="cuda").manual_seed(seed)
    std = std or 1.0 / np.sqrt(dh)
    if decode:
        K = (torch.randn(n_q, n_k, dh, generator=g, device="cuda") * std).bfloat16()
        V = (torch.randn(n_q, n_k, dh, generator=g, device="cuda") * std).bfloat16()
    else:
        K = (torch.randn(n_k, dh, generator=g, device="cuda") * std).bfloat16()
        V = (torch.randn(n_k, dh, generator=g, device="cuda") * std).bfloat16()
    Q = (torch.randn(n_q, hq, dh, generator=g, device="cuda") * std).bfloat16()
    rng = np.random.default_rng(seed)
    idx = np.full((n_q, k), -1, dtype=np.int32)
    for t in range(n_q):
        m = int(rng.integers(0, k + 1)) if t % 3 == 0 else k
        m = min(m, n_k)
        idx[t, :m] = rng.choice(n_k, size=m, replace=False)
        rng.shuffle(idx[t])          # -1 anywhere: the kernel must skip them
    out, lse = sa.sparse_attn(Q, K, V, torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    out, lse = out.float().cpu().numpy(), lse.cpu().numpy()
    Qh = Q.double().cpu().numpy()
    Kh, Vh = K.double().cpu().numpy(), V.double().cpu().numpy()
    for t in range(n_q):
        if decode:
            o, l = oracle.sparse_attention_row(Qh[t], Kh[t], Vh[t], idx[t])
        else:
            o, l = oracle.sparse_attention_row(Qh[t], Kh, Vh, idx[t])
        check_attention_row(out[t], o, lse[t], l, f"row {t}")


def test_sparse_attn_prefill_shapes(sa):
    _attn_case(sa, 40, 3000, 16, 128, 2048, seed=0)
    _attn_case(sa, 40, 500, 8, 64, 64, seed=1)
    _attn_case(sa, 9, 100, 16, 64, 37, seed=2)


def test_sparse_attn_sharp_softmax(sa):
    # unscaled N(0,1) Q/K: logits of order 10, exercises the running-max rescale
    _attn_case(sa, 24, 4000, 16, 128, 2048, seed=3, std=1.0)


def test_sparse_attn_decode_splits(sa):
    _attn_case(sa, 5, 3000, 16, 128, 2048, seed=4, decode=True)
    _attn_case(sa, 3, 700, 16, 128, 600, seed=5, decode=True, std=1.0)


# ------------------------------------------------------------------ prefill
def _check_prefill(sa, wl, seed, rows, mode="flat", k=None, keep=64, chunk_rows=0, flat_path="auto", hook=0,
                   status=None, inp=None):
    k = k or wl.k
    inp = inp or PrefillInputs(wl, "cuda", seed=seed)
    host = inp.to_host()
    pre = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, k, mode=mode,
                     keep_blocks=keep, chunk_rows=chunk_rows, flat_path=flat_path, test_hook=hook, status=status)
    out, lse, idx = pre()
    torch.cuda.synchronize()
    out, lse, idx = out.float().cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()
    ref = oracle.prefill_rows(host, rows, k, mode=mode, keep=keep, attention=False)
    for t in rows:
        r = ref[t]
        check_topk_row(idx[t], r["cand"], r["scores"], k, f"row {t}")
    att = attention_rows(host, {t: idx[t] for t in rows})
    for t in rows:
        check_attention_row(out[t], att[t][0], lse[t], att[t][1], f"row {t}")
    return inp, host, idx, ref


def test_prefill_flat_tiny_all_rows(sa):
    wl = WORKLOADS["tiny_t512"]
    _check_prefill(sa, wl, 0, range(wl.T))


def test_prefill_flat_fp8_ragged(sa):
    wl = WORKLOADS["prefill_t16k"].with_(T=2500)
    rows = sample_rows(wl.T, 120, seed=1, k=256)
    _check_prefill(sa, wl, 1, rows, k=256)


def test_prefill_flat_fp8_chunked(sa):
    wl = WORKLOADS["prefill_t16k"].with_(T=1300)
    rows = sample_rows(wl.T, 60, seed=2, k=300, extra=(499, 500, 501, 999, 1000))
    _check_prefill(sa, wl, 2, rows, k=300, chunk_rows=500)


def test_prefill_flat_streaming_ragged(sa):
    # no score table: sampled thresholds, appending scan, exact list select
    wl = WORKLOADS["prefill_t16k"].with_(T=40000, k=256)
    rows = sample_rows(wl.T, 96, seed=5, k=256, extra=(1023, 1024, 1025, 39999))
    st = sa.new_status("cuda")
    _check_prefill(sa, wl, 5, rows, k=256, flat_path="stream", chunk_rows=16000, status=st)
    s = st.cpu().tolist()
    assert s[0] == 0, s
    assert s[2] <= 40, f"too many whole-row fallbacks: {s}"


def test_prefill_flat_streaming_forced_fallbacks(sa):
    # theta = +inf: every list misses low, every row takes the whole-row fallback
    wl = WORKLOADS["prefill_t16k"].with_(T=3000, k=128)
    rows = sample_rows(wl.T, 48, seed=6, k=128)
    inp = PrefillInputs(wl, "cuda", seed=6)
    st = sa.new_status("cuda")
    _check_prefill(sa, wl, 6, rows, k=128, flat_path="stream", hook=sa.SA_HOOK_THETA_POS_INF, status=st, inp=inp)
    assert st.cpu().tolist()[2] == wl.T
    # theta = -inf: every key is listed; rows with more than 4k = 512 visible
    # keys overflow their list and fall back
    st = sa.new_status("cuda")
    _check_prefill(sa, wl, 6, rows, k=128, flat_path="stream", hook=sa.SA_HOOK_THETA_NEG_INF, status=st, inp=inp)
    s = st.cpu().tolist()
    assert s[3] == wl.T - 512 and s[2] == wl.T - 512, s


@pytest.mark.parametrize("T,k,chunk", [(3000, 128, 0), (20000, 256, 7000)])
def test_prefill_flat_streaming_running_threshold(sa, T, k, chunk):
    # every threshold starts at -inf and the scan runs in phases of cap - k
    # keys: without the running threshold every row with more than cap = 4k
    # visible keys would overflow its list; with it, each list is cut to its
    # k best between phases, no row overflows or falls back, and the rows
    # still match the oracle exactly
    wl = WORKLOADS["prefill_t16k"].with_(T=T, k=k)
    rows = sample_rows(wl.T, 48, seed=7, k=k, extra=(4 * k - 1, 4 * k, 4 * k + 1))
    st = sa.new_status("cuda")
    _check_prefill(sa, wl, 7, rows, k=k, flat_path="stream", chunk_rows=chunk, hook=sa.SA_HOOK_THETA_RUNNING,
                   status=st)
    assert st.cpu().tolist() == [0, 0, 0, 0]


def test_prefill_flat_streaming_fallback_in_device_batches(sa):
    # theta = +inf: every row of every chunk is queued for the whole-row
    # fallback; at 40,000 keys a batch holds 1 GiB / (4 n_k) = 6710 rows, so
    # each 16,000-row chunk runs three batches gated by the queue's length on
    # the device. Rows around the batch edges are checked against the oracle.
    wl = WORKLOADS["prefill_t16k"].with_(T=40000, k=256)
    rows = sample_rows(wl.T, 40, seed=8, k=256,
                       extra=(6709, 6710, 13419, 13420, 15999, 16000, 22709, 22710, 32000, 39999))
    st = sa.new_status("cuda")
    _check_prefill(sa, wl, 8, rows, k=256, flat_path="stream", chunk_rows=16000, hook=sa.SA_HOOK_THETA_POS_INF,
                   status=st)
    s = st.cpu().tolist()
    assert s[0] == 0 and s[2] == wl.T, s


def test_prefill_flat_streaming_replays_as_a_cuda_graph(sa):
    """The streaming FLAT prefill (sampled thresholds, appending scan, list
    select, device-queued fallback) makes no host round trip, so it can be
    captured in a CUDA graph; the replay selects the same key sets and gives
    the same attention as the eager call."""
    wl = WORKLOADS["prefill_t16k"].with_(T=20000, k=256)
    inp = PrefillInputs(wl, "cuda", seed=9)
    st = sa.new_status("cuda")
    pre = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, wl.k,
                     flat_path="stream", chunk_rows=8000, status=st)
    out, lse, idx = pre()
    torch.cuda.synchronize()
    ref_idx = np.sort(idx.cpu().numpy(), axis=1)
    ref_out, ref_lse = out.float().cpu().numpy(), lse.cpu().numpy()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        pre(s)
    idx.fill_(-7)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert st.cpu().tolist()[0] == 0
    assert np.array_equal(np.sort(idx.cpu().numpy(), axis=1), ref_idx)
    go, gl = out.float().cpu().numpy(), lse.cpu().numpy()
    for t in range(0, wl.T, 997):
        check_attention_row(go[t], ref_out[t], gl[t], ref_lse[t], f"replayed row {t}")
    del g


def _two_stage_kept_sets(sa, inp, k_all):
    """Kept blocks of every row, read through the public API: with k = keep *
    64 every visible key of the kept blocks is selected."""
    pre = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, k_all,
                     mode="two_stage", keep_blocks=k_all // 64)
    _, _, idx = pre()
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    return [np.unique(r[r >= 0] // 64) for r in idx]


def _check_two_stage(sa, wl, seed, rows, k, keep=64):
    inp = PrefillInputs(wl, "cuda", seed=seed)
    host = inp.to_host()
    kept_gpu = _two_stage_kept_sets(sa, inp, keep * 64)
    ref = oracle.prefill_rows(host, rows, k, mode="two_stage", keep=keep, attention=False)
    n_diff = 0
    for t in rows:
        ko = ref[t]["kept"]
        kg = kept_gpu[t]
        if not np.array_equal(ko, kg):
            # several results are correct: differing blocks must sit at the cut
            bs = ref[t]["bscores"].astype(np.float64)
            cur = t // 64
            others = np.arange(1, cur)
            srt = np.sort(bs[1:cur])[::-1]
            cut = srt[keep - 3]
            for b in set(ko.tolist()) ^ set(kg.tolist()):
                assert b not in (0, cur), f"row {t}: forced block {b} differs"
                assert abs(bs[b] - cut) <= 2e-3 * np.abs(bs[:cur]).max(), f"row {t}: block {b} far from the cut"
            n_diff += 1
    assert n_diff <= max(2, len(rows) // 20)
    pre = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, k,
                     mode="two_stage", keep_blocks=keep)
    out, lse, idx = pre()
    torch.cuda.synchronize()
    out, lse, idx = out.float().cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()
    ii = oracle.indexer.IndexerInputs(host)
    for t in rows:
        # stage 2 judged against the oracle's token scores over the GPU's kept blocks
        cand = oracle.two_stage_candidates(kept_gpu[t], t, 64)
        sc = oracle.scores_row(oracle.indexer.dequant(ii.q[t]), ii.sq[t], ii.kv[cand], ii.sk[cand], ii.w[t])
        check_topk_row(idx[t], cand, sc, k, f"row {t}")
    att = attention_rows(host, {t: idx[t] for t in rows})
    for t in rows:
        check_attention_row(out[t], att[t][0], lse[t], att[t][1], f"row {t}")


def test_prefill_two_stage_small(sa):
    wl = WORKLOADS["two_stage_t64k"].with_(T=6000, k=512)
    rows = sample_rows(wl.T, 80, seed=3, k=512, extra=(63, 64, 4095, 4096, 5999))
    _check_two_stage(sa, wl, 3, rows, k=512)


def test_prefill_attention_grouped_and_per_query_schedules(sa):
    """The grouped two-stage schedule (stage 2 scoring each union block once
    for 8 queries, attention over each group's union of keys on the tensor
    cores) and the per-query schedule both give a valid exact top-k and the
    oracle's attention over their own index rows, on a ragged chunking
    (windows of queries that end mid-group); FLAT query order too. The two
    schedules sum the heads in different orders, so near-ties at the cut may
    resolve differently: each is judged against the oracle's scores."""
    wl = WORKLOADS["two_stage_t64k"].with_(T=6000, k=512)
    inp = PrefillInputs(wl, "cuda", seed=8)
    host = inp.to_host()
    rows = sample_rows(wl.T, 60, seed=8, k=512, extra=(0, 1, 1499, 1500, 2047, 2048, 5999))
    kept_gpu = _two_stage_kept_sets(sa, inp, 64 * 64)
    ii = oracle.indexer.IndexerInputs(host)
    sets = {}
    for name, hook in (("grouped", 0), ("per_query", sa.SA_HOOK_ATTN_UNGROUPED)):
        pre = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, 512,
                         mode="two_stage", chunk_rows=1500, test_hook=hook)
        out, lse, idx = pre()
        torch.cuda.synchronize()
        out, lse, idx = out.float().cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()
        for t in rows:
            cand = oracle.two_stage_candidates(kept_gpu[t], t, 64)
            sc = oracle.scores_row(oracle.indexer.dequant(ii.q[t]), ii.sq[t], ii.kv[cand], ii.sk[cand], ii.w[t])
            check_topk_row(idx[t], cand, sc, 512, f"{name} row {t}")
        att = attention_rows(host, {t: idx[t] for t in rows})
        for t in rows:
            check_attention_row(out[t], att[t][0], lse[t], att[t][1], f"{name} row {t}")
        sets[name] = np.sort(idx, axis=1)
    # the schedules differ at most in near-ties, on few rows
    n_diff = int((sets["grouped"] != sets["per_query"]).any(axis=1).sum())
    assert n_diff <= wl.T // 50, n_diff
    wl = WORKLOADS["tiny_t512"]
    _check_prefill(sa, wl, 9, range(0, wl.T, 7), hook=sa.SA_HOOK_ATTN_UNGROUPED)
    _check_prefill(sa, wl, 9, range(0, wl.T, 7))


def test_prefill_two_stage_equals_flat_below_64_blocks(sa):
    wl = WORKLOADS["two_stage_t64k"].with_(T=3000, k=256, topic_run=256)
    inp = PrefillInputs(wl, "cuda", seed=4)
    a = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, 256, mode="flat")()
    b = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, 256,
                   mode="two_stage")()
    torch.cuda.synchronize()
    ia, ib = a[2].cpu().numpy(), b[2].cpu().numpy()
    for t in range(wl.T):
        assert sorted(ia[t].tolist()) == sorted(ib[t].tolist()), f"row {t}"


# ------------------------------------------------------------------- decode
def _check_decode(sa, wl, seed, seqs=None, seq_lens=None, k=None, hook=0, status=None):
    k = k or wl.k
    inp = DecodeInputs(wl, "cuda", seed=seed)
    if seq_lens is not None:
        inp.seq_lens = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    host = inp.to_host()
    dec = sa.Decode(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, inp.seq_lens, k,
                    test_hook=hook, status=status)
    out, lse, idx = dec()
    torch.cuda.synchronize()
    out, lse, idx = out.float().cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()
    seqs = range(wl.batch) if seqs is None else seqs
    ref = oracle.decode_rows(host, seqs, k, attention=False)
    for b in seqs:
        check_topk_row(idx[b], ref[b]["cand"], ref[b]["scores"], k, f"seq {b}")
        o, l = decode_attention_row(host, b, idx[b])
        check_attention_row(out[b], o, lse[b], l, f"seq {b}")


def test_decode_graphs_per_context_bucket(sa):
    """Decode graphs captured per context-length bucket (1.125 * 2^e keys):
    each replay runs the narrowest bucket that holds the batch's longest
    sequence, over mixed lengths, and matches the oracle; a call whose
    max_len is shorter than a sequence reports it in the status word."""
    k = 256
    wl = WORKLOADS["decode_b64_l128k"].with_(batch=4, L=8192)
    inp = DecodeInputs(wl, "cuda", seed=12)
    st = sa.new_status("cuda")
    dec = sa.Decode(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, inp.seq_lens, k,
                    status=st)
    graphs = sa.DecodeGraphs(dec, wl.L, smallest=1024)
    assert graphs.buckets == [1152, 2304, 4608, 8192]
    for lens, bucket in (([1000, 2000, 300, 2300], 2304), ([8000, 5000, 100, 7000], 8192),
                         ([1100, 50, 900, 1152], 1152), ([4608, 4000, 1, 2305], 4608)):
        inp.seq_lens.copy_(torch.tensor(lens, dtype=torch.int32))
        assert graphs.replay(max(lens)) == bucket
        torch.cuda.synchronize()
        assert st.cpu().tolist()[0] == 0
        host = inp.to_host()
        idx, out, lse = dec.idx.cpu().numpy(), dec.out.float().cpu().numpy(), dec.lse.cpu().numpy()
        ref = oracle.decode_rows(host, range(wl.batch), k, attention=False)
        for b in range(wl.batch):
            check_topk_row(idx[b], ref[b]["cand"], ref[b]["scores"], k, f"bucket {bucket} seq {b}")
            o, l = decode_attention_row(host, b, idx[b])
            check_attention_row(out[b], o, lse[b], l, f"bucket {bucket} seq {b}")
    inp.seq_lens.copy_(torch.tensor([1000, 2000, 300, 100], dtype=torch.int32))
    short = sa.Decode(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, inp.seq_lens, k,
                      status=st, max_len=1152)
    short()
    torch.cuda.synchronize()
    assert st.cpu().tolist()[0] == sa.SA_ERR_INVALID_ARGUMENT


def test_decode_cuda_graph_replay(sa):
    """One decode step captured as a CUDA graph and replayed: the replay
    matches the oracle, and a replay after new inputs were written into the
    same buffers matches the oracle on those inputs."""
    k = 256
    wl = WORKLOADS["decode_b64_l128k"].with_(batch=3, L=4000)
    inp = DecodeInputs(wl, "cuda", seed=21)
    dec = sa.Decode(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, inp.seq_lens, k)
    g = dec.graph()
    for seed in (21, 22):
        nxt = DecodeInputs(wl, "cuda", seed=seed)
        for name in ("q_idx", "q_scale", "k_idx", "k_scale", "w", "Q", "K", "V", "seq_lens"):
            getattr(inp, name).copy_(getattr(nxt, name))
        dec.out.zero_()
        g.replay()
        torch.cuda.synchronize()
        host = inp.to_host()
        out, lse, idx = dec.out.float().cpu().numpy(), dec.lse.cpu().numpy(), dec.idx.cpu().numpy()
        ref = oracle.decode_rows(host, range(wl.batch), k, attention=False)
        for b in range(wl.batch):
            check_topk_row(idx[b], ref[b]["cand"], ref[b]["scores"], k, f"seed {seed} seq {b}")
            o, l = decode_attention_row(host, b, idx[b])
            check_attention_row(out[b], o, lse[b], l, f"seed {seed} seq {b}")


def test_quantize_rows_e4m3_matches_oracle(sa):
    """Device per-row FP8 encoding against the oracle's: identical scales, and
    identical decoded values (bytes too wherever the value is not zero; a
    negative value that rounds to zero may keep its sign)."""
    g = torch.Generator(device="cuda").manual_seed(31)
    x = torch.randn(200, 128, generator=g, device="cuda") * torch.logspace(-6, 3, 200, device="cuda")[:, None]
    x[0] = 0.0                                                   # all-zero row: scale 1
    x[1, 7] = 1.0e4                                              # one huge entry
    x[2, :4] = torch.tensor([448.0, 1.0625, 1.1875, -1.0625], device="cuda")   # exact ties at scale 1
    x[2, 4:] = 0.5
    cases = [x, torch.randn(33, 37, generator=g, device="cuda"), torch.randn(4, 16, 128, generator=g, device="cuda")]
    for xc in cases:
        for dt in (torch.float32, torch.bfloat16):
            xs = xc.to(dt)
            b, s = sa.quantize_rows_e4m3(xs)
            torch.cuda.synchronize()
            ref_b, ref_s = oracle.quantize_rows(xs.float().cpu().numpy())
            b = b.cpu().numpy()
            assert np.array_equal(s.cpu().numpy(), ref_s), (dt, xc.shape)
            dec, ref = oracle.e4m3_decode(b), oracle.e4m3_decode(ref_b)
            assert np.array_equal(dec, ref), (dt, xc.shape)
            nz = ref != 0
            assert np.array_equal(b[nz], ref_b[nz]), (dt, xc.shape)


def test_expand_sinks_window_matches_oracle(sa):
    """Served index rows (4 sinks, a 512-key window, the selected keys neither
    covers) against the oracle row by row, on early rows (inside the sinks and
    the window) and later ones, with -1 padding anywhere in the input rows; and
    attention over the expanded rows against the oracle."""
    from oracle.pipeline import expand_sinks_window_row
    rng = np.random.default_rng(41)
    n_q, k, q_pos0 = 300, 64, 400
    idx = np.full((n_q, k), -1, dtype=np.int32)
    for t in range(n_q):
        p = q_pos0 + t
        m = min(k, p + 1) if t % 4 else int(rng.integers(0, min(k, p + 1) + 1))
        idx[t, :m] = rng.choice(p + 1, size=m, replace=False)
        rng.shuffle(idx[t])
    for n_sink, n_window, pos0 in ((4, 512, q_pos0), (4, 512, 0), (0, 32, q_pos0), (16, 0, q_pos0)):
        out = sa.expand_sinks_window(torch.from_numpy(idx).cuda(), pos0, n_sink, n_window)
        torch.cuda.synchronize()
        out = out.cpu().numpy()
        for t in range(n_q):
            ref = expand_sinks_window_row(idx[t], pos0 + t, n_sink, n_window)
            assert np.array_equal(out[t], ref), (n_sink, n_window, pos0, t)
    # attention over the served rows
    g = torch.Generator(device="cuda").manual_seed(42)
    n_k = q_pos0 + n_q
    K = (torch.randn(n_k, 128, generator=g, device="cuda") / np.sqrt(128)).bfloat16()
    V = (torch.randn(n_k, 128, generator=g, device="cuda") / np.sqrt(128)).bfloat16()
    Q = (torch.randn(n_q, 16, 128, generator=g, device="cuda") / np.sqrt(128)).bfloat16()
    J = sa.expand_sinks_window(torch.from_numpy(idx).cuda(), q_pos0, 4, 512)
    o, l = sa.sparse_attn(Q, K, V, J)
    torch.cuda.synchronize()
    o, l, J = o.float().cpu().numpy(), l.cpu().numpy(), J.cpu().numpy()
    Qh, Kh, Vh = Q.double().cpu().numpy(), K.double().cpu().numpy(), V.double().cpu().numpy()
    for t in range(0, n_q, 7):
        ro, rl = oracle.sparse_attention_row(Qh[t], Kh, Vh, J[t])
        check_attention_row(o[t], ro, l[t], rl, f"row {t}")


def test_decode_ragged_lengths(sa):
    wl = WORKLOADS["decode_b64_l128k"].with_(batch=4, L=5000)
    _check_decode(sa, wl, 0, seq_lens=[5000, 4097, 130, 2048], k=512)


def test_decode_forced_fallbacks(sa):
    # theta = +inf: every list is empty, every sequence falls back to its row;
    # theta = -inf: every visible score is listed and the 3000-key rows
    # overflow their 4k = 512 list, then fall back
    wl = WORKLOADS["decode_b64_l128k"].with_(batch=3, L=3000)
    st = sa.new_status("cuda")
    _check_decode(sa, wl, 1, k=128, hook=sa.SA_HOOK_THETA_POS_INF, status=st)
    assert st.cpu().tolist()[2] == 3
    st = sa.new_status("cuda")
    _check_decode(sa, wl, 1, k=128, hook=sa.SA_HOOK_THETA_NEG_INF, status=st)
    s = st.cpu().tolist()
    assert s[2] == 3 and s[3] == 3, s


def test_decode_equals_prefill_last_row(sa):
    wl = WORKLOADS["prefill_t16k"].with_(T=3000, k=512)
    inp = PrefillInputs(wl, "cuda", seed=6)
    T = wl.T
    pre = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, 512)()
    dec = sa.Decode(inp.q_idx[T - 1:T], inp.q_scale[T - 1:T], inp.k_idx[None], inp.k_scale[None], inp.w[T - 1:T],
                    inp.Q[T - 1:T], inp.K[None], inp.V[None], torch.tensor([T], dtype=torch.int32, device="cuda"),
                    512)()
    torch.cuda.synchronize()
    assert sorted(pre[2][T - 1].tolist()) == sorted(dec[2][0].tolist())
    assert torch.equal(pre[0][T - 1], dec[0][0]) or (pre[0][T - 1].float() - dec[0][0].float()).abs().max() < 1e-2


# ------------------------------------------------- full sizes, sampled rows
def test_full_prefill_t16k_sampled(sa):
    wl = WORKLOADS["prefill_t16k"]
    rows = sample_rows(wl.T, 256, seed=10, k=wl.k)
    _check_prefill(sa, wl, 0, rows)


def test_full_two_stage_t64k_sampled(sa):
    wl = WORKLOADS["two_stage_t64k"]
    rows = sample_rows(wl.T, 256, seed=11, k=wl.k, extra=(63, 64, 4095, 4096))
    _check_two_stage(sa, wl, 0, rows, k=wl.k)


def test_full_decode_b64_l128k(sa):
    wl = WORKLOADS["decode_b64_l128k"]
    _check_decode(sa, wl, 0)


def test_full_prefill_t1m_streaming_sampled(sa):
    # 2^20 tokens: FLAT prefill without a score table; 256 stratified rows
    # checked against the oracle (host copies of the sampled query rows only)
    wl = WORKLOADS["prefill_t1m"]
    inp = PrefillInputs(wl, "cuda", seed=0)
    st = sa.new_status("cuda")
    out, lse, idx = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, wl.k,
                               status=st, want_lse=True)()
    torch.cuda.synchronize()
    s = st.cpu().tolist()
    assert s[0] == 0, s
    rows = sample_rows(wl.T, 256, seed=12, k=wl.k, extra=(8191, 8192, 16383, 16384))
    r_t = torch.as_tensor(rows, device="cuda")
    host = {"q_idx": inp.q_idx[r_t].cpu(), "q_scale": inp.q_scale[r_t].cpu(), "w": inp.w[r_t].cpu(),
            "Q": inp.Q[r_t].cpu(), "k_idx": inp.k_idx.cpu(), "k_scale": inp.k_scale.cpu(),
            "K": inp.K.cpu(), "V": inp.V.cpu()}
    ref = oracle.prefill_rows(host, range(len(rows)), wl.k, attention=False, positions=rows)
    gi = idx[r_t].cpu().numpy()
    go, gl = out[r_t].float().cpu().numpy(), lse[r_t].cpu().numpy()
    att = attention_rows(host, {i: gi[i] for i in range(len(rows))})
    for i, t in enumerate(rows):
        check_topk_row(gi[i], ref[i]["cand"], ref[i]["scores"], wl.k, f"row {t}")
        check_attention_row(go[i], att[i][0], gl[i], att[i][1], f"row {t}")
    assert s[2] <= wl.T // 1000, f"whole-row fallbacks: {s}"
