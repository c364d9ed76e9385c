"""The C ABI without a GPU: the library loads, exports every symbol that
include/sa.h declares, and validates arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sa():
    from conftest import ensure_built
    ensure_built()
    import indexer_selected_top_b200 as m
    return m


def _declared():
    text = open(os.path.join(ROOT, "include", "sa.h")).read()
    return sorted(set(re.findall(r"^\s*(?:sa_status|const char\*)\s+(sa_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("sa_index_scores", "sa_topk", "sa_sparse_attn", "sa_prefill", "sa_decode", "sa_workspace_size",
              "sa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(sa):
    lib = ctypes.CDLL(sa.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(_declared()) <= set(sa.EXPORTS) | {"sa_status_string"}


def test_status_strings(sa):
    assert sa.status_string(0) == "SA_OK"
    assert sa.status_string(3) == "SA_ERR_WORKSPACE_TOO_SMALL"
    assert sa.status_string(99) == "SA_ERR_UNKNOWN"


def test_host_validation_rejects_before_launch(sa):
    lib = sa._lib
    # sa_topk: bad sizes
    assert lib.sa_topk(None, 4, 0, 0, 0, 8, None, None, 0, None) == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_topk(None, 4, 10, 5, 0, 8, None, None, 0, None) == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_topk(None, 4, 10, 10, 0, 8, None, None, 0, None) == sa.SA_ERR_INVALID_ARGUMENT  # null ptrs
    assert lib.sa_topk(None, 0, 10, 10, 0, 8, None, None, 0, None) == sa.SA_OK                   # empty
    # indexer: unsupported head count / dtype, misaligned pointer
    ind = sa.IndexerIn(n_q=4, n_k=16, q_pos0=0, n_heads=7, d_idx=128, dtype=sa.SA_FP8_E4M3, q=256, q_scale=512,
                       k=1024, k_scale=2048, w=4096, batch=0, seq_lens=None)
    assert lib.sa_index_scores(ctypes.byref(ind), 8192, 16, None, 0, None) == sa.SA_ERR_UNSUPPORTED
    ind.n_heads = 64
    ind.q = 257
    assert lib.sa_index_scores(ctypes.byref(ind), 8192, 16, None, 0, None) == sa.SA_ERR_INVALID_ARGUMENT
    ind.q = 256
    assert lib.sa_index_scores(ctypes.byref(ind), 8192, 8, None, 0, None) == sa.SA_ERR_INVALID_ARGUMENT  # ld < n_k
    ind.q_scale = None
    assert lib.sa_index_scores(ctypes.byref(ind), 8192, 16, None, 0, None) == sa.SA_ERR_INVALID_ARGUMENT
    # attention: unsupported head_dim
    att = sa.AttnIn(n_q=4, n_k=16, n_q_heads=16, head_dim=96, softmax_scale=0.0, q=256, k_cache=512, v_cache=768,
                    batch=0)
    assert lib.sa_sparse_attn(ctypes.byref(att), 1024, 8, 2048, None, None, 0, None) == sa.SA_ERR_UNSUPPORTED


def test_workspace_sizes_and_too_small(sa):
    ind = sa.IndexerIn(n_q=65536, n_k=65536, q_pos0=0, n_heads=64, d_idx=128, dtype=sa.SA_FP8_E4M3, q=256,
                       q_scale=512, k=1024, k_scale=2048, w=4096, batch=0, seq_lens=None)
    att = sa.AttnIn(n_q=65536, n_k=65536, n_q_heads=16, head_dim=128, softmax_scale=0.0, q=256, k_cache=512,
                    v_cache=768, batch=0)
    two = sa.PrefillOpts(k=2048, mode=sa.SA_MODE_TWO_STAGE, block_size=64, keep_blocks=64, chunk_rows=0,
                         status=None, test_hook=0)
    n_two = sa.workspace_size(sa.SA_OP_PREFILL, ind, att, two)
    # per 32768-row chunk: block scores + kept + candidate scores + index rows, plus pooled keys
    assert n_two >= 32768 * (1024 * 4 + 64 * 4 + 4096 * 4 + 2048 * 4)
    flat = sa.PrefillOpts(k=2048, mode=sa.SA_MODE_FLAT, block_size=64, keep_blocks=64, chunk_rows=0, status=None,
                          test_hook=0)
    n_flat = sa.workspace_size(sa.SA_OP_PREFILL, ind, att, flat)
    assert n_flat >= 16384 * 65536 * 4 and n_flat <= (4 << 30) + 32768 * 2048 * 4 + 4096
    r = sa._lib.sa_prefill(ctypes.byref(ind), ctypes.byref(att), ctypes.byref(two), None, 4096, None, 256, 1024,
                           None)
    assert r == sa.SA_ERR_WORKSPACE_TOO_SMALL
    dind = sa.IndexerIn(n_q=64, n_k=131072, q_pos0=0, n_heads=64, d_idx=128, dtype=sa.SA_FP8_E4M3, q=256,
                        q_scale=512, k=1024, k_scale=2048, w=4096, batch=64, seq_lens=None)
    datt = sa.AttnIn(n_q=64, n_k=131072, n_q_heads=16, head_dim=128, softmax_scale=0.0, q=256, k_cache=512,
                     v_cache=768, batch=64)
    dopts = sa.DecodeOpts(k=2048, status=None, test_hook=0)
    assert sa.workspace_size(sa.SA_OP_DECODE, dind, datt, dopts) >= 64 * 131072 * 4
    assert sa.workspace_size(sa.SA_OP_SPARSE_ATTN, att=datt, opts=2048) > 0
    assert sa.workspace_size(sa.SA_OP_SPARSE_ATTN, att=att, opts=2048) == 0


def test_new_entry_points_validate_on_the_host(sa):
    lib = sa._lib
    # sa_quantize_rows_e4m3(x, dtype, n_rows, d, out, scale, stream)
    assert lib.sa_quantize_rows_e4m3(None, sa.SA_F32, 0, 128, None, None, None) == sa.SA_OK            # empty
    assert lib.sa_quantize_rows_e4m3(None, sa.SA_F32, 4, 128, 256, 512, None) == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_quantize_rows_e4m3(256, sa.SA_F32, 4, 0, 256, 512, None) == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_quantize_rows_e4m3(256, sa.SA_F32, 4, 4097, 256, 512, None) == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_quantize_rows_e4m3(256, sa.SA_F32, -1, 128, 256, 512, None) == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_quantize_rows_e4m3(256, sa.SA_FP8_E4M3, 4, 128, 256, 512, None) == sa.SA_ERR_UNSUPPORTED
    # sa_expand_sinks_window(idx, n_q, k, q_pos0, n_sink, n_window, out, stream)
    assert lib.sa_expand_sinks_window(None, 0, 8, 0, 4, 16, None, None) == sa.SA_OK                    # empty
    assert lib.sa_expand_sinks_window(None, 4, 8, 0, 4, 16, None, None) == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_expand_sinks_window(256, 4, 0, 0, 4, 16, 512, None) == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_expand_sinks_window(256, 4, 8, 0, -1, 16, 512, None) == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_expand_sinks_window(256, 4, 8, -5, 4, 16, 512, None) == sa.SA_ERR_INVALID_ARGUMENT


def test_two_stage_workspace_covers_the_group_tables(sa):
    """The two-stage workspace grows with the query rows (per-row candidate
    scores, selection bitmaps, group unions) and stays 256-byte sized."""
    sizes = []
    for n_q in (1000, 8192, 65536):
        ind = sa.IndexerIn(n_q=n_q, n_k=65536, q_pos0=65536 - n_q, n_heads=64, d_idx=128, dtype=sa.SA_FP8_E4M3,
                           q=256, q_scale=512, k=1024, k_scale=2048, w=4096, batch=0, seq_lens=None)
        att = sa.AttnIn(q=256, k_cache=512, v_cache=1024, n_q=n_q, n_k=65536, n_q_heads=16, head_dim=128,
                        softmax_scale=0.0, batch=0)
        opts = sa.PrefillOpts(k=2048, mode=1, block_size=64, keep_blocks=64, chunk_rows=0, status=None,
                              test_hook=0, stage_events=None, n_stage_events=0, flat_path=0)
        sizes.append(sa.workspace_size(sa.SA_OP_PREFILL, ind, att, opts))
    assert sizes[0] < sizes[1] < sizes[2]
    # one chunk of at most 32768 rows: at least its candidate scores, index
    # rows and group key lists (8 k entries of 4 + 1 bytes per group of 8)
    R = 32768
    assert sizes[2] >= R * (4096 * 4 + 2048 * 4) + R // 8 * 8 * 2048 * 5


def test_lsa_entry_points_validate_on_the_host(sa):
    """sa_lsa_build_buckets / sa_lsa_search reject bad parameters before any
    CUDA call, and an empty call is a no-op."""
    lib = sa._lib
    import ctypes
    good = sa.lsa_params()
    bad = [sa.lsa_params(n_pool=3),                       # n_cluster % n_pool
           sa.lsa_params(max_bucket_keys=30),             # cap % n_pool
           sa.lsa_params(n_buckets=129),                  # m > pool keys per block
           sa.lsa_params(n_pool=0)]
    for prm in bad:
        assert lib.sa_lsa_build_buckets(ctypes.byref(prm), 256, 4096, 0, 1, 512, 768, 1024, None, None) \
            == sa.SA_ERR_INVALID_ARGUMENT
    # m equal to the pool keys per block needs no cap rule (no merges)
    assert lib.sa_lsa_build_buckets(ctypes.byref(sa.lsa_params(n_buckets=128, max_bucket_keys=4)), None, 0, 0, 0,
                                    None, None, None, None, None) == sa.SA_OK
    assert lib.sa_lsa_build_buckets(ctypes.byref(sa.lsa_params(d_idx=128)), 256, 4096, 0, 1, 512, 768, 1024, None,
                                    None) == sa.SA_ERR_UNSUPPORTED
    assert lib.sa_lsa_build_buckets(ctypes.byref(sa.lsa_params(n_pool=1)), 256, 4096, 0, 1, 512, 768, 1024, None,
                                    None) == sa.SA_ERR_UNSUPPORTED          # 512 pool keys per block
    assert lib.sa_lsa_build_buckets(ctypes.byref(good), 256, 1000, 0, 2, 512, 768, 1024, None, None) \
        == sa.SA_ERR_INVALID_ARGUMENT                                       # blocks beyond n_k
    assert lib.sa_lsa_build_buckets(ctypes.byref(good), None, 4096, 0, 0, None, None, None, None, None) == sa.SA_OK
    o = sa.LsaSearchOpts(p=512, k=2048, n_sink=4, n_window=512, status=None)
    n = ctypes.c_size_t(0)
    assert lib.sa_lsa_search_workspace_size(ctypes.byref(good), ctypes.byref(o), 65536, 0, 128, ctypes.byref(n)) \
        == sa.SA_OK
    # one chunk of 8192 rows: normalised queries, the score rows, lengths and top-p ids
    assert n.value >= 8192 * (64 * 2 + 8192 * 4 + 4 + 512 * 4)
    assert lib.sa_lsa_search(ctypes.byref(good), ctypes.byref(o), None, 0, 0, None, None, None, 128, None, None, 0,
                             None) == sa.SA_OK
    assert lib.sa_lsa_search(ctypes.byref(good), ctypes.byref(o), 256, 16, 0, 512, 768, 1024, 128, 2048, None, 0,
                             None) == sa.SA_ERR_INVALID_ARGUMENT             # no workspace
    for p, k, ns in [(0, 2048, 4), (512, 0, 4), (512, 2048, -1)]:
        ob = sa.LsaSearchOpts(p=p, k=k, n_sink=ns, n_window=512, status=None)
        assert lib.sa_lsa_search_workspace_size(ctypes.byref(good), ctypes.byref(ob), 16, 0, 8, ctypes.byref(n)) \
            == sa.SA_ERR_INVALID_ARGUMENT
    big_p = sa.LsaSearchOpts(p=4096, k=2048, n_sink=4, n_window=512, status=None)
    assert lib.sa_lsa_search_workspace_size(ctypes.byref(good), ctypes.byref(big_p), 16, 0, 8, ctypes.byref(n)) \
        == sa.SA_ERR_UNSUPPORTED
    # 32,832 buckets: beyond the written-S regime, so AUTO takes the threshold regime and TABLE refuses
    assert lib.sa_lsa_search_workspace_size(ctypes.byref(good), ctypes.byref(o), 16, 0, 513, ctypes.byref(n)) \
        == sa.SA_OK
    ot = sa.LsaSearchOpts(p=512, k=2048, n_sink=4, n_window=512, status=None, regime=sa.SA_LSA_TABLE, test_hook=0)
    assert lib.sa_lsa_search_workspace_size(ctypes.byref(good), ctypes.byref(ot), 16, 0, 513, ctypes.byref(n)) \
        == sa.SA_ERR_UNSUPPORTED


def test_lsa_decode_validates_on_the_host(sa):
    import ctypes
    lib = sa._lib
    good = sa.lsa_params()
    o = sa.LsaSearchOpts(p=512, k=2048, n_sink=4, n_window=512, status=None)
    n = ctypes.c_size_t(0)
    assert lib.sa_lsa_decode_workspace_size(ctypes.byref(good), ctypes.byref(o), 64, 256, ctypes.byref(n)) == sa.SA_OK
    assert n.value >= 64 * (64 * 2 + 256 * 64 * 4 + 4 + 512 * 4)
    assert lib.sa_lsa_decode_workspace_size(ctypes.byref(good), ctypes.byref(o), 64, 513, ctypes.byref(n)) \
        == sa.SA_ERR_UNSUPPORTED
    assert lib.sa_lsa_decode_workspace_size(ctypes.byref(sa.lsa_params(n_pool=3)), ctypes.byref(o), 64, 16,
                                            ctypes.byref(n)) == sa.SA_ERR_INVALID_ARGUMENT
    # batch 0: a no-op; missing lengths, caches or workspace: rejected before any launch
    assert lib.sa_lsa_decode(ctypes.byref(good), ctypes.byref(o), None, 0, None, None, None, 16, None, None, None,
                             None, 0, None) == sa.SA_OK
    assert lib.sa_lsa_decode(ctypes.byref(good), ctypes.byref(o), 256, 4, 512, 768, 1024, 16, None, 2048, 4096,
                             8192, 1 << 20, None) == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_lsa_decode(ctypes.byref(good), ctypes.byref(o), 256, 4, None, 768, 1024, 16, 1280, 2048, 4096,
                             8192, 1 << 20, None) == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_lsa_decode(ctypes.byref(good), ctypes.byref(o), 256, 4, 512, 768, 1024, 16, 1280, 2048, 4096,
                             8192, 256, None) == sa.SA_ERR_WORKSPACE_TOO_SMALL


def test_lsa_search_regimes_validate_and_size(sa):
    """TABLE is limited to 32,768 buckets, STREAM to 2^21; AUTO switches at
    32,768; a STREAM workspace holds the lists (3p packed keys per row) and
    no score matrix."""
    import ctypes
    lib = sa._lib
    good = sa.lsa_params()
    n = ctypes.c_size_t(0)

    def size(regime, n_blocks, p=512):
        o = sa.LsaSearchOpts(p=p, k=2048, n_sink=4, n_window=512, status=None, regime=regime, test_hook=0)
        st = lib.sa_lsa_search_workspace_size(ctypes.byref(good), ctypes.byref(o), 65536, 0, n_blocks,
                                              ctypes.byref(n))
        return st, n.value

    assert size(3, 16)[0] == sa.SA_ERR_INVALID_ARGUMENT
    assert size(sa.SA_LSA_TABLE, 1024)[0] == sa.SA_ERR_UNSUPPORTED          # 65,536 buckets
    st, auto_big = size(sa.SA_LSA_AUTO, 1024)
    st2, stream_big = size(sa.SA_LSA_STREAM, 1024)
    assert st == st2 == sa.SA_OK and auto_big == stream_big
    assert stream_big >= 8192 * 3 * 512 * 8 + 8192 * 512 * 8                # lists and packed top-p
    assert stream_big < 8192 * 65536 * 4                                     # no score matrix per chunk
    assert size(sa.SA_LSA_STREAM, (1 << 21) // 64 + 1)[0] == sa.SA_ERR_UNSUPPORTED
    assert size(sa.SA_LSA_AUTO, 128)[1] == size(sa.SA_LSA_TABLE, 128)[1]     # AUTO: TABLE below 32,768


def test_lsa_calls_validate_before_touching_the_status_word(sa):
    """A call that fails validation queues nothing, not even the zeroing of its
    status word: with a (bogus) status pointer and a bad argument, the answer is
    the validation error, not a CUDA error (there is no device here)."""
    import ctypes
    lib = sa._lib
    good = sa.lsa_params()
    bogus = 4096
    assert lib.sa_lsa_build_buckets(ctypes.byref(good), None, 4096, 0, 1, 512, 768, 1024, bogus, None) \
        == sa.SA_ERR_INVALID_ARGUMENT
    o = sa.LsaSearchOpts(p=512, k=2048, n_sink=4, n_window=512, status=bogus, regime=0, test_hook=0)
    assert lib.sa_lsa_search(ctypes.byref(good), ctypes.byref(o), None, 16, 0, 512, 768, 1024, 8, 2048, 8192,
                             1 << 30, None) == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_lsa_search(ctypes.byref(good), ctypes.byref(o), 256, 16, 0, 512, 768, 1024, 8, 2048, 8192, 256,
                             None) == sa.SA_ERR_WORKSPACE_TOO_SMALL
    assert lib.sa_lsa_decode(ctypes.byref(good), ctypes.byref(o), 256, 4, 512, 768, 1024, 16, None, 2048, 4096,
                             8192, 1 << 20, None) == sa.SA_ERR_INVALID_ARGUMENT


def test_lsa_attention_validates_on_the_host(sa):
    import ctypes
    lib = sa._lib
    n = ctypes.c_size_t(0)
    att = sa.AttnIn(n_q=1000, n_k=4096, n_q_heads=16, head_dim=128, softmax_scale=0.0, q=256, k_cache=512,
                    v_cache=768, batch=0)
    assert lib.sa_lsa_attention_workspace_size(ctypes.byref(att), 2564, 0, 4, 512, ctypes.byref(n)) == sa.SA_OK
    assert n.value > 0
    # the queries' own keys must be in the cache
    assert lib.sa_lsa_attention_workspace_size(ctypes.byref(att), 2564, 3500, 4, 512, ctypes.byref(n)) \
        == sa.SA_ERR_INVALID_ARGUMENT
    assert lib.sa_lsa_attention_workspace_size(ctypes.byref(att), 100, 0, 4, 512, ctypes.byref(n)) \
        == sa.SA_ERR_INVALID_ARGUMENT                                       # width below sinks + window
    other = sa.AttnIn(n_q=1000, n_k=4096, n_q_heads=8, head_dim=64, softmax_scale=0.0, q=256, k_cache=512,
                      v_cache=768, batch=0)
    assert lib.sa_lsa_attention_workspace_size(ctypes.byref(other), 2564, 0, 4, 512, ctypes.byref(n)) \
        == sa.SA_ERR_UNSUPPORTED
    big = sa.AttnIn(n_q=1000, n_k=1 << 20, n_q_heads=16, head_dim=128, softmax_scale=0.0, q=256, k_cache=512,
                    v_cache=768, batch=0)
    assert lib.sa_lsa_attention_workspace_size(ctypes.byref(big), 2564, 0, 4, 512, ctypes.byref(n)) \
        == sa.SA_ERR_UNSUPPORTED
    # rejected before any device work, even with a (bogus) status pointer
    assert lib.sa_lsa_attention(ctypes.byref(att), None, 2564, 0, 4, 512, 1024, None, 4096, 8192, 1 << 30, None) \
        == sa.SA_ERR_INVALID_ARGUMENT


def test_debug_checks_build_and_the_release_refusal(sa):
    """Release builds check nothing and say so; the debug build (the same
    sources with -DSA_DEBUG_CHECKS) compiles, exports the same calls, and its
    reader reaches for the device record (no device here: a CUDA error)."""
    import ctypes
    import importlib.util
    out = (ctypes.c_uint32 * 4)()
    assert sa._lib.sa_debug_errors(ctypes.cast(out, ctypes.c_void_p), 0) == sa.SA_ERR_UNSUPPORTED
    spec = importlib.util.spec_from_file_location("_sa_build", os.path.join(ROOT, "indexer_selected_top_b200",
                                                                            "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    path = mod.build_debug()
    dbg = ctypes.CDLL(path)
    for name in sa.EXPORTS:
        assert hasattr(dbg, name), name
    dbg.sa_debug_errors.argtypes = [ctypes.c_void_p, ctypes.c_int32]
    assert dbg.sa_debug_errors(None, 0) == sa.SA_ERR_INVALID_ARGUMENT
    assert dbg.sa_debug_errors(ctypes.cast(out, ctypes.c_void_p), 0) in (sa.SA_OK, sa.SA_ERR_CUDA)
