"""Every Python wrapper of the binding, driven to its status check without a GPU.

The wrappers hand their arguments to the library through ctypes and turn a
status code into SaError. A wrapper whose call or status check is malformed
(wrong arity, a wrong argument type, a bad _check call) would only show on a
GPU. Here the library handle is replaced by a proxy that checks each call
against the real function's declared argtypes (count, and the conversion ctypes
itself applies), answers the size queries (workspace bytes, chunk rows) on
the host, and returns SA_ERR_INVALID_ARGUMENT for every other entry point:
each wrapper must then raise SaError naming that entry point. No compute entry point of the library
is called, and every tensor stays in host memory."""
import ctypes

import pytest
import torch


@pytest.fixture(scope="module")
def sa():
    from conftest import ensure_built
    ensure_built()
    import indexer_selected_top_b200 as m
    return m


class _DeviceLike(torch.Tensor):
    """A host tensor that reports is_cuda, so the wrappers' input checks pass."""

    @property
    def is_cuda(self):
        return True


def _t(x):
    return x.as_subclass(_DeviceLike)


class _Proxy:
    def __init__(self, real, calls):
        self._real, self._calls = real, calls

    def __getattr__(self, name):
        fn = getattr(self._real, name)
        if name == "sa_status_string":
            return fn

        def call(*args):
            assert fn.argtypes is not None, f"{name}: argtypes not declared"
            assert len(args) == len(fn.argtypes), f"{name}: {len(args)} arguments, {len(fn.argtypes)} declared"
            for a, t in zip(args, fn.argtypes):
                t.from_param(a)                      # raises as ctypes would on a wrong type
            self._calls.append(name)
            if name.endswith("workspace_size") or name == "sa_prefill_chunk_rows":
                out = args[-1]._obj                  # byref(c_size_t) / byref(c_int32)
                out.value = 4096
                return 0
            return 1                                 # SA_ERR_INVALID_ARGUMENT
        return call


@pytest.fixture
def proxied(sa, monkeypatch):
    calls = []
    monkeypatch.setattr(sa, "_lib", _Proxy(sa._lib, calls))
    monkeypatch.setattr(sa, "_stream", lambda stream=None: ctypes.c_void_p(None))
    return sa, calls


def _raises(sa, calls, name, fn, *a, **kw):
    calls.clear()
    with pytest.raises(sa.SaError) as e:
        fn(*a, **kw)
    assert name in str(e.value), (name, str(e.value))
    assert e.value.code == sa.SA_ERR_INVALID_ARGUMENT
    assert calls[-1] == name, calls


def _prefill_inputs():
    T, H, d, Hq, dh = 64, 64, 128, 16, 128
    q = torch.zeros((T, H, d), dtype=torch.uint8)
    qs = torch.ones((T, H))
    k = torch.zeros((T, d), dtype=torch.uint8)
    ks = torch.ones(T)
    w = torch.ones((T, H))
    Q = torch.zeros((T, Hq, dh), dtype=torch.bfloat16)
    K = torch.zeros((T, dh), dtype=torch.bfloat16)
    return q, qs, k, ks, w, Q, K, K.clone()


def _decode_inputs():
    B, L, H, d, Hq, dh = 2, 300, 64, 128, 16, 128
    q = torch.zeros((B, H, d), dtype=torch.uint8)
    qs = torch.ones((B, H))
    k = torch.zeros((B, L, d), dtype=torch.uint8)
    ks = torch.ones((B, L))
    w = torch.ones((B, H))
    Q = torch.zeros((B, Hq, dh), dtype=torch.bfloat16)
    K = torch.zeros((B, L, dh), dtype=torch.bfloat16)
    return q, qs, k, ks, w, Q, K, K.clone(), torch.full((B,), L, dtype=torch.int32)


def test_core_wrappers_reach_their_status_check(proxied):
    sa, calls = proxied
    q, qs, k, ks, w, Q, K, V = _prefill_inputs()
    _raises(sa, calls, "sa_index_scores", sa.index_scores, q, qs, k, ks, w)
    _raises(sa, calls, "sa_topk", sa.topk, torch.zeros((4, 16)), 8)
    idx = torch.zeros((Q.shape[0], 32), dtype=torch.int32)
    _raises(sa, calls, "sa_sparse_attn", sa.sparse_attn, Q, K, V, idx)
    for mode in ("flat", "two_stage"):
        _raises(sa, calls, "sa_prefill", sa.prefill, q, qs, k, ks, w, Q, K, V, 32, mode=mode)
    dq, dqs, dk, dks, dw, dQ, dK, dV, lens = _decode_inputs()
    _raises(sa, calls, "sa_decode", sa.decode, dq, dqs, dk, dks, dw, dQ, dK, dV, lens, 32)
    _raises(sa, calls, "sa_sparse_attn_decode_noalloc", sa.sparse_attn_decode_noalloc, dQ, dK, dV,
            torch.zeros((2, 32), dtype=torch.int32))


def test_chunk_rows_query_wrapper_reaches_its_status_check(sa, monkeypatch):
    calls = []

    class _Fail(_Proxy):
        def __getattr__(self, name):
            inner = super().__getattr__(name)
            if name != "sa_prefill_chunk_rows":
                return inner

            def call(*args):
                inner(*args)
                return 1
            return call
    monkeypatch.setattr(sa, "_lib", _Fail(sa._lib, calls))
    q, qs, k, ks, w, Q, K, V = _prefill_inputs()
    _raises(sa, calls, "sa_prefill_chunk_rows", sa.Prefill, q, qs, k, ks, w, Q, K, V, 32)


def test_workspace_query_wrapper_reaches_its_status_check(sa, monkeypatch):
    calls = []

    class _Fail(_Proxy):
        def __getattr__(self, name):
            inner = super().__getattr__(name)
            if name != "sa_workspace_size":
                return inner

            def call(*args):
                inner(*args)
                return 1
            return call
    monkeypatch.setattr(sa, "_lib", _Fail(sa._lib, calls))
    q, qs, k, ks, w, Q, K, V = _prefill_inputs()
    ind, att = sa.indexer_in(q, qs, k, ks, w), sa.attn_in(Q, K, V)
    for opts in (None, 32, sa.PrefillOpts(k=32)):
        _raises(sa, calls, "sa_workspace_size", sa.workspace_size, sa.SA_OP_PREFILL, ind, att, opts)


def test_encoding_and_row_wrappers_reach_their_status_check(proxied):
    sa, calls = proxied
    _raises(sa, calls, "sa_quantize_rows_e4m3", sa.quantize_rows_e4m3, _t(torch.zeros((4, 128))))
    _raises(sa, calls, "sa_quantize_rows_e4m3", sa.quantize_rows_e4m3,
            _t(torch.zeros((4, 128), dtype=torch.bfloat16)))
    _raises(sa, calls, "sa_expand_sinks_window", sa.expand_sinks_window,
            _t(torch.zeros((4, 16), dtype=torch.int32)), 0, 4, 32)
    _raises(sa, calls, "sa_debug_errors", sa.debug_errors)


def test_lsa_wrappers_reach_their_status_check(proxied):
    sa, calls = proxied
    prm = sa.lsa_params(n_pool=4, n_cluster=512, n_buckets=64, max_bucket_keys=32)
    T, d = 1024, 64
    k_idx = _t(torch.zeros((T, d), dtype=torch.bfloat16))
    q_idx = _t(torch.zeros((T, d), dtype=torch.bfloat16))
    _raises(sa, calls, "sa_lsa_build_buckets", sa.lsa_build_buckets, k_idx, prm)
    nb = T // 512
    cache = (torch.zeros((nb * 64, d), dtype=torch.bfloat16), torch.zeros(nb * 64, dtype=torch.int32),
             torch.zeros(nb * 512, dtype=torch.int32))
    _raises(sa, calls, "sa_lsa_search", sa.lsa_search, q_idx, prm, cache, nb, 0, 128, 512, 4, 512)
    Q = torch.zeros((T, 16, 128), dtype=torch.bfloat16)
    K = torch.zeros((T, 128), dtype=torch.bfloat16)
    J = torch.zeros((T, 4 + 512 + 512), dtype=torch.int32)
    _raises(sa, calls, "sa_lsa_attention", sa.lsa_attention, Q, K, K.clone(), J, 0, 4, 512)
    pre = sa.LsaPrefill(k_idx, q_idx, Q, K, K.clone(), prm, 128, 512)
    _raises(sa, calls, "sa_lsa_build_buckets", pre)
    B = 3
    caches = (torch.zeros((B, nb * 64, d), dtype=torch.bfloat16), torch.zeros((B, nb * 64), dtype=torch.int32),
              torch.zeros((B, nb * 512), dtype=torch.int32))
    dec = sa.LsaDecode(torch.zeros((B, d), dtype=torch.bfloat16), prm, caches,
                       torch.full((B,), nb, dtype=torch.int32), torch.full((B,), T, dtype=torch.int32), 128, 512)
    _raises(sa, calls, "sa_lsa_decode", dec)


def test_lsa_attention_falls_back_to_the_per_query_call_when_unsupported(sa, monkeypatch):
    """A shape the tensor-core LSA attention does not take runs sa_sparse_attn
    over the same rows; that branch's status check is reached too."""
    calls = []

    class _Unsupported(_Proxy):
        def __getattr__(self, name):
            inner = super().__getattr__(name)
            if name != "sa_lsa_attention_workspace_size":
                return inner

            def call(*args):
                inner(*args)
                return 2                             # SA_ERR_UNSUPPORTED
            return call
    monkeypatch.setattr(sa, "_lib", _Unsupported(sa._lib, calls))
    monkeypatch.setattr(sa, "_stream", lambda stream=None: ctypes.c_void_p(None))
    T = 64
    Q = torch.zeros((T, 16, 128), dtype=torch.bfloat16)
    K = torch.zeros((T, 128), dtype=torch.bfloat16)
    J = torch.zeros((T, 64), dtype=torch.int32)
    _raises(sa, calls, "sa_sparse_attn", sa.lsa_attention, Q, K, K.clone(), J, 0, 4, 32)
