"""The allocation-free decode attention entry point.

sa_sparse_attn_decode_noalloc exists for callers that cannot hand the
library any device workspace (a plugin inside a serving engine that owns all
device memory, or a decode loop that may not call the CUDA allocator once it
is running). It keeps its split-K partial results in a fixed array inside the
library instead. These checks call it through the C ABI twice in a row, with
different shapes so the second call runs on the first call's leftovers, and
compare each result with sa_sparse_attn given its own workspace and with the
oracle's fp64 attention over the same index rows. The file
sorts last so a run that stops at the first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

from helpers import check_attention_row

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import ensure_built
    ensure_built()
    import indexer_selected_top_b200 as m
    return m


def _case(B, L, hq, dh, k, seed, std):
    g = torch.Generator(device="cuda").manual_seed(seed)
    K = (torch.randn(B, L, dh, generator=g, device="cuda") * std).bfloat16()
    V = (torch.randn(B, L, dh, generator=g, device="cuda") * std).bfloat16()
    Q = (torch.randn(B, hq, dh, generator=g, device="cuda") * std).bfloat16()
    rng = np.random.default_rng(seed)
    idx = np.full((B, k), -1, dtype=np.int32)
    for b in range(B):
        m = min(L, k if b % 2 == 0 else int(rng.integers(1, k + 1)))
        idx[b, :m] = rng.choice(L, size=m, replace=False)
    return Q, K, V, torch.from_numpy(idx).cuda()


def _call_noalloc(sa, Q, K, V, idx):
    att = sa.attn_in(Q, K, V)
    out = torch.empty_like(Q)
    lse = torch.empty(Q.shape[:2], dtype=torch.float32, device=Q.device)
    code = sa._lib.sa_sparse_attn_decode_noalloc(ctypes.byref(att), idx.data_ptr(), idx.shape[1], out.data_ptr(),
                                                 lse.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == sa.SA_OK, sa.status_string(code)
    return out, lse


@pytest.mark.parametrize("cases", [
    # decode-sized batch at k = 2048, then a smaller, sharper call on its leftovers
    [(64, 4096, 16, 128, 2048, 1, 1.0 / np.sqrt(128)), (3, 900, 16, 128, 700, 2, 1.0)],
    # the other head shape: 8 heads of 64, k not a multiple of the 256-key split
    [(5, 3000, 8, 64, 1000, 4, 1.0 / 8.0), (2, 700, 8, 64, 300, 5, 1.0)],
])
def test_noalloc_matches_workspace_path_twice(sa, cases):
    """Two calls in a row: each result equals sa_sparse_attn's (same
    tolerance as every attention parity test), and both equal the oracle's
    fp64 softmax attention over the same index rows."""
    from oracle import sparse_attention_row
    for B, L, hq, dh, k, seed, std in cases:
        Q, K, V, idx = _case(B, L, hq, dh, k, seed, std)
        ref_out, ref_lse = sa.sparse_attn(Q, K, V, idx)
        out, lse = _call_noalloc(sa, Q, K, V, idx)
        torch.cuda.synchronize()
        ro, rl = ref_out.float().cpu().numpy(), ref_lse.cpu().numpy()
        go, gl = out.float().cpu().numpy(), lse.cpu().numpy()
        Qh, Kh, Vh, ih = Q.double().cpu().numpy(), K.double().cpu().numpy(), V.double().cpu().numpy(), \
            idx.cpu().numpy()
        for b in range(B):
            check_attention_row(go[b], ro[b], gl[b], rl[b], f"B={B} seq {b} vs sa_sparse_attn")
            o, l = sparse_attention_row(Qh[b], Kh[b], Vh[b], ih[b])
            check_attention_row(go[b], o, gl[b], l, f"B={B} seq {b} vs oracle")


def test_noalloc_rejects_sizes_beyond_its_array(sa):
    # 64 sequences x 16 splits (k = 4096) x 16 heads x 128 = 2^21 floats fits;
    # 65 sequences do not.
    Q, K, V, idx = _case(65, 300, 16, 128, 4096, 3, 0.1)
    att = sa.attn_in(Q, K, V)
    out = torch.empty_like(Q)
    code = sa._lib.sa_sparse_attn_decode_noalloc(ctypes.byref(att), idx.data_ptr(), idx.shape[1], out.data_ptr(),
                                                 None, None)
    assert code == sa.SA_ERR_WORKSPACE_TOO_SMALL
