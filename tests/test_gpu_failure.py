"""Failure detection on the GPU without a fault: a device wait that can
never complete (the stall hook withholds one MMA completion signal) must give
up within its bounded budget, report SA_ERR_TIMEOUT and the wait site in the
device status word, and leave the context usable."""
import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, PrefillInputs
from helpers import check_topk_row

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import ensure_built
    ensure_built()
    import indexer_selected_top_b200 as m
    return m


def test_stalled_wait_times_out_and_context_survives(sa):
    wl = WORKLOADS["prefill_t16k"].with_(T=300, k=64)
    inp = PrefillInputs(wl, "cuda", seed=3)
    st = sa.new_status("cuda")
    pre = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, wl.k,
                     status=st, test_hook=sa.SA_HOOK_STALL_WAIT)
    pre()
    torch.cuda.synchronize()
    s = st.cpu().tolist()
    assert s[0] == sa.SA_ERR_TIMEOUT, s
    assert s[1] != 0, s                                   # which wait gave up
    # the context is intact: a normal call right after is exact
    st2 = sa.new_status("cuda")
    out, lse, idx = sa.Prefill(inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.Q, inp.K, inp.V, wl.k,
                               status=st2)()
    torch.cuda.synchronize()
    assert st2.cpu().tolist()[0] == 0
    host = inp.to_host()
    idx = idx.cpu().numpy()
    ref = oracle.prefill_rows(host, [0, 63, 64, 299], wl.k, attention=False)
    for t, r in ref.items():
        check_topk_row(idx[t], r["cand"], r["scores"], wl.k, f"row {t}")
