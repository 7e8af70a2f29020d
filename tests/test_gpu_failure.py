"""Failure detection on the GPU, without a fault: the lightning-indexer
kernel's bounded waits are set far below the latency of its own copies, so its
roles give up. The kernel records DSA_ERR_TIMEOUT, lets the copies and MMAs it
already issued complete, frees its tensor memory and returns. The host reads
the status, and the same context then runs the same call at the default bound
to the same result, bit for bit."""
import dataclasses

import pytest
import torch

from sparse_attention_long_tcgen05_b200.inputs import WORKLOADS, make_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    from sparse_attention_long_tcgen05_b200 import _build
    _build.build()
    from sparse_attention_long_tcgen05_b200 import dsa
    yield dsa
    dsa.dsa_set_wait_limit_ns(0)


def test_indexer_wait_timeout_is_reported_and_the_context_recovers(dsa):
    wl = dataclasses.replace(WORKLOADS[1], L=777)
    inp = make_prefill(wl, device="cuda", seed=3)
    ind = dsa.indexer_in(inp.q_idx, inp.k_idx, inp.w, inp.q_scale, inp.k_scale)
    L = wl.L
    ref = torch.empty(L, L, device="cuda")
    dsa.dsa_indexer_scores(ind, None, L, ref, L)
    assert dsa.dsa_check_status() == dsa.DSA_OK
    scores = torch.full((L, L), 5.0, device="cuda")
    for _ in range(2):
        try:
            dsa.dsa_set_wait_limit_ns(1)      # every wait that is not complete at once runs out
            dsa.dsa_indexer_scores(ind, None, L, scores, L)
            st = dsa.dsa_check_status()
        finally:
            dsa.dsa_set_wait_limit_ns(0)      # back to the 1 s default
        assert st == dsa.DSA_ERR_TIMEOUT, dsa.status_string(st)
        assert dsa.dsa_check_status() == dsa.DSA_OK    # reading the status cleared it
    # the context is intact: the same call at the default bound gives the
    # reference scores bit for bit
    torch.cuda.synchronize()
    dsa.dsa_indexer_scores(ind, None, L, scores, L)
    assert dsa.dsa_check_status() == dsa.DSA_OK
    assert torch.equal(scores, ref)
