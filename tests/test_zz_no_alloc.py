"""dsa_select_noalloc: the selection for callers that cannot allocate device
memory (a plugin whose host application owns all device memory, or a loop that
must not call cudaMalloc). It keeps its score rows in the library's fixed
16 MiB per-GPU scratch instead of a caller workspace.

Checked through the C ABI against dsa_select (the workspace form), bit for
bit as every top-k result is, on two calls in a row -- the second call finds
the first one's leftovers in the shared scratch. The problems are sized so the
scratch holds only part of the query rows at once (several blocks per call).
This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes alone in a fresh process.
"""
import ctypes
import dataclasses

import pytest
import torch

from sparse_attention_long_tcgen05_b200.inputs import WORKLOADS, make_decode, make_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    from sparse_attention_long_tcgen05_b200 import _build
    _build.build()
    from sparse_attention_long_tcgen05_b200 import dsa
    return dsa


def _noalloc(dsa, ind, k, idx):
    """The new entry point, called through the C ABI."""
    st = dsa.LIB.dsa_select_noalloc(ctypes.byref(ind.struct), k, ctypes.c_void_p(idx.data_ptr()),
                                    idx.stride(0),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == dsa.DSA_OK, dsa.status_string(st)


def _with_workspace(dsa, ind, k, n_q):
    idx = torch.empty(n_q, k, dtype=torch.int32, device="cuda")
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_SELECT, ind, None, 0, 0, k))
    dsa.dsa_select(ind, k, idx, ws)
    return idx


def test_noalloc_select_prefill_matches_workspace_form(dsa):
    # 5000 keys per score row: the 16 MiB scratch holds 836 rows at once, so
    # the 5000 queries run as 6 blocks
    wl = dataclasses.replace(WORKLOADS[1], L=5000)
    inp = make_prefill(wl, device="cuda", seed=11)
    ind = dsa.indexer_in(inp.q_idx, inp.k_idx, inp.w, inp.q_scale, inp.k_scale)
    ref = _with_workspace(dsa, ind, wl.k, wl.L)
    for _ in range(2):
        got = torch.full_like(ref, -7)
        _noalloc(dsa, ind, wl.k, got)
        assert dsa.dsa_check_status() == 0
        assert torch.equal(got, ref)


def test_noalloc_select_query_suffix_matches_workspace_form(dsa):
    # the queries are the last 2000 tokens of 6000 keys (a chunk of a longer
    # prefill): each block's rows see keys 0..4000+q0+rows-1; the scratch holds
    # 696 rows of 6000 scores, so the 2000 queries run as 3 blocks
    wl = dataclasses.replace(WORKLOADS[1], L=6000)
    inp = make_prefill(wl, device="cuda", seed=13)
    off = 4000
    ind = dsa.indexer_in(inp.q_idx[off:], inp.k_idx, inp.w[off:], inp.q_scale[off:],
                         inp.k_scale)
    ref = _with_workspace(dsa, ind, wl.k, wl.L - off)
    for _ in range(2):
        got = torch.full_like(ref, -7)
        _noalloc(dsa, ind, wl.k, got)
        assert dsa.dsa_check_status() == 0
        assert torch.equal(got, ref)


def test_noalloc_select_paged_matches_workspace_form(dsa):
    # 2048 pages x 64 = 131072 columns per row: 32 rows per block, 40 sequences
    wl = dataclasses.replace(WORKLOADS[4], ctx_max=131072)
    g = torch.Generator().manual_seed(5)
    ctx = torch.randint(1, 4000, (40,), generator=g).tolist()
    ctx[0], ctx[1] = 1, 2049
    inp = make_decode(wl, device="cuda", seed=12, ctx_lens=ctx)
    lay = dsa.paged_layout(inp.block_table, inp.ctx_lens, inp.num_pages)
    ind = dsa.indexer_in(inp.q_idx, inp.k_cache, inp.w, inp.q_scale,
                         inp.k_cache_scale.view(-1), kv=lay)
    ref = _with_workspace(dsa, ind, wl.k, len(ctx))
    for _ in range(2):
        got = torch.full_like(ref, -7)
        _noalloc(dsa, ind, wl.k, got)
        assert dsa.dsa_check_status() == 0
        assert torch.equal(got, ref)


def test_noalloc_rejects_rows_beyond_the_scratch(dsa):
    """One score row of more than 4,194,304 keys does not fit: a clear error,
    nothing launched."""
    n_keys = (16 << 20) // 4 + 64
    q = torch.zeros(4, 64, 128, dtype=torch.uint8, device="cuda")
    k = torch.zeros(n_keys, 128, dtype=torch.uint8, device="cuda")
    s = torch.ones(n_keys, device="cuda")
    w = torch.zeros(4, 64, device="cuda")
    ind = dsa.indexer_in(q, k, w, s[:4], s)
    idx = torch.empty(4, 8, dtype=torch.int32, device="cuda")
    n0 = dsa.dsa_launch_counter()
    st = dsa.LIB.dsa_select_noalloc(ctypes.byref(ind.struct), 8, ctypes.c_void_p(idx.data_ptr()),
                                    8, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == dsa.DSA_ERR_WORKSPACE_TOO_SMALL
    assert dsa.dsa_launch_counter() == n0
