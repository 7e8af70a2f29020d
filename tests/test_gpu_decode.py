"""Parity of paged decode (one query per sequence against its 64-token-paged
FP8 key cache and bf16 latent cache, shuffled block table) against the oracle."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_attention_long_tcgen05_b200.inputs import WORKLOADS, make_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    from sparse_attention_long_tcgen05_b200 import dsa
    import dsa_testlib as T
    return dsa, T


def _structs(dsa, inp, block_table=None):
    bt = inp.block_table if block_table is None else block_table
    lay = dsa.paged_layout(bt, inp.ctx_lens, inp.num_pages)
    ind = dsa.indexer_in(inp.q_idx, inp.k_cache, inp.w, inp.q_scale,
                         inp.k_cache_scale.view(-1), kv=lay)
    att = dsa.attn_in(inp.q, inp.kv_cache, inp.wl.scale, 512, kv_layout=lay)
    ind.tensors.append(bt)
    att.tensors.append(bt)
    return ind, att


def _run(dsa, inp, block_table=None):
    ind, att = _structs(dsa, inp, block_table)
    B, k = inp.q.shape[0], inp.wl.k
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, ind, att, 0, 0, k))
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    out = torch.empty(B, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, 128, device="cuda")
    dsa.dsa_forward(ind, att, k, idx, out, lse, ws)
    assert dsa.dsa_check_status() == 0
    return ind, att, idx, out, lse


def _logical(cache, table_row, ctx):
    """Logical rows 0..ctx-1 of one sequence, gathered on the device."""
    n_pages = (ctx + 63) // 64
    pages = table_row[:n_pages].long()
    return cache[pages].reshape(n_pages * 64, *cache.shape[2:])[:ctx]


def _check(dsa, T, inp, ind, att, idx, out, lse, seqs):
    k = inp.wl.k
    max_cols = inp.block_table.shape[1] * 64
    scores = torch.empty(inp.q.shape[0], max_cols, device="cuda")
    dsa.dsa_indexer_scores(ind, None, inp.q.shape[0], scores, max_cols)
    assert dsa.dsa_check_status() == 0
    g_idx = idx.cpu().numpy()
    for b in seqs:
        ctx = int(inp.ctx_lens[b])
        row = inp.block_table[b]
        kc = _logical(inp.k_cache, row, ctx).cpu().numpy()
        ks = _logical(inp.k_cache_scale[..., None], row, ctx)[:, 0].cpu().numpy()
        k_deq = O.dequantize(kc, ks)
        q_deq = O.dequantize(inp.q_idx[b].cpu().numpy()[None], inp.q_scale[b:b + 1].cpu().numpy())
        ref = np.full(max_cols, -np.inf)
        ref[:ctx] = O.indexer_row(q_deq[0], k_deq, inp.w[b].double().cpu().numpy())
        g = scores[b].cpu().numpy()
        T.assert_indexer_close(g[None], ref[None])
        # fused selection == oracle top-k of the standalone scores (bit-exact)
        want = O.topk_row(g.astype(np.float64), ctx - 1, k)
        assert np.array_equal(g_idx[b], want), b
        # attention over those logical positions
        kv_rows = _logical(inp.kv_cache, row, ctx)
        sel = g_idx[b][g_idx[b] >= 0]
        kv_sel = kv_rows[torch.from_numpy(sel).long().cuda()].double().cpu().numpy()
        o_ref, l_ref, _ = O.attend(inp.q[b].double().cpu().numpy(), kv_sel, kv_sel[:, :512],
                                   inp.wl.scale)
        T.assert_attention_close(out[b].float().cpu().numpy(), lse[b].cpu().numpy(), o_ref, l_ref)


def test_decode_small_page_edges(libs):
    """Context lengths on and around page and tile boundaries, one of them a
    single token."""
    dsa, T = libs
    wl = dataclasses.replace(WORKLOADS[4], ctx_max=8192)
    inp = make_decode(wl, device="cuda", seed=2, ctx_lens=[1, 63, 64, 65, 127, 128, 129, 3000,
                                                            8192])
    ind, att, idx, out, lse = _run(dsa, inp)
    _check(dsa, T, inp, ind, att, idx, out, lse, range(inp.q.shape[0]))


def test_decode_block_table_permutation_invariance(libs):
    """Moving the pages (and the table with them) changes no output bit."""
    dsa, T = libs
    wl = dataclasses.replace(WORKLOADS[4], ctx_max=20000)
    inp = make_decode(wl, device="cuda", seed=3, ctx_lens=[20000, 777, 12345, 4096])
    _, _, idx_a, out_a, lse_a = _run(dsa, inp)
    perm = torch.randperm(inp.num_pages, device="cuda")
    inv = torch.argsort(perm)
    moved = dataclasses.replace(
        inp, k_cache=inp.k_cache[perm].contiguous(),
        k_cache_scale=inp.k_cache_scale[perm].contiguous(),
        kv_cache=inp.kv_cache[perm].contiguous(),
        block_table=torch.where(inp.block_table >= 0, inv[inp.block_table.long().clamp(min=0)],
                                -1).int().contiguous())
    _, _, idx_b, out_b, lse_b = _run(dsa, moved)
    assert torch.equal(idx_a, idx_b)
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b)


def test_decode_B64_full(libs):
    dsa, T = libs
    inp = make_decode(WORKLOADS[4], device="cuda", seed=0)
    ind, att, idx, out, lse = _run(dsa, inp)
    _check(dsa, T, inp, ind, att, idx, out, lse, range(inp.q.shape[0]))
