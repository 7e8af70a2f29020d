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


def _queries(wl, n_q, seed):
    """Synthetic query side for n_q query tokens (indexer q/w/scale, MQA q)."""
    from sparse_attention_long_tcgen05_b200.inputs import quantize_e4m3_per_token
    g = torch.Generator(device="cuda").manual_seed(seed)
    q_i = torch.randn(n_q, wl.H_I, wl.d_I, generator=g, device="cuda")
    w = torch.randn(n_q, wl.H_I, generator=g, device="cuda") / 8.0
    q = torch.randn(n_q, wl.H, wl.D_K, generator=g, device="cuda").to(torch.bfloat16)
    codes, scale = quantize_e4m3_per_token(q_i)
    return codes, scale, w.contiguous(), q.contiguous()


def test_decode_several_tokens_per_sequence(libs):
    """Multi-token decode / chunked prefill over the paged cache: m query tokens
    per sequence at positions ctx-m .. ctx-1 (explicit q_seq and q_pos, the
    queries of a sequence interleaved with other sequences'), checked per query
    against the oracle over keys 0..pos of its own sequence."""
    dsa, T = libs
    wl = dataclasses.replace(WORKLOADS[4], ctx_max=12000)
    ctx = [300, 2100, 5000, 64, 129, 12000]
    m = [3, 5, 1, 4, 2, 6]
    inp = make_decode(wl, device="cuda", seed=31, ctx_lens=ctx)
    seq_l, pos_l = [], []
    for b in range(len(ctx)):
        for j in range(m[b]):
            seq_l.append(b)
            pos_l.append(ctx[b] - m[b] + j)
    perm = np.random.default_rng(31).permutation(len(seq_l))
    seq_l = [seq_l[i] for i in perm]
    pos_l = [pos_l[i] for i in perm]
    n_q = len(seq_l)
    q_seq = torch.tensor(seq_l, dtype=torch.int32, device="cuda")
    q_pos = torch.tensor(pos_l, dtype=torch.int32, device="cuda")
    q_idx, q_scale, w, q = _queries(wl, n_q, seed=32)
    lay = dsa.paged_layout(inp.block_table, inp.ctx_lens, inp.num_pages, q_seq, q_pos)
    ind = dsa.indexer_in(q_idx, inp.k_cache, w, q_scale, inp.k_cache_scale.view(-1), kv=lay)
    att = dsa.attn_in(q, inp.kv_cache, wl.scale, 512, kv_layout=lay)
    k = wl.k
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, ind, att, 0, 0, k))
    idx = torch.empty(n_q, k, dtype=torch.int32, device="cuda")
    out = torch.empty(n_q, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(n_q, 128, device="cuda")
    dsa.dsa_forward(ind, att, k, idx, out, lse, ws)
    assert dsa.dsa_check_status() == 0
    max_cols = inp.block_table.shape[1] * 64
    scores = torch.empty(n_q, max_cols, device="cuda")
    dsa.dsa_indexer_scores(ind, None, n_q, scores, max_cols)
    assert dsa.dsa_check_status() == 0
    g_idx = idx.cpu().numpy()
    for i in range(n_q):
        b, p = seq_l[i], pos_l[i]
        row = inp.block_table[b]
        kc = _logical(inp.k_cache, row, p + 1).cpu().numpy()
        ks = _logical(inp.k_cache_scale[..., None], row, p + 1)[:, 0].cpu().numpy()
        k_deq = O.dequantize(kc, ks)
        q_deq = O.dequantize(q_idx[i].cpu().numpy()[None], q_scale[i:i + 1].cpu().numpy())
        ref = np.full(max_cols, -np.inf)
        ref[:p + 1] = O.indexer_row(q_deq[0], k_deq, w[i].double().cpu().numpy())
        g = scores[i].cpu().numpy()
        T.assert_indexer_close(g[None], ref[None])
        assert np.array_equal(g_idx[i], O.topk_row(g.astype(np.float64), p, k)), i
        kv_rows = _logical(inp.kv_cache, row, p + 1)
        sel = g_idx[i][g_idx[i] >= 0]
        kv_sel = kv_rows[torch.from_numpy(sel).long().cuda()].double().cpu().numpy()
        o_ref, l_ref, _ = O.attend(q[i].double().cpu().numpy(), kv_sel, kv_sel[:, :512], wl.scale)
        T.assert_attention_close(out[i].float().cpu().numpy(), lse[i].cpu().numpy(), o_ref, l_ref)
    # the selection-only calls agree with the fused one
    idx2 = torch.empty_like(idx)
    dsa.dsa_select(ind, k, idx2, dsa.workspace(
        dsa.dsa_workspace_size(dsa.DSA_OP_SELECT, ind, None, 0, 0, k)))
    assert dsa.dsa_check_status() == 0
    assert torch.equal(idx, idx2)


def test_paged_chunk_equals_contiguous_chunk(libs):
    """The last 300 tokens of a 5000-token prefill, once against the contiguous
    keys (n_q < n_keys) and once with the same keys written into shuffled
    64-token pages (q_seq = 0, q_pos = 4700..4999): the same indexer scores,
    selection and attention output, bit for bit."""
    dsa, T = libs
    from sparse_attention_long_tcgen05_b200.inputs import make_prefill
    L, m, k = 5000, 300, 2048
    wl = dataclasses.replace(WORKLOADS[1], L=L)
    inp = make_prefill(wl, device="cuda", seed=33)
    off = L - m
    ind_c = dsa.indexer_in(inp.q_idx[off:], inp.k_idx, inp.w[off:], inp.q_scale[off:],
                           inp.k_scale)
    att_c = dsa.attn_in(inp.q[off:], inp.kv, wl.scale, 512)
    # the same keys in shuffled pages
    n_pages = (L + 63) // 64
    perm = torch.randperm(n_pages, generator=torch.Generator().manual_seed(33)).cuda()
    k_pad = torch.zeros(n_pages * 64, 128, dtype=torch.uint8, device="cuda")
    s_pad = torch.ones(n_pages * 64, device="cuda")
    kv_pad = torch.zeros(n_pages * 64, 576, dtype=torch.bfloat16, device="cuda")
    k_pad[:L], s_pad[:L], kv_pad[:L] = inp.k_idx, inp.k_scale, inp.kv
    k_cache = torch.empty_like(k_pad).view(n_pages, 64, 128)
    s_cache = torch.empty_like(s_pad).view(n_pages, 64)
    kv_cache = torch.empty_like(kv_pad).view(n_pages, 64, 576)
    k_cache[perm] = k_pad.view(n_pages, 64, 128)
    s_cache[perm] = s_pad.view(n_pages, 64)
    kv_cache[perm] = kv_pad.view(n_pages, 64, 576)
    table = perm.int().view(1, n_pages).contiguous()
    ctx = torch.tensor([L], dtype=torch.int32, device="cuda")
    q_seq = torch.zeros(m, dtype=torch.int32, device="cuda")
    q_pos = torch.arange(off, L, dtype=torch.int32, device="cuda")
    lay = dsa.paged_layout(table, ctx, n_pages, q_seq, q_pos)
    ind_p = dsa.indexer_in(inp.q_idx[off:], k_cache, inp.w[off:], inp.q_scale[off:],
                           s_cache.view(-1), kv=lay)
    att_p = dsa.attn_in(inp.q[off:], kv_cache, wl.scale, 512, kv_layout=lay)
    res = []
    for ind, att in ((ind_c, att_c), (ind_p, att_p)):
        sc = torch.empty(m, L, device="cuda")
        dsa.dsa_indexer_scores(ind, None, m, sc, L)
        ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, ind, att, 0, 0, k))
        idx = torch.empty(m, k, dtype=torch.int32, device="cuda")
        out = torch.empty(m, 128, 512, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(m, 128, device="cuda")
        dsa.dsa_forward(ind, att, k, idx, out, lse, ws)
        assert dsa.dsa_check_status() == 0
        res.append((sc, idx, out, lse))
    (sc_c, idx_c, out_c, lse_c), (sc_p, idx_p, out_p, lse_p) = res
    assert torch.equal(sc_c, sc_p)
    assert torch.equal(idx_c, idx_p)
    assert torch.equal(out_c, out_p) and torch.equal(lse_c, lse_p)
