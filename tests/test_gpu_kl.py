"""Parity of the indexer's KL training signal (dsa_select_scored ->
dsa_sparse_mqa_fwd -> dsa_indexer_kl, tensor-core kernels through the C ABI)
against the oracle, on the GPU's own selection and selected scores.

Tolerances, from the arithmetic: the GPU forms p from the forward's log-sum-exp,
which matches the oracle within 2e-3 (the attention parity bound), so every
p_j -- and the gradient r_j - p_j, whose r_j comes from the same float32
scores -- may differ from the oracle by a relative ~2e-3 of p_j; the tests allow
|g - g_oracle| <= 5e-3 * p_j + 1e-7 per entry and a relative 5e-3 (+ 1e-4) on
the loss."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_attention_long_tcgen05_b200.inputs import WORKLOADS, make_decode, make_prefill, \
    sample_rows

pytestmark = pytest.mark.gpu

G_REL, G_ABS = 5e-3, 1e-7
KL_REL, KL_ABS = 5e-3, 1e-4


@pytest.fixture(scope="module")
def libs():
    from sparse_attention_long_tcgen05_b200 import dsa
    import dsa_testlib as T
    return dsa, T


def _wl(L, k=2048):
    return dataclasses.replace(WORKLOADS[1], name=f"prefill_L{L}", L=L, k=k)


def _signal(dsa, ind, att, n_q, k):
    """selection with its scores, forward lse, then the KL signal."""
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_SELECT, ind, None, 0, 0, k))
    idx = torch.empty(n_q, k, dtype=torch.int32, device="cuda")
    sel = torch.empty(n_q, k, device="cuda")
    dsa.dsa_select_scored(ind, k, idx, sel, ws)
    out = torch.empty(n_q, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(n_q, 128, device="cuda")
    dsa.dsa_sparse_mqa_fwd(att, idx, k, out, lse)
    loss = torch.empty(n_q, device="cuda")
    grad = torch.full((n_q, k), 9.0, device="cuda")
    dsa.dsa_indexer_kl(att, idx, k, lse, sel, loss, grad)
    assert dsa.dsa_check_status() == 0
    return idx, sel, loss, grad


def _check(q_rows, kv, idx, sel, loss, grad, scale):
    """q_rows [n, 128, 576] float64 host, kv [rows, 576] float64 host (the rows idx
    names), idx / sel / loss / grad GPU tensors of the same n rows."""
    idx_h = idx.cpu().numpy()
    sel_h = sel.double().cpu().numpy()
    p, kl, g = O.indexer_kl_rows(q_rows, kv, idx_h, list(range(len(idx_h))), scale, sel_h)
    gg = grad.double().cpu().numpy()
    assert np.all(gg[idx_h < 0] == 0.0)
    err = np.abs(gg - g)
    bad = err > G_REL * p + G_ABS
    assert not bad.any(), f"{bad.sum()} gradient entries out of tolerance; worst {err.max():.3g}"
    lg = loss.double().cpu().numpy()
    assert np.all(np.abs(lg - kl) <= KL_REL * np.abs(kl) + KL_ABS), \
        f"loss max rel err {np.max(np.abs(lg - kl) / np.maximum(np.abs(kl), 1e-30)):.3g}"
    return p, kl


def test_select_scored_equals_standalone_scores(libs):
    """The kept scores are the standalone indexer scores at the kept keys, bit
    for bit, and the selection is dsa_select's."""
    dsa, T = libs
    L, k = 3000, 2048
    inp = make_prefill(_wl(L, k), device="cuda", seed=51)
    ind, _ = T.prefill_structs(inp)
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_SELECT, ind, None, 0, 0, k))
    idx = torch.empty(L, k, dtype=torch.int32, device="cuda")
    sel = torch.empty(L, k, device="cuda")
    dsa.dsa_select_scored(ind, k, idx, sel, ws)
    idx2 = torch.empty_like(idx)
    dsa.dsa_select(ind, k, idx2, ws)
    scores = torch.empty(L, L, device="cuda")
    dsa.dsa_indexer_scores(ind, None, L, scores, L)
    assert dsa.dsa_check_status() == 0
    assert torch.equal(idx, idx2)
    want = torch.where(idx >= 0, torch.gather(scores, 1, idx.clamp(min=0).long()),
                       torch.full_like(sel, float("-inf")))
    assert torch.equal(sel, want)


@pytest.mark.parametrize("L,k", [(700, 256), (2500, 2048)])
def test_kl_prefill_every_row(libs, L, k):
    """Every row: rows with fewer than k preceding keys select all of them
    (the dense warm-up signal), the others their top k."""
    dsa, T = libs
    inp = make_prefill(_wl(L, k), device="cuda", seed=52)
    ind, att = T.prefill_structs(inp)
    idx, sel, loss, grad = _signal(dsa, ind, att, L, k)
    _check(inp.q.double().cpu().numpy(), inp.kv.double().cpu().numpy(), idx, sel, loss, grad,
           inp.wl.scale)


def test_kl_dense_stage_over_the_whole_prefix(libs):
    """With k >= t + 1 for every row the selection is the whole prefix: the
    signal is the dense warm-up's, against the oracle over keys 0..t with the
    full standalone score row."""
    dsa, T = libs
    L, k = 900, 1024
    inp = make_prefill(_wl(L, k), device="cuda", seed=53)
    ind, att = T.prefill_structs(inp)
    idx, sel, loss, grad = _signal(dsa, ind, att, L, k)
    scores = torch.empty(L, L, device="cuda")
    dsa.dsa_indexer_scores(ind, None, L, scores, L)
    sc = scores.double().cpu().numpy()
    q = inp.q.double().cpu().numpy()
    kv = inp.kv.double().cpu().numpy()
    lg = loss.double().cpu().numpy()
    gg = grad.double().cpu().numpy()
    for t in range(0, L, 37):
        p, _, kl, g = O.indexer_kl_row(q[t], kv[: t + 1], inp.wl.scale, sc[t, : t + 1])
        assert abs(lg[t] - kl) <= KL_REL * abs(kl) + KL_ABS
        assert np.all(np.abs(gg[t, : t + 1] - g) <= G_REL * p + G_ABS)


def test_kl_paged_decode(libs):
    """Decode over a shuffled paged cache, one query per sequence."""
    dsa, T = libs
    wl = dataclasses.replace(WORKLOADS[4], ctx_max=9000)
    inp = make_decode(wl, device="cuda", seed=54, ctx_lens=[1, 100, 2048, 2049, 5000, 9000])
    lay = dsa.paged_layout(inp.block_table, inp.ctx_lens, inp.num_pages)
    ind = dsa.indexer_in(inp.q_idx, inp.k_cache, inp.w, inp.q_scale, inp.k_cache_scale.view(-1),
                         kv=lay)
    att = dsa.attn_in(inp.q, inp.kv_cache, wl.scale, 512, kv_layout=lay)
    B, k = inp.q.shape[0], wl.k
    idx, sel, loss, grad = _signal(dsa, ind, att, B, k)
    lg = loss.double().cpu().numpy()
    gg = grad.double().cpu().numpy()
    idx_h = idx.cpu().numpy()
    sel_h = sel.double().cpu().numpy()
    for b in range(B):
        ctx = int(inp.ctx_lens[b])
        n_pages = (ctx + 63) // 64
        rows = inp.kv_cache[inp.block_table[b, :n_pages].long()].reshape(-1, 576)[:ctx]
        m = idx_h[b] >= 0
        keys = rows[torch.from_numpy(idx_h[b][m]).long().cuda()].double().cpu().numpy()
        p, _, kl, g = O.indexer_kl_row(inp.q[b].double().cpu().numpy(), keys, wl.scale,
                                       sel_h[b][m])
        assert abs(lg[b] - kl) <= KL_REL * abs(kl) + KL_ABS, (b, lg[b], kl)
        assert np.all(np.abs(gg[b][m] - g) <= G_REL * p + G_ABS), b


def test_kl_L32768_sampled_rows(libs):
    """The 32K workload (needles): the signal of every row is computed, 128
    seeded rows are checked against the oracle."""
    dsa, T = libs
    inp = make_prefill(WORKLOADS[2], device="cuda", seed=0)
    L, k = inp.wl.L, inp.wl.k
    ind, att = T.prefill_structs(inp)
    idx, sel, loss, grad = _signal(dsa, ind, att, L, k)
    rows = sample_rows(L, 128, seed=1)
    r = torch.tensor(rows, device="cuda")
    kv_sub, idx_local = T.gather_kv_rows(inp.kv, idx[r].cpu().numpy())
    _check(inp.q[r].double().cpu().numpy(), kv_sub, torch.from_numpy(idx_local).cuda(), sel[r],
           loss[r], grad[r], inp.wl.scale)


def test_kl_ragged_k_tight_gradient_rows(libs):
    """k = 100 (the last 64-key block holds 36 entries) with a gradient exactly
    k wide: every row matches the oracle, and nothing is written past the last
    row (a guard region after the buffer keeps its values)."""
    dsa, T = libs
    L, k = 300, 100
    inp = make_prefill(_wl(L, k), device="cuda", seed=55)
    ind, att = T.prefill_structs(inp)
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_SELECT, ind, None, 0, 0, k))
    idx = torch.empty(L, k, dtype=torch.int32, device="cuda")
    sel = torch.empty(L, k, device="cuda")
    dsa.dsa_select_scored(ind, k, idx, sel, ws)
    out = torch.empty(L, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(L, 128, device="cuda")
    dsa.dsa_sparse_mqa_fwd(att, idx, k, out, lse)
    loss = torch.empty(L, device="cuda")
    buf = torch.full((L * k + 4096,), 7.0, device="cuda")
    grad = buf[: L * k].view(L, k)
    dsa.dsa_indexer_kl(att, idx, k, lse, sel, loss, grad)
    assert dsa.dsa_check_status() == 0
    assert torch.all(buf[L * k:] == 7.0)
    _check(inp.q.double().cpu().numpy(), inp.kv.double().cpu().numpy(), idx, sel, loss, grad,
           inp.wl.scale)
