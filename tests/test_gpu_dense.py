"""Parity of the dense causal MLA-MQA attention (the baseline DSA replaces)
against the oracle's dense causal attention, and its identity with the sparse
path when the selection holds every preceding key."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_attention_long_tcgen05_b200.inputs import WORKLOADS, make_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    from sparse_attention_long_tcgen05_b200 import dsa
    import dsa_testlib as T
    return dsa, T


def _wl(L):
    return dataclasses.replace(WORKLOADS[1], name=f"prefill_L{L}", L=L)


def _dense(dsa, att, n_q):
    out = torch.empty(n_q, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(n_q, 128, device="cuda")
    dsa.dsa_dense_mqa_fwd(att, out, lse)
    assert dsa.dsa_check_status() == 0
    return out, lse


def test_dense_f32_tiny_all_rows(libs):
    dsa, T = libs
    inp = make_prefill(WORKLOADS[0], device="cuda", seed=0)
    L = inp.wl.L
    _, att = T.prefill_structs(inp)
    out = torch.empty(L, inp.wl.H, inp.wl.D_V, device="cuda")
    lse = torch.empty(L, inp.wl.H, device="cuda")
    dsa.dsa_dense_mqa_fwd(att, out, lse)
    assert dsa.dsa_check_status() == 0
    h = lambda t: t.double().cpu().numpy()
    o_ref, l_ref = O.dense_causal_attention(h(inp.q), h(inp.kv), h(inp.v), inp.wl.scale)
    T.assert_attention_close(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, max_abs=1e-4,
                             rel_rms=1e-5, lse_abs=1e-4)


@pytest.mark.parametrize("L", [1, 100, 700])
def test_dense_bf16_all_rows(libs, L):
    """One to eleven 64-key blocks per query, the last one ragged."""
    dsa, T = libs
    inp = make_prefill(_wl(L), device="cuda", seed=41)
    _, att = T.prefill_structs(inp)
    out, lse = _dense(dsa, att, L)
    kv = inp.kv.double().cpu().numpy()
    o_ref, l_ref = O.dense_causal_attention(inp.q.double().cpu().numpy(), kv, kv[:, :512],
                                            inp.wl.scale)
    T.assert_attention_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


def test_dense_equals_sparse_with_the_whole_prefix(libs):
    """Selecting every key 0..t (k >= t + 1) makes sparse attention the dense
    one: the two calls agree bit for bit on every row."""
    dsa, T = libs
    L, k = 1500, 2048
    inp = make_prefill(_wl(L), device="cuda", seed=42)
    _, att = T.prefill_structs(inp)
    ar = torch.arange(k, device="cuda", dtype=torch.int32)
    idx = torch.where(ar[None, :] <= torch.arange(L, device="cuda")[:, None], ar[None, :], -1)
    idx = idx.to(torch.int32).contiguous()
    out_s = torch.empty(L, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse_s = torch.empty(L, 128, device="cuda")
    dsa.dsa_sparse_mqa_fwd(att, idx, k, out_s, lse_s)
    assert dsa.dsa_check_status() == 0
    out_d, lse_d = _dense(dsa, att, L)
    assert torch.equal(out_d, out_s) and torch.equal(lse_d, lse_s)


def test_dense_late_chunk_sampled_rows(libs):
    """A chunk of 256 queries at positions 32512..32767 of a 32K sequence (512
    key blocks each), against the oracle on 12 sampled rows."""
    dsa, T = libs
    L, n_q = 32768, 256
    inp = make_prefill(_wl(L), device="cuda", seed=43)
    off = L - n_q
    att = dsa.attn_in(inp.q[off:], inp.kv, inp.wl.scale, 512)
    out, lse = _dense(dsa, att, n_q)
    rows = [0, 1, 97, 128, 200, 255, 13, 64, 150, 222, 31, 180]
    kv = inp.kv.double().cpu().numpy()
    for r in rows:
        t = off + r
        o_ref, l_ref, _ = O.attend(inp.q[t].double().cpu().numpy(), kv[:t + 1], kv[:t + 1, :512],
                                   inp.wl.scale)
        T.assert_attention_close(out[r].float().cpu().numpy(), lse[r].cpu().numpy(), o_ref,
                                 l_ref)


def test_dense_paged_equals_contiguous(libs):
    """Queries over a paged cache (shuffled 64-token pages, several queries per
    sequence at chosen positions) give the contiguous results bit for bit."""
    dsa, T = libs
    L = 3000
    inp = make_prefill(_wl(L), device="cuda", seed=44)
    n_pages = (L + 63) // 64
    perm = torch.randperm(n_pages, generator=torch.Generator().manual_seed(44)).cuda()
    kv_pad = torch.zeros(n_pages * 64, 576, dtype=torch.bfloat16, device="cuda")
    kv_pad[:L] = inp.kv
    kv_cache = torch.empty_like(kv_pad).view(n_pages, 64, 576)
    kv_cache[perm] = kv_pad.view(n_pages, 64, 576)
    table = perm.int().view(1, n_pages).contiguous()
    ctx = torch.tensor([L], dtype=torch.int32, device="cuda")
    pos = torch.tensor([0, 63, 64, 65, 1000, 2047, 2048, 2999], dtype=torch.int32, device="cuda")
    q_seq = torch.zeros(len(pos), dtype=torch.int32, device="cuda")
    lay = dsa.paged_layout(table, ctx, n_pages, q_seq, pos)
    q = inp.q[pos.long()].contiguous()
    att_p = dsa.attn_in(q, kv_cache, inp.wl.scale, 512, kv_layout=lay)
    out_p, lse_p = _dense(dsa, att_p, len(pos))
    _, att_c = T.prefill_structs(inp)
    out_c, lse_c = _dense(dsa, att_c, L)
    assert torch.equal(out_p, out_c[pos.long()]) and torch.equal(lse_p, lse_c[pos.long()])
