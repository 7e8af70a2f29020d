"""Parity of the sparse MQA attention backward (dsa_sparse_mqa_bwd: tcgen05
kernel through the C ABI) against the oracle's sparse_mqa_backward.

Inputs: the workloads' bf16 q and latent kv, a seeded upstream gradient and a
seeded valid selection drawn by torch (inputs.random_selection), so the check
does not depend on the indexer; the GPU forward provides out and lse, which the
backward consumes, while the oracle recomputes its own forward in float64.

Tolerances, from the arithmetic: the kernel rounds P and dZ to bf16 for the
tensor cores (relative 2^-9 per term) and exchanges the two CTAs' partial logits
and partial dP - D as fp16 (relative 2^-11 of those partial sums: for the logits
far below the bf16 rounding of P once scaled, for dP - D relative to the very
quantity dZ is proportional to); every dq and dkv element is a sum of many such terms with
independent rounding, so its error is a few 1e-3 of the typical magnitude of
the sum. The tests allow a relative RMS error of 1e-2 per tensor and a largest
element error of 2e-2 of the tensor's largest magnitude; rows of dq are checked
one by one against their own RMS (5e-2). dkv sums contributions of many queries
through fp32 reductions; where the full set of queries is too large for the
oracle, two exact identities of the gradient stand in: the key gradients of a
query sum to zero (so dkv's rope columns sum to zero over the rows) and its
value gradients sum to dO (so the first 512 columns sum to the sum of dO)."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_attention_long_tcgen05_b200.inputs import WORKLOADS, make_grad_out, make_prefill, \
    random_selection, sample_rows

pytestmark = pytest.mark.gpu

REL_RMS, MAX_REL, ROW_REL = 1e-2, 2e-2, 5e-2


@pytest.fixture(scope="module")
def dsa():
    from sparse_attention_long_tcgen05_b200 import dsa as d
    return d


def _wl(L, k=2048):
    return dataclasses.replace(WORKLOADS[1], name=f"prefill_L{L}", L=L, k=k)


def _backward(dsa, q, kv, idx, k, d_out, scale, n_keys):
    n_q = q.shape[0]
    att = dsa.attn_in(q, kv, scale, 512)
    assert kv.shape[0] == n_keys
    out = torch.empty(n_q, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(n_q, 128, device="cuda")
    dsa.dsa_sparse_mqa_fwd(att, idx, k, out, lse)
    dq = torch.full((n_q, 128, 576), float("nan"), dtype=torch.bfloat16, device="cuda")
    dkv = torch.zeros(kv.shape[0], 576, device="cuda")
    delta = torch.empty(n_q, 128, 2, device="cuda")
    dsa.dsa_sparse_mqa_bwd(att, idx, k, out, lse, d_out, dq, dkv, delta)
    assert dsa.dsa_check_status() == 0
    return out, dq, dkv, delta


def _close(got, ref, what):
    err = got - ref
    rms = np.sqrt(np.mean(err ** 2)) / max(np.sqrt(np.mean(ref ** 2)), 1e-30)
    mx = np.abs(err).max() / max(np.abs(ref).max(), 1e-30)
    print(f"{what}: rel-RMS {rms:.3g}, max {mx:.3g} of the largest magnitude")
    assert rms <= REL_RMS and mx <= MAX_REL, f"{what}: rel-RMS {rms:.3g}, max {mx:.3g}"
    return rms, mx


def _check_dq_rows(dq_got, dq_ref, rows):
    """Each row against its own RMS, floored at 1e-2 of the tensor's RMS: a row
    whose exact gradient vanishes (a query with one key: P = 1, dZ = dP - D = 0)
    keeps only rounding noise."""
    floor = 1e-2 * np.sqrt(np.mean(dq_ref ** 2))
    worst = 0.0
    for r, row in enumerate(rows):
        g, f = dq_got[r], dq_ref[r]
        scale = max(np.sqrt(np.mean(f ** 2)), floor, 1e-30)
        e = np.sqrt(np.mean((g - f) ** 2)) / scale
        worst = max(worst, e)
        assert e <= ROW_REL and np.abs(g - f).max() / scale <= 10 * ROW_REL, \
            f"dq row {row}: rel-RMS {e:.3g}, max {np.abs(g - f).max() / scale:.3g} of its RMS"
    print(f"dq rows: worst row rel-RMS {worst:.3g}")


def _all_rows(dsa, L, n_keys, k, seed):
    wl = _wl(n_keys, k)
    inp = make_prefill(wl, device="cuda", seed=seed)
    q = inp.q[n_keys - L:].contiguous()
    idx = random_selection(L, n_keys, k, device="cuda", seed=seed + 1)
    d_out = make_grad_out(L, device="cuda", seed=seed + 2)
    _, dq, dkv, _ = _backward(dsa, q, inp.kv, idx, k, d_out, wl.scale, n_keys)
    rows = list(range(L))
    dq_ref, dkv_ref = O.sparse_mqa_backward(q.double().cpu().numpy(), inp.kv.double().cpu().numpy(),
                                            idx.cpu().numpy(), rows,
                                            d_out.double().cpu().numpy(), wl.scale, 512)
    dq_h = dq.double().cpu().numpy()
    assert not np.isnan(dq_h).any()
    _close(dq_h, dq_ref, "dq")
    _check_dq_rows(dq_h, dq_ref, rows)
    _close(dkv.double().cpu().numpy(), dkv_ref, "dkv")


def test_bwd_every_row_dense_and_sparse(dsa):
    """L=300, k=128: rows 0..127 select their whole prefix (ragged last
    block), later rows 128 keys spread over it; every dq and dkv row."""
    _all_rows(dsa, 300, 300, 128, seed=61)


def test_bwd_k2048_query_suffix(dsa):
    """Query suffix (positions 2044..2299 of 2300 keys) with the full k=2048:
    32 key blocks per query; every dq and dkv row."""
    _all_rows(dsa, 256, 2300, 2048, seed=62)


def test_bwd_ragged_k(dsa):
    """k=1000 (15 full blocks and one of 40 keys), L=1200; every row."""
    _all_rows(dsa, 1200, 1200, 1000, seed=63)


def test_bwd_empty_and_single_key_rows(dsa):
    """A row with no valid entry gets dq = 0 and adds nothing to dkv; a row
    with one key attends to it alone (P = 1, dZ = 0, dV = dO)."""
    L, k = 200, 64
    wl = _wl(L, k)
    inp = make_prefill(wl, device="cuda", seed=64)
    idx = random_selection(L, L, k, device="cuda", seed=65)
    idx[7] = -1
    idx[150] = -1
    idx[150, 5] = 149
    d_out = make_grad_out(L, device="cuda", seed=66)
    _, dq, dkv, _ = _backward(dsa, inp.q, inp.kv, idx, k, d_out, wl.scale, L)
    assert torch.all(dq[7] == 0)
    rows = list(range(L))
    dq_ref, dkv_ref = O.sparse_mqa_backward(inp.q.double().cpu().numpy(),
                                            inp.kv.double().cpu().numpy(), idx.cpu().numpy(),
                                            rows, d_out.double().cpu().numpy(), wl.scale, 512)
    _close(dq.double().cpu().numpy(), dq_ref, "dq")
    _close(dkv.double().cpu().numpy(), dkv_ref, "dkv")


def _invariants(dkv, d_out, idx):
    """Column sums of dkv against the identities (float64 on the host)."""
    live = (idx >= 0).any(dim=1)
    col = dkv.double().sum(dim=0).cpu().numpy()
    want_v = d_out[live].double().sum(dim=(0, 1)).cpu().numpy()
    mag = dkv.double().abs().sum(dim=0).cpu().numpy()
    # each column sum is a sum of fp32 reductions of bf16-rounded terms: its
    # error is a small multiple of 2^-9 times the sum of magnitudes
    assert np.all(np.abs(col[512:]) <= 4e-3 * mag[512:] + 1e-3), np.abs(col[512:]).max()
    assert np.all(np.abs(col[:512] - want_v) <= 4e-3 * mag[:512] + 1e-3), \
        np.abs(col[:512] - want_v).max()


@pytest.mark.parametrize("wl_index,n_rows", [(1, 128), (3, 64)])
def test_bwd_full_size_sampled_rows(dsa, wl_index, n_rows):
    """The 4096 and 131072 prefills with k=2048: dq on seeded sampled rows
    against the oracle, dkv through the two column-sum identities."""
    wl = WORKLOADS[wl_index]
    L, k = wl.L, wl.k
    inp = make_prefill(wl, device="cuda", seed=0)
    idx = random_selection(L, L, k, device="cuda", seed=70)
    d_out = make_grad_out(L, device="cuda", seed=71)
    out, dq, dkv, _ = _backward(dsa, inp.q, inp.kv, idx, k, d_out, wl.scale, L)
    del out
    rows = sample_rows(L, n_rows, seed=1, k=k)
    r = torch.tensor(rows, device="cuda")
    idx_r = idx[r].cpu().numpy()
    used = np.unique(idx_r[idx_r >= 0])
    remap = np.full(L, -1, dtype=np.int64)
    remap[used] = np.arange(used.size)
    idx_local = np.where(idx_r >= 0, remap[np.maximum(idx_r, 0)], -1)
    kv_sub = inp.kv[torch.from_numpy(used).cuda()].double().cpu().numpy()
    dq_ref, _ = O.sparse_mqa_backward(inp.q[r].double().cpu().numpy(), kv_sub, idx_local,
                                      list(range(len(rows))), d_out[r].double().cpu().numpy(),
                                      wl.scale, 512)
    dq_h = dq[r].double().cpu().numpy()
    _close(dq_h, dq_ref, "dq")
    _check_dq_rows(dq_h, dq_ref, rows)
    _invariants(dkv, d_out, idx)


def test_bwd_strided_index_and_dkv(dsa):
    """An index row pitch larger than k and dkv rows wider than 576 floats: dq
    equals the contiguous call's bit for bit, dkv (whose fp32 reductions land
    in completion order) matches the oracle, and the padding of the wide dkv
    rows is left untouched."""
    L, k = 400, 192
    wl = _wl(L, k)
    inp = make_prefill(wl, device="cuda", seed=67)
    idx = random_selection(L, L, k, device="cuda", seed=68)
    d_out = make_grad_out(L, device="cuda", seed=69)
    _, dq_ref_gpu, _, _ = _backward(dsa, inp.q, inp.kv, idx, k, d_out, wl.scale, L)
    wide_idx = torch.full((L, k + 40), -7, dtype=torch.int32, device="cuda")
    wide_idx[:, :k] = idx
    att = dsa.attn_in(inp.q, inp.kv, wl.scale, 512)
    out = torch.empty(L, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(L, 128, device="cuda")
    dsa.dsa_sparse_mqa_fwd(att, idx, k, out, lse)
    dq = torch.empty(L, 128, 576, dtype=torch.bfloat16, device="cuda")
    dkv_wide = torch.full((L, 640), 3.0, device="cuda")
    dkv_wide[:, :576] = 0.0
    delta = torch.empty(L, 128, 2, device="cuda")
    dsa.dsa_sparse_mqa_bwd(att, wide_idx[:, :k], k, out, lse, d_out, dq, dkv_wide, delta)
    assert dsa.dsa_check_status() == 0
    assert torch.equal(dq, dq_ref_gpu)
    assert torch.all(dkv_wide[:, 576:] == 3.0)
    _, dkv_ref = O.sparse_mqa_backward(inp.q.double().cpu().numpy(), inp.kv.double().cpu().numpy(),
                                       idx.cpu().numpy(), list(range(L)),
                                       d_out.double().cpu().numpy(), wl.scale, 512)
    _close(dkv_wide[:, :576].double().cpu().numpy(), dkv_ref, "dkv (wide rows)")
