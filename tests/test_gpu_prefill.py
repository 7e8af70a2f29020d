"""Parity of the FP8-indexer / bf16-attention prefill path (tensor-core
kernels, called through the C ABI) against the oracle.

Small cases cover every row and end in ragged tails (key tiles of 128, query
groups of 4, key blocks of 64); the L=4096 workload is checked on every row
(indexer values and mask, the selection, the attention output); the 32K and
128K workloads on the same seeded sample of 512 query rows, in the launch
configuration the benchmark times (dsa_forward)."""
import dataclasses
import os

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_attention_long_tcgen05_b200.inputs import WORKLOADS, make_prefill, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    from sparse_attention_long_tcgen05_b200 import dsa
    import dsa_testlib as T
    return dsa, T


def _wl(L, k=2048):
    return dataclasses.replace(WORKLOADS[1], name=f"prefill_L{L}", L=L, k=k)


def _scores(dsa, ind, rows_list, n_cols):
    rows = torch.tensor(rows_list, dtype=torch.int32, device="cuda")
    out = torch.empty(len(rows_list), n_cols, device="cuda")
    dsa.dsa_indexer_scores(ind, rows, len(rows_list), out, n_cols)
    assert dsa.dsa_check_status() == 0
    return out


@pytest.mark.parametrize("L", [1, 130, 777])
def test_indexer_fp8_small_all_rows(libs, L):
    dsa, T = libs
    inp = make_prefill(_wl(L), device="cuda", seed=3)
    ind, _ = T.prefill_structs(inp)
    scores = torch.full((L, L + 5), 7.0, device="cuda")
    dsa.dsa_indexer_scores(ind, None, L, scores, L)
    assert dsa.dsa_check_status() == 0
    g = scores.cpu().numpy()
    assert np.all(g[:, L:] == 7.0), "wrote past n_cols"
    rows = list(range(L))
    qi, ki, w, _ = T.oracle_prefill_inputs(inp, rows)
    ref = T.oracle_scores(qi, ki, w, rows, L)
    T.assert_indexer_close(g[:, :L], ref)


def test_indexer_fp8_query_suffix_positions(libs):
    """n_q < n_keys: query i sits at position n_keys - n_q + i (chunked prefill)."""
    dsa, T = libs
    L, n_q = 1000, 300
    inp = make_prefill(_wl(L), device="cuda", seed=4)
    off = L - n_q
    ind = dsa.indexer_in(inp.q_idx[off:], inp.k_idx, inp.w[off:], inp.q_scale[off:],
                         inp.k_scale)
    scores = torch.empty(n_q, L, device="cuda")
    dsa.dsa_indexer_scores(ind, None, n_q, scores, L)
    assert dsa.dsa_check_status() == 0
    rows = list(range(off, L))
    qi, ki, w, _ = T.oracle_prefill_inputs(inp, rows)
    ref = T.oracle_scores(qi, ki, w, rows, L)
    T.assert_indexer_close(scores.cpu().numpy(), ref)


def test_indexer_rows_subset_bitexact_with_all_rows(libs):
    """Scores for an arbitrary row subset equal the all-rows scores bit for bit
    (rows are grouped 4 to an MMA in any order)."""
    dsa, T = libs
    L = 1100
    inp = make_prefill(_wl(L), device="cuda", seed=5)
    ind, _ = T.prefill_structs(inp)
    full = torch.empty(L, L, device="cuda")
    dsa.dsa_indexer_scores(ind, None, L, full, L)
    rows = [1099, 3, 640, 641, 0, 17, 1000]
    sub = _scores(dsa, ind, rows, L)
    assert torch.equal(sub, full[torch.tensor(rows, device="cuda")])


def test_topk_bitexact_L4096_all_rows(libs):
    dsa, T = libs
    inp = make_prefill(WORKLOADS[1], device="cuda", seed=0)
    L, k = inp.wl.L, inp.wl.k
    ind, _ = T.prefill_structs(inp)
    scores = torch.empty(L, L, device="cuda")
    dsa.dsa_indexer_scores(ind, None, L, scores, L)
    idx = torch.empty(L, k, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(scores, torch.arange(L, dtype=torch.int32, device="cuda"), k, idx)
    assert dsa.dsa_check_status() == 0
    ref = T.topk_oracle_on(scores.double().cpu().numpy(), np.arange(L), k)
    assert np.array_equal(idx.cpu().numpy(), ref)


def test_topk_ties_and_signed_zero(libs):
    dsa, T = libs
    rng = np.random.default_rng(1)
    R, n = 37, 5000
    pool = np.array([-1.0, -0.0, 0.0, 0.25, 2.0, -np.inf, np.nan], dtype=np.float32)
    s = rng.choice(pool, size=(R, n)).astype(np.float32)
    s[5] = 0.0
    s[6] = -0.0
    s[7] = rng.standard_normal(n).astype(np.float32)
    pos = rng.integers(0, n, R).astype(np.int32)
    pos[:3] = [0, 2047, n - 1]
    for k in (1, 7, 2048):
        idx = torch.empty(R, k, dtype=torch.int32, device="cuda")
        dsa.dsa_topk(torch.from_numpy(s).cuda(), torch.from_numpy(pos).cuda(), k, idx)
        assert dsa.dsa_check_status() == 0
        ref = T.topk_oracle_on(s.astype(np.float64), pos, k)
        assert np.array_equal(idx.cpu().numpy(), ref), k


def test_topk_heavy_ties_fallback(libs):
    """More tied contenders than the shared-memory collection holds: the exact
    select over the row in global memory takes over and gives the same rule."""
    dsa, T = libs
    rng = np.random.default_rng(2)
    R, n = 6, 30000
    s = rng.choice(np.array([1.0, 2.0], dtype=np.float32), size=(R, n), p=[0.4, 0.6])
    s[1] = 5.0
    s[2, ::3] = 7.0
    s[3] = rng.standard_normal(n).astype(np.float32)   # no ties: collection path
    pos = np.array([n - 1, n - 1, 25000, n - 1, 15000, 2048], dtype=np.int32)
    for k in (2048, 100):
        idx = torch.empty(R, k, dtype=torch.int32, device="cuda")
        dsa.dsa_topk(torch.from_numpy(s).cuda(), torch.from_numpy(pos).cuda(), k, idx)
        assert dsa.dsa_check_status() == 0
        ref = T.topk_oracle_on(s.astype(np.float64), pos, k)
        assert np.array_equal(idx.cpu().numpy(), ref), k


def test_topk_row_layouts(libs):
    """Score rows read as float4 (16-byte aligned rows, pitch a multiple of 4)
    and rows read one score at a time (odd pitch or an unaligned first row),
    each with ragged lengths, give the oracle's selection bit for bit; rows of
    subnormal scores put the selection threshold among the subnormals."""
    dsa, T = libs
    rng = np.random.default_rng(11)
    R, n = 24, 9000
    pos = rng.integers(2040, n, R).astype(np.int32)
    pos[:4] = [n - 1, n - 2, n - 3, n - 4]
    for pitch, offset in ((9000, 0), (9004, 0), (9003, 0), (9004, 1), (9001, 3)):
        buf = torch.from_numpy(rng.standard_normal(R * pitch + offset).astype(np.float32))
        buf[offset:].view(R, pitch)[:, :n:7] = 2.5          # ties around the k-th score
        rows = buf[offset:].view(R, pitch)
        rows[4] *= 1e-41                                    # subnormal scores only
        rows[5] = -rows[5].abs() * 1e-42                    # negative subnormals and zeros
        rows[5, ::5] = 0.0
        rows[5, 1::5] = -0.0
        s = buf.cuda()[offset:offset + R * pitch].view(R, pitch)[:, :n]
        for k in (2048, 33):
            idx = torch.empty(R, k, dtype=torch.int32, device="cuda")
            dsa.dsa_topk(s, torch.from_numpy(pos).cuda(), k, idx)
            assert dsa.dsa_check_status() == 0
            ref = T.topk_oracle_on(s.double().cpu().numpy(), pos, k)
            assert np.array_equal(idx.cpu().numpy(), ref), (pitch, offset, k)


def test_topk_long_rows(libs):
    """Rows of up to 70,000 scores, bit for bit against the oracle's selection:
    random rows, a row whose large scores sit in regularly spaced 32-score runs,
    ties around the k-th score, all-equal rows (signed zeros included),
    non-finite values, and lengths of 16,384 and 16,389."""
    dsa, T = libs
    rng = np.random.default_rng(7)
    n = 70000
    R = 8
    s = rng.standard_normal((R, n)).astype(np.float32)
    n_lines = (n + 31) // 32                           # row 1: large values in spaced runs
    for li in [q * n_lines // 256 for q in range(136)]:
        s[1, 32 * li:32 * li + 32] = 10.0 + rng.random(32, dtype=np.float32)
    s[2] = rng.choice(np.array([0.5, 1.0, 1.5, 3.0], dtype=np.float32), size=n,
                      p=[0.5, 0.3, 0.17, 0.03])         # ties around the k-th score
    s[3] = 4.0                                          # all equal
    s[4, rng.integers(0, n, 5000)] = np.nan
    s[4, rng.integers(0, n, 5000)] = -np.inf
    s[4, rng.integers(0, n, 300)] = np.inf
    s[5] = np.abs(s[5]) * np.where(rng.random(n) < 0.5, -0.0, 0.0).astype(np.float32)
    pos = np.array([n - 1, n - 1, n - 1, 60000, n - 1, n - 1, 16383, 16388], dtype=np.int32)
    for k in (2048, 64, 1):
        idx = torch.empty(R, k, dtype=torch.int32, device="cuda")
        dsa.dsa_topk(torch.from_numpy(s).cuda(), torch.from_numpy(pos).cuda(), k, idx)
        assert dsa.dsa_check_status() == 0
        ref = T.topk_oracle_on(s.astype(np.float64), pos, k)
        assert np.array_equal(idx.cpu().numpy(), ref), k


def _attention_case(dsa, T, L, k, seed, rows=None):
    inp = make_prefill(_wl(L, k), device="cuda", seed=seed)
    rng = np.random.default_rng(seed)
    idx_h = T.topk_oracle_on(rng.standard_normal((L, L)), np.arange(L), k)
    idx = torch.from_numpy(idx_h).cuda()
    _, att = T.prefill_structs(inp)
    out = torch.empty(L, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(L, 128, device="cuda")
    dsa.dsa_sparse_mqa_fwd(att, idx, k, out, lse)
    assert dsa.dsa_check_status() == 0
    rows = list(range(L)) if rows is None else rows
    q = inp.q[torch.tensor(rows, device="cuda")].double().cpu().numpy()
    kv_sub, idx_local = T.gather_kv_rows(inp.kv, idx_h[rows])
    o_ref, l_ref = O.sparse_mqa(q, kv_sub, None, idx_local, list(range(len(rows))),
                                inp.wl.scale, 512)
    r = torch.tensor(rows, device="cuda")
    return T.assert_attention_close(out[r].float().cpu().numpy(), lse[r].cpu().numpy(), o_ref,
                                    l_ref)


def test_attention_bf16_dense_prefix(libs):
    """k >= L: every row attends to its whole prefix (one to five 64-key blocks,
    the last one ragged)."""
    dsa, T = libs
    _attention_case(dsa, T, L=300, k=2048, seed=6)


def test_attention_bf16_ragged_k(libs):
    dsa, T = libs
    _attention_case(dsa, T, L=1000, k=300, seed=7)


def test_attention_bf16_L4096_sampled(libs):
    dsa, T = libs
    rows = sample_rows(4096, 96, seed=1)
    _attention_case(dsa, T, L=4096, k=2048, seed=0, rows=rows)


def test_attention_single_key_rows(libs):
    """Rows whose selection is one key output that key's value row (softmax of
    one logit is 1)."""
    dsa, T = libs
    L = 200
    inp = make_prefill(_wl(L), device="cuda", seed=8)
    k = 64
    idx = torch.full((L, k), -1, dtype=torch.int32, device="cuda")
    sel = torch.randint(0, L, (L,), device="cuda")
    sel = torch.minimum(sel, torch.arange(L, device="cuda"))
    ar = torch.arange(L, device="cuda")
    idx[ar, (ar * 7) % k] = sel.int()
    _, att = T.prefill_structs(inp)
    out = torch.empty(L, 128, 512, dtype=torch.bfloat16, device="cuda")
    dsa.dsa_sparse_mqa_fwd(att, idx, k, out, None)
    assert dsa.dsa_check_status() == 0
    want = inp.kv[sel.long(), :512][:, None, :].expand(L, 128, 512)
    assert torch.equal(out, want)


def _forward(dsa, T, inp):
    wl = inp.wl
    L, k = wl.L, wl.k
    ind, att = T.prefill_structs(inp)
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, ind, att, 0, 0, k))
    idx = torch.empty(L, k, dtype=torch.int32, device="cuda")
    out = torch.empty(L, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(L, 128, device="cuda")
    dsa.dsa_forward(ind, att, k, idx, out, lse, ws)
    assert dsa.dsa_check_status() == 0
    return ind, att, idx, out, lse


def _check_forward_rows(dsa, T, inp, ind, att, idx, out, lse, rows, chunk=128):
    """Element-wise parity of the fused forward on the given query rows,
    checked in chunks of rows so the host copies stay bounded at 128K:
    indexer values against the oracle, the fused selection against the
    oracle's top-k of the same float32 scores (bit-exact), and the attention
    output against the oracle's attention over that selection."""
    wl = inp.wl
    L, k = wl.L, wl.k
    k_deq = T.oracle_key_side(inp)
    overlaps = []
    for c0 in range(0, len(rows), chunk):
        part = list(rows[c0:c0 + chunk])
        # indexer values on these rows
        sc = _scores(dsa, ind, part, L)
        qi, w, q = T.oracle_query_side(inp, part)
        ref_scores = T.oracle_scores(qi, k_deq, w, part, L)
        g_sc = sc.cpu().numpy()
        T.assert_indexer_close(g_sc, ref_scores)
        # the fused selection equals top-k of the standalone scores, bit for
        # bit, and equals the oracle's top-k of those same scores
        r = torch.tensor(part, device="cuda")
        g_idx = idx[r].cpu().numpy()
        ref_idx = T.topk_oracle_on(g_sc.astype(np.float64), np.array(part), k)
        assert np.array_equal(g_idx, ref_idx)
        # attention on these rows with those indices
        kv_sub, idx_local = T.gather_kv_rows(inp.kv, g_idx)
        o_ref, l_ref = O.sparse_mqa(q, kv_sub, None, idx_local, list(range(len(part))),
                                    wl.scale, 512)
        T.assert_attention_close(out[r].float().cpu().numpy(), lse[r].cpu().numpy(), o_ref,
                                 l_ref)
        # diagnostic: overlap with the oracle's own selection (its own scores)
        own = T.topk_oracle_on(ref_scores, np.array(part), k)
        overlaps += [len(set(a[a >= 0]) & set(b[b >= 0])) / max(1, (b >= 0).sum())
                     for a, b in zip(g_idx, own)]
    assert np.mean(overlaps) > 0.95, np.mean(overlaps)


def test_forward_L4096(libs):
    dsa, T = libs
    inp = make_prefill(WORKLOADS[1], device="cuda", seed=0)
    ind, att, idx, out, lse = _forward(dsa, T, inp)
    L, k = inp.wl.L, inp.wl.k
    # every row: the fused selection is the standalone top-k of standalone scores
    scores = torch.empty(L, L, device="cuda")
    dsa.dsa_indexer_scores(ind, None, L, scores, L)
    idx_s = torch.empty(L, k, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(scores, torch.arange(L, dtype=torch.int32, device="cuda"), k, idx_s)
    assert torch.equal(idx, idx_s)
    out_s = torch.empty_like(out)
    lse_s = torch.empty_like(lse)
    dsa.dsa_sparse_mqa_fwd(att, idx_s, k, out_s, lse_s)
    assert torch.equal(out, out_s) and torch.equal(lse, lse_s)
    # structure of the selection: causal, ascending, min(k, t+1) entries
    ih = idx.cpu().numpy()
    cnt = (ih >= 0).sum(1)
    assert np.array_equal(cnt, np.minimum(k, np.arange(L) + 1))
    assert np.all(ih.max(1) <= np.arange(L))
    # every row: indexer values, selection and attention against the oracle
    _check_forward_rows(dsa, T, inp, ind, att, idx, out, lse, list(range(L)), chunk=512)


@pytest.mark.parametrize("L", [5000, 16384])
def test_forward_score_blocks_every_row(libs, L):
    """Prefills whose scores span several blocks (5000: 4144 rows, then a ragged
    856; 16384: 13 blocks of 1184 rows and a ragged 992), so each indexer launch
    after the first overwrites the block the previous top-k reads: the fused
    selection equals the standalone top-k of the standalone scores in every
    row."""
    dsa, T = libs
    inp = make_prefill(_wl(L), device="cuda", seed=3)
    ind, att, idx, out, lse = _forward(dsa, T, inp)
    L, k = inp.wl.L, inp.wl.k
    scores = torch.empty(L, L, device="cuda")
    dsa.dsa_indexer_scores(ind, None, L, scores, L)
    idx_s = torch.empty(L, k, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(scores, torch.arange(L, dtype=torch.int32, device="cuda"), k, idx_s)
    assert dsa.dsa_check_status() == 0
    assert torch.equal(idx, idx_s)


def test_forward_L32768_needles(libs):
    dsa, T = libs
    inp = make_prefill(WORKLOADS[2], device="cuda", seed=0)
    ind, att, idx, out, lse = _forward(dsa, T, inp)
    rows = sample_rows(inp.wl.L, 512, seed=1)
    _check_forward_rows(dsa, T, inp, ind, att, idx, out, lse, rows)
    # the planted x3 keys are over-represented in the selections of long rows
    needles = set(inp.needles.cpu().tolist())
    ih = idx.cpu().numpy()
    long_rows = [t for t in rows if t >= 8192]
    frac = np.mean([np.isin(ih[t][ih[t] >= 0], list(needles)).mean() for t in long_rows])
    base = 64 / 4096
    # a x3 key clears a selection threshold that keeps ~5-25% of the prefix
    # about 2-4x as often as an ordinary key
    assert frac > 2 * base, frac


@pytest.mark.skipif(os.environ.get("DSA_SKIP_128K") == "1", reason="DSA_SKIP_128K=1")
def test_forward_L131072_sampled(libs):
    dsa, T = libs
    inp = make_prefill(WORKLOADS[3], device="cuda", seed=0)
    ind, att, idx, out, lse = _forward(dsa, T, inp)
    n = int(os.environ.get("DSA_128K_ROWS", "512"))
    rows = sample_rows(inp.wl.L, n, seed=1)
    _check_forward_rows(dsa, T, inp, ind, att, idx, out, lse, rows)
    ih = idx[torch.tensor(rows, device="cuda")].cpu().numpy()
    assert np.array_equal((ih >= 0).sum(1), np.minimum(2048, np.array(rows) + 1))


def _suffix_structs(dsa, inp, off):
    """Structs for the queries off..L-1 of a prefill against all L keys (a
    chunk of a longer prefill): query i sits at position off + i."""
    wl = inp.wl
    ind = dsa.indexer_in(inp.q_idx[off:], inp.k_idx, inp.w[off:], inp.q_scale[off:],
                         inp.k_scale)
    att = dsa.attn_in(inp.q[off:], inp.kv, wl.scale, wl.D_V)
    return ind, att


def test_attention_bf16_query_suffix(libs):
    """Chunked prefill: 300 queries at positions 700..999 attend over their own
    selections among 1000 keys (entries up to each query's position)."""
    dsa, T = libs
    L, off, k = 1000, 700, 512
    inp = make_prefill(_wl(L, k), device="cuda", seed=21)
    rng = np.random.default_rng(21)
    rows = np.arange(off, L)
    idx_h = T.topk_oracle_on(rng.standard_normal((L - off, L)), rows, k)
    _, att = _suffix_structs(dsa, inp, off)
    out = torch.empty(L - off, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(L - off, 128, device="cuda")
    dsa.dsa_sparse_mqa_fwd(att, torch.from_numpy(idx_h).cuda(), k, out, lse)
    assert dsa.dsa_check_status() == 0
    q = inp.q[off:].double().cpu().numpy()
    kv_sub, idx_local = T.gather_kv_rows(inp.kv, idx_h)
    o_ref, l_ref = O.sparse_mqa(q, kv_sub, None, idx_local, list(range(L - off)), inp.wl.scale,
                                512)
    T.assert_attention_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


@pytest.mark.parametrize("L,off", [(3000, 1700), (9000, 8000)])
def test_forward_query_suffix_every_row(libs, L, off):
    """dsa_forward on a chunk of a longer prefill (queries off..L-1 against all
    L keys; 9000/8000 gives rows with more than k candidates and a suffix that
    is not a multiple of the 4-query groups): every row's indexer values,
    selection and attention against the oracle at the query's own position,
    and the selection equals the same rows of the whole prefill's selection."""
    dsa, T = libs
    k = 2048
    inp = make_prefill(_wl(L, k), device="cuda", seed=22)
    ind, att = _suffix_structs(dsa, inp, off)
    n_q = L - off
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, ind, att, 0, 0, k))
    idx = torch.empty(n_q, k, dtype=torch.int32, device="cuda")
    out = torch.empty(n_q, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(n_q, 128, device="cuda")
    dsa.dsa_forward(ind, att, k, idx, out, lse, ws)
    assert dsa.dsa_check_status() == 0
    # standalone scores of the suffix rows (row r = query r, position off + r)
    sc = torch.empty(n_q, L, device="cuda")
    dsa.dsa_indexer_scores(ind, None, n_q, sc, L)
    assert dsa.dsa_check_status() == 0
    pos = np.arange(off, L)
    k_deq = T.oracle_key_side(inp)
    qi, w, q = T.oracle_query_side(inp, list(pos))
    ref = T.oracle_scores(qi, k_deq, w, list(pos), L)
    g_sc = sc.cpu().numpy()
    T.assert_indexer_close(g_sc, ref)
    g_idx = idx.cpu().numpy()
    assert np.array_equal(g_idx, T.topk_oracle_on(g_sc.astype(np.float64), pos, k))
    kv_sub, idx_local = T.gather_kv_rows(inp.kv, g_idx)
    o_ref, l_ref = O.sparse_mqa(q, kv_sub, None, idx_local, list(range(n_q)), inp.wl.scale, 512)
    T.assert_attention_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)
    # the same rows of the whole prefill select the same keys
    full_ind, _ = T.prefill_structs(inp)
    ws2 = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_SELECT, full_ind, None, 0, 0, k))
    idx_full = torch.empty(L, k, dtype=torch.int32, device="cuda")
    dsa.dsa_select(full_ind, k, idx_full, ws2)
    assert dsa.dsa_check_status() == 0
    assert torch.equal(idx_full[off:], idx)
