"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each check takes the oracle function it pins as an argument so that
test_pins_catch_planted_mistakes can run the same check against a copy of the
oracle with a planted mistake (on the CPU) and see it fail.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _num(x):
    if isinstance(x, str):
        return float(x)          # "nan", "-inf", "-0.0"
    return float(x)


# ----------------------------------------------------------------- checks

def check_e4m3_golden(decode):
    g = _load("e4m3_codes.json")
    codes = np.array([c["code"] for c in g["cases"]], dtype=np.uint8)
    got = decode(codes)
    for c, v in zip(g["cases"], got):
        want = _num(c["value"])
        if math.isnan(want):
            assert math.isnan(v), c
        else:
            assert v == want and math.copysign(1, v) == math.copysign(1, want), (c, v)


def check_e4m3_vs_torch(decode):
    """All 256 codes against torch's float8_e4m3fn -> float32 conversion."""
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float32)
    ref = ref.double().numpy()
    got = decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin])


def check_indexer_golden(indexer_scores):
    g = _load("indexer_worked_example.json")
    q = np.array(g["q"], dtype=np.float64)
    k = np.array(g["k"], dtype=np.float64)
    w = np.array(g["w"], dtype=np.float64)
    exp = np.array([[_num(x) for x in row] for row in g["expected"]])
    got = indexer_scores(q, k, w, [0, 1, 2], [0, 1, 2], 3)
    assert np.array_equal(np.isneginf(got), np.isneginf(exp))
    fin = np.isfinite(exp)
    assert np.allclose(got[fin], exp[fin], rtol=0, atol=1e-15)


def _indexer_bruteforce(q, k, w, t):
    """Explicit loops, one multiply-add at a time."""
    H, d = q.shape[1], q.shape[2]
    out = []
    for s in range(t + 1):
        acc = 0.0
        for j in range(H):
            dot = 0.0
            for c in range(d):
                dot += float(q[t, j, c]) * float(k[s, c])
            acc += float(w[t, j]) * (dot if dot > 0 else 0.0)
        out.append(acc)
    return np.array(out)


def check_indexer_bruteforce(indexer_scores):
    rng = np.random.default_rng(5)
    L, H, d = 9, 3, 5
    q = rng.standard_normal((L, H, d))
    k = rng.standard_normal((L, d))
    w = rng.standard_normal((L, H))
    rows = list(range(L))
    got = indexer_scores(q, k, w, rows, rows, L)
    for t in rows:
        ref = _indexer_bruteforce(q, k, w, t)
        assert np.allclose(got[t, : t + 1], ref, rtol=1e-12, atol=1e-12)
        assert np.all(np.isneginf(got[t, t + 1:]))


def check_indexer_properties(indexer_scores):
    rng = np.random.default_rng(6)
    L, H, d = 12, 4, 8
    q = rng.standard_normal((L, H, d))
    k = rng.standard_normal((L, d))
    w_pos = rng.uniform(0, 1, (L, H))
    rows = list(range(L))
    base = indexer_scores(q, k, w_pos, rows, rows, L)
    # w >= 0 => every score >= 0 (ReLU gating)
    assert np.all(base[np.isfinite(base)] >= 0)
    # positive homogeneity in k (ReLU(c x) = c ReLU(x) for c > 0): the
    # needle workload's x3 keys rely on it
    c = 3.0
    scaled = indexer_scores(q, c * k, w_pos, rows, rows, L)
    fin = np.isfinite(base)
    assert np.allclose(scaled[fin], c * base[fin], rtol=1e-12, atol=1e-12)
    # a negative dot contributes nothing: flipping k where every head's dot is
    # negative gives a zero score
    one_head_q = np.zeros((L, 1, d)); one_head_q[:, 0, 0] = 1.0
    kk = np.zeros((L, d)); kk[:, 0] = -np.arange(1, L + 1)
    ww = np.ones((L, 1))
    z = indexer_scores(one_head_q, kk, ww, rows, rows, L)
    assert np.all(z[np.isfinite(z)] == 0.0)


def check_topk_golden(topk_row):
    g = _load("topk_worked_example.json")
    scores = np.array([_num(x) for x in g["scores"]])
    for case in g["cases"]:
        got = topk_row(scores, case["pos"], case["k"])
        assert got.tolist() == case["expected"], (case, got)


def _topk_by_rank(scores, pos, k):
    """Independent selection: keep s iff fewer than k candidates beat it,
    where a beats b iff a.score > b.score or (equal score and a.index < b.index)."""
    n = pos + 1
    v = [float(x) + 0.0 for x in scores[:n]]
    keep = []
    for s in range(n):
        beaten_by = sum(1 for a in range(n) if v[a] > v[s] or (v[a] == v[s] and a < s))
        if beaten_by < k:
            keep.append(s)
    return keep + [-1] * (k - len(keep))


def check_topk_bruteforce(topk_row):
    rng = np.random.default_rng(7)
    for trial in range(60):
        n = int(rng.integers(1, 70))
        k = int(rng.integers(1, 40))
        # few distinct values (many ties), both signed zeros
        pool = np.array([-2.0, -0.0, 0.0, 0.5, 1.0, 3.0])
        scores = rng.choice(pool, size=n)
        if trial % 3 == 0:
            scores = rng.standard_normal(n)
        pos = n - 1
        got = topk_row(scores, pos, k).tolist()
        assert got == _topk_by_rank(scores, pos, k), (scores, k, got)


def check_topk_invariants(topk_row):
    rng = np.random.default_rng(8)
    for _ in range(20):
        n = int(rng.integers(1, 300))
        k = int(rng.integers(1, 64))
        scores = np.round(rng.standard_normal(n), 1)   # ties
        got = topk_row(scores, n - 1, k)
        sel = got[got >= 0]
        assert sel.size == min(k, n)
        assert np.all(np.diff(sel) > 0) and (sel.size == 0 or sel[-1] <= n - 1)
        assert np.all(got[sel.size:] == -1)
        out = np.setdiff1d(np.arange(n), sel)
        if out.size and sel.size:
            # every excluded score <= every included; equal only at a higher index
            assert scores[out].max() <= scores[sel].min()
            eq_out = out[scores[out] == scores[sel].min()]
            eq_in = sel[scores[sel] == scores[sel].min()]
            if eq_out.size:
                assert eq_out.min() > eq_in.max()
    # all-equal scores select the first k positions
    assert topk_row(np.zeros(100), 99, 10).tolist() == list(range(10))


def check_attention_golden(attend):
    g = _load("attention_worked_example.json")
    out, lse, p = attend(np.array(g["q"]), np.array(g["keys"]), np.array(g["values"]),
                         g["scale"])
    assert np.allclose(out, np.array(g["expected_out"]), rtol=1e-13, atol=1e-13)
    assert np.allclose(lse, np.array(g["expected_lse"]), rtol=1e-13, atol=1e-13)


def check_sparse_equals_dense(sparse_mqa, topk_row):
    """k >= t+1 selects every prefix key, so sparse attention must equal dense
    causal attention; the dense reference is torch's scaled_dot_product_attention
    (is_causal=True) in float64."""
    rng = np.random.default_rng(9)
    L, H, dk, dv = 20, 3, 6, 4
    q = rng.standard_normal((L, H, dk))
    kv = rng.standard_normal((L, dk))
    scale = 1 / math.sqrt(dk)
    k = L
    rows = list(range(L))
    scores = rng.standard_normal((L, L))
    idx = np.stack([topk_row(scores[t], t, k) for t in rows])
    out, lse = sparse_mqa(q, kv, None, idx, rows, scale, dv)
    tq = torch.from_numpy(q).permute(1, 0, 2)[None]           # [1, H, L, dk]
    tk = torch.from_numpy(kv)[None, None].expand(1, H, L, dk)
    tv = torch.from_numpy(kv[:, :dv])[None, None].expand(1, H, L, dv)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True,
                                                           scale=scale)
    ref = ref[0].permute(1, 0, 2).numpy()
    assert np.allclose(out, ref, rtol=1e-10, atol=1e-12)
    # lse against the log of the causal partition function
    z = scale * np.einsum("thd,sd->ths", q, kv)
    mask = np.tril(np.ones((L, L), dtype=bool))[:, None, :]
    ref_lse = np.log(np.where(mask, np.exp(z), 0.0).sum(-1))
    assert np.allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def check_dense_vs_sdpa(dense):
    rng = np.random.default_rng(10)
    L, H, dk, dv = 17, 2, 5, 3
    q = rng.standard_normal((L, H, dk))
    k = rng.standard_normal((L, dk))
    v = rng.standard_normal((L, dv))
    scale = 0.7
    out, _ = dense(q, k, v, scale)
    tq = torch.from_numpy(q).permute(1, 0, 2)[None]
    tk = torch.from_numpy(k)[None, None].expand(1, H, L, dk)
    tv = torch.from_numpy(v)[None, None].expand(1, H, L, dv)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True,
                                                           scale=scale)[0].permute(1, 0, 2)
    assert np.allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)


def check_attention_properties(attend, sparse_mqa_row):
    rng = np.random.default_rng(11)
    H, n, dk, dv = 4, 33, 8, 6
    q_t = rng.standard_normal((H, dk))
    keys = rng.standard_normal((n, dk))
    vals = rng.standard_normal((n, dv))
    out, lse, p = attend(q_t, keys, vals, 0.3)
    assert np.allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    # one selected key: output is exactly that value row
    kv = rng.standard_normal((10, dk))
    one = np.array([4, -1, -1])
    o1, l1 = sparse_mqa_row(q_t, kv, None, one, 0.3, dv)
    assert np.array_equal(o1, np.broadcast_to(kv[4, :dv], (H, dv)))
    assert np.allclose(l1, 0.3 * (q_t @ kv[4]), rtol=1e-13, atol=1e-13)
    # permuting the KV rows together with the indices changes nothing
    perm = rng.permutation(10)
    inv = np.argsort(perm)
    idx = np.array([0, 3, 7, 9, -1])
    oa, la = sparse_mqa_row(q_t, kv, None, idx, 0.3, dv)
    ob, lb = sparse_mqa_row(q_t, kv[perm], None, inv[idx[:4]].tolist() + [-1], 0.3, dv)
    assert np.allclose(oa, ob, rtol=1e-12, atol=1e-12)
    assert np.allclose(la, lb, rtol=1e-12, atol=1e-12)


def _kl_case(seed=0, H=3, n=7, d=5):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((H, d)), rng.standard_normal((n, d)), 0.7,
            rng.standard_normal(n) * 2.0)


def check_kl_gradient_finite_differences(kl_row):
    """d kl / d scores from central differences of the loss itself."""
    q, keys, scale, sc = _kl_case(1)
    _, _, _, g = kl_row(q, keys, scale, sc)
    eps = 1e-6
    fd = np.zeros_like(sc)
    for i in range(sc.size):
        e = np.zeros_like(sc)
        e[i] = eps
        fd[i] = (kl_row(q, keys, scale, sc + e)[2] - kl_row(q, keys, scale, sc - e)[2]) / (2 * eps)
    assert np.allclose(g, fd, atol=1e-8), (g, fd)


def check_kl_zero_at_match(kl_row):
    """KL >= 0, and it vanishes (with its gradient) exactly when the indexer's
    distribution equals the target: scores = log p + c."""
    q, keys, scale, sc = _kl_case(2)
    p, r, kl, g = kl_row(q, keys, scale, sc)
    assert kl > 1e-3 and abs(p.sum() - 1.0) < 1e-12 and abs(r.sum() - 1.0) < 1e-12
    assert abs(g.sum()) < 1e-12
    p2, r2, kl2, g2 = kl_row(q, keys, scale, np.log(p) + 3.25)
    assert abs(kl2) < 1e-12 and np.abs(g2).max() < 1e-12 and np.allclose(r2, p)


def check_kl_one_head_is_softmax(kl_row):
    """With one head the target is that head's softmax of the scaled logits
    (torch's softmax); with two heads it is the mean of the two."""
    q, keys, scale, sc = _kl_case(3, H=2)
    p1 = kl_row(q[:1], keys, scale, sc)[0]
    t = torch.softmax(torch.from_numpy(scale * (q[:1] @ keys.T)), dim=-1)[0].numpy()
    assert np.allclose(p1, t, atol=1e-13)
    p2 = kl_row(q, keys, scale, sc)[0]
    t2 = torch.softmax(torch.from_numpy(scale * (q @ keys.T)), dim=-1).mean(0).numpy()
    assert np.allclose(p2, t2, atol=1e-13)


def check_kl_bruteforce(kl_row):
    """Python loops with math.exp / math.log on a tiny case."""
    import math
    q, keys, scale, sc = _kl_case(4, H=2, n=3, d=2)
    H, n = q.shape[0], keys.shape[0]
    p = [0.0] * n
    for h in range(H):
        z = [scale * sum(q[h, c] * keys[i, c] for c in range(q.shape[1])) for i in range(n)]
        den = sum(math.exp(x) for x in z)
        for i in range(n):
            p[i] += math.exp(z[i]) / den / H
    den = sum(math.exp(x) for x in sc)
    r = [math.exp(x) / den for x in sc]
    kl = sum(p[i] * (math.log(p[i]) - math.log(r[i])) for i in range(n))
    P, R, KL, G = kl_row(q, keys, scale, sc)
    assert np.allclose(P, p, atol=1e-14) and np.allclose(R, r, atol=1e-14)
    assert abs(KL - kl) < 1e-13 and np.allclose(G, np.array(r) - np.array(p), atol=1e-14)


def check_kl_dense_stage_reduction(kl_rows, topk_row):
    """With k >= t + 1 the selection is every preceding key, so the sparse-stage
    signal over the selection is the dense warm-up signal over the whole prefix
    (computed here directly from the row's keys 0..t)."""
    rng = np.random.default_rng(5)
    L, H, d = 9, 4, 6
    q = rng.standard_normal((L, H, d))
    kv = rng.standard_normal((L, d))
    scores = rng.standard_normal((L, L))
    rows = list(range(L))
    idx = np.stack([topk_row(scores[t], t, 16) for t in rows])
    sel = np.where(idx >= 0, np.take_along_axis(scores, np.maximum(idx, 0), 1), -np.inf)
    p, kl, g = kl_rows(q, kv, idx, rows, 0.5, sel)
    for t in rows:
        P, R, KL, G = O.indexer_kl_row(q[t], kv[: t + 1], 0.5, scores[t, : t + 1])
        assert abs(kl[t] - KL) < 1e-12 and np.allclose(p[t, : t + 1], P, atol=1e-14)
        assert np.allclose(g[t, : t + 1], G, atol=1e-14) and np.all(g[t, t + 1:] == 0)


def _bwd_case(seed=0, L=6, H=2, d=5, dv=3):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((L, H, d))
    kv = rng.standard_normal((L + 2, d))
    d_out = rng.standard_normal((L, H, dv))
    idx = np.full((L, 4), -1)
    for t in range(L):
        sel = rng.choice(L + 2, size=min(t + 1, 4), replace=False)
        idx[t, : sel.size] = np.sort(sel)
    return q, kv, d_out, idx


def check_bwd_finite_differences(bwd):
    """dq and dkv against central differences of loss = sum(dO * O), O from the
    (separately pinned) forward sparse_mqa."""
    q, kv, d_out, idx = _bwd_case(7)
    rows = list(range(q.shape[0]))
    scale, dv = 0.7, d_out.shape[2]

    def loss(qq, kk):
        out, _ = O.sparse_mqa(qq, kk, None, idx, rows, scale, dv)
        return float(np.sum(out * d_out))

    dq, dkv = bwd(q, kv, idx, rows, d_out, scale, dv)
    eps = 1e-6
    fq = np.zeros_like(q)
    for i in np.ndindex(q.shape):
        e = np.zeros_like(q)
        e[i] = eps
        fq[i] = (loss(q + e, kv) - loss(q - e, kv)) / (2 * eps)
    fk = np.zeros_like(kv)
    for i in np.ndindex(kv.shape):
        e = np.zeros_like(kv)
        e[i] = eps
        fk[i] = (loss(q, kv + e) - loss(q, kv - e)) / (2 * eps)
    assert np.allclose(dq, fq, atol=1e-7), np.abs(dq - fq).max()
    assert np.allclose(dkv, fk, atol=1e-7), np.abs(dkv - fk).max()


def check_bwd_vs_torch_autograd(bwd):
    """Selecting every preceding key reduces the sparse gradient to dense causal
    MQA attention's, taken here from torch autograd through
    scaled_dot_product_attention (float64, CPU), with the keys broadcast over
    the heads and the values the first dv columns of the same rows."""
    rng = np.random.default_rng(8)
    L, H, d, dv, scale = 7, 3, 6, 4, 0.45
    q = rng.standard_normal((L, H, d))
    kv = rng.standard_normal((L, d))
    d_out = rng.standard_normal((L, H, dv))
    idx = np.stack([O.topk_row(np.zeros(L), t, L) for t in range(L)])
    dq, dkv = bwd(q, kv, idx, list(range(L)), d_out, scale, dv)
    tq = torch.from_numpy(q).permute(1, 0, 2)[None].clone().requires_grad_(True)
    tkv = torch.from_numpy(kv).clone().requires_grad_(True)
    k = tkv[None, None].expand(1, H, L, d)
    v = tkv[None, None, :, :dv].expand(1, H, L, dv)
    out = torch.nn.functional.scaled_dot_product_attention(tq, k, v, is_causal=True, scale=scale)
    out.backward(torch.from_numpy(d_out).permute(1, 0, 2)[None])
    assert np.allclose(dq, tq.grad[0].permute(1, 0, 2).numpy(), atol=1e-12)
    assert np.allclose(dkv, tkv.grad.numpy(), atol=1e-12)


def check_bwd_invariants(bwd):
    """Exact at any size: every softmax row's logit gradient sums to zero, so
    the key gradients of a query sum to zero and the rope columns of dkv (keys
    only) sum to zero over the rows; the value gradients of a query sum to its
    dO (the probabilities sum to one), so the first dv columns of dkv sum to the
    sum of dO over queries with a non-empty selection and over heads. A query
    with an empty selection gets dq = 0."""
    q, kv, d_out, idx = _bwd_case(9, L=12, H=3, d=7, dv=4)
    idx[5] = -1
    rows = list(range(q.shape[0]))
    dq, dkv = bwd(q, kv, idx, rows, d_out, 0.6, 4)
    assert np.allclose(dkv[:, 4:].sum(axis=0), 0.0, atol=1e-12)
    live = [t for t in rows if (idx[t] >= 0).any()]
    assert np.allclose(dkv[:, :4].sum(axis=0), d_out[live].sum(axis=(0, 1)), atol=1e-12)
    assert np.all(dq[5] == 0.0)


def check_paged(paged_rows):
    rng = np.random.default_rng(12)
    P, n_pages, d = 4, 7, 3
    logical = rng.standard_normal((n_pages * P, d))
    table = rng.permutation(n_pages)
    cache = np.zeros((n_pages, P, d))
    for lp, phys in enumerate(table):
        cache[phys] = logical[lp * P:(lp + 1) * P]
    ctx = n_pages * P - 2
    assert np.array_equal(paged_rows(cache, table, ctx), logical[:ctx])


def check_dequantize_roundtrip(dequantize):
    """quantize (torch float8 cast, per-token amax/448 scale) then dequantize
    reproduces the input within e4m3's half-ulp (2^-4 relative for normals)."""
    from sparse_attention_long_tcgen05_b200.inputs import quantize_e4m3_per_token
    g = torch.Generator().manual_seed(3)
    x = torch.randn(16, 4, 32, generator=g)
    codes, scale = quantize_e4m3_per_token(x)
    back = dequantize(codes.numpy(), scale.numpy())
    xs = x.double().numpy()
    amax = np.abs(xs).reshape(16, -1).max(1)[:, None, None]
    err = np.abs(back - xs)
    # normal range: relative 2^-4; subnormal range: absolute 2^-10 of amax
    assert np.all(err <= np.maximum(np.abs(xs) * 2.0 ** -4, amax * 2.0 ** -10) + 1e-12)
    # the largest element of each token maps to exactly +-448 * scale
    assert np.allclose(np.abs(back).reshape(16, -1).max(1), amax[:, 0, 0], rtol=1e-6)


# ----------------------------------------------------------------- tests

def test_e4m3_golden():
    check_e4m3_golden(O.e4m3_decode)


def test_e4m3_vs_torch():
    check_e4m3_vs_torch(O.e4m3_decode)


def test_dequantize_roundtrip():
    check_dequantize_roundtrip(O.dequantize)


def test_indexer_golden():
    check_indexer_golden(O.indexer_scores)


def test_indexer_bruteforce():
    check_indexer_bruteforce(O.indexer_scores)


def test_indexer_properties():
    check_indexer_properties(O.indexer_scores)


def test_topk_golden():
    check_topk_golden(O.topk_row)


def test_topk_bruteforce():
    check_topk_bruteforce(O.topk_row)


def test_topk_invariants():
    check_topk_invariants(O.topk_row)


def test_attention_golden():
    check_attention_golden(O.attend)


def test_sparse_equals_dense_causal():
    check_sparse_equals_dense(O.sparse_mqa, O.topk_row)


def test_dense_vs_sdpa():
    check_dense_vs_sdpa(O.dense_causal_attention)


def test_attention_properties():
    check_attention_properties(O.attend, O.sparse_mqa_row)


def test_kl_gradient_finite_differences():
    check_kl_gradient_finite_differences(O.indexer_kl_row)


def test_kl_zero_at_match():
    check_kl_zero_at_match(O.indexer_kl_row)


def test_kl_one_head_is_softmax():
    check_kl_one_head_is_softmax(O.indexer_kl_row)


def test_kl_bruteforce():
    check_kl_bruteforce(O.indexer_kl_row)


def test_kl_dense_stage_reduction():
    check_kl_dense_stage_reduction(O.indexer_kl_rows, O.topk_row)


def test_bwd_finite_differences():
    check_bwd_finite_differences(O.sparse_mqa_backward)


def test_bwd_vs_torch_autograd():
    check_bwd_vs_torch_autograd(O.sparse_mqa_backward)


def test_bwd_invariants():
    check_bwd_invariants(O.sparse_mqa_backward)


def test_paged_rows():
    check_paged(O.paged_rows)


def test_forward_prefill_rows_consistent():
    """The whole-forward helper is the composition of the pinned steps."""
    rng = np.random.default_rng(13)
    L, HI, dI, H, dk, dv, k = 40, 3, 8, 2, 6, 4, 7
    qi = rng.standard_normal((L, HI, dI)); ki = rng.standard_normal((L, dI))
    w = rng.standard_normal((L, HI)); q = rng.standard_normal((L, H, dk))
    kv = rng.standard_normal((L, dk))
    rows = [0, 5, 6, 39]
    sc, idx, out, lse = O.forward_prefill_rows(qi, ki, w, q, kv, None, rows, k, 0.5, dv)
    for r, t in enumerate(rows):
        assert idx[r].tolist() == O.topk_row(sc[r], t, k).tolist()
        o, l = O.sparse_mqa_row(q[t], kv, None, idx[r], 0.5, dv)
        assert np.array_equal(out[r], o) and np.array_equal(lse[r], l)


# ------------------------------------------------- planted mistakes (CPU)

def _mut_decode_bias(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    v = O.e4m3_decode(codes)
    return v * 2.0                                   # wrong exponent bias


def _mut_decode_subnormal(codes):
    v = O.e4m3_decode(codes).copy()
    c = np.asarray(codes, dtype=np.uint8)
    sub = ((c >> 3) & 0xF) == 0
    v[sub] = v[sub] * 2                              # subnormal scale 2^-5
    return v


def _mut_indexer_no_relu(q, k, w, rows, q_pos, n_cols):
    out = np.full((len(rows), n_cols), -np.inf)
    for r, (row, pos) in enumerate(zip(rows, q_pos)):
        out[r, : pos + 1] = w[row] @ (q[row] @ k[: pos + 1].T)
    return out


def _mut_indexer_exclusive(q, k, w, rows, q_pos, n_cols):
    out = O.indexer_scores(q, k, w, rows, q_pos, n_cols)
    for r, pos in enumerate(q_pos):
        out[r, pos] = -np.inf                        # drops the s == t key
    return out


def _mut_indexer_relu_after_sum(q, k, w, rows, q_pos, n_cols):
    out = np.full((len(rows), n_cols), -np.inf)
    for r, (row, pos) in enumerate(zip(rows, q_pos)):
        out[r, : pos + 1] = np.maximum(w[row] @ (q[row] @ k[: pos + 1].T), 0)
    return out


def _mut_topk_higher_index_wins(scores, pos, k):
    n = pos + 1
    v = np.asarray(scores, dtype=np.float64)[:n] + 0.0
    order = np.lexsort((-np.arange(n), -v))
    keep = np.sort(order[: min(k, n)])
    out = np.full(k, -1, dtype=np.int32); out[: keep.size] = keep
    return out


def _mut_topk_exclusive(scores, pos, k):
    return O.topk_row(scores, pos - 1, k) if pos > 0 else O.topk_row(scores, pos, k)


def _mut_topk_signed_zero(scores, pos, k):
    n = pos + 1
    v = np.asarray(scores, dtype=np.float64)[:n]
    key = np.where(np.signbit(v) & (v == 0), -1e-300, v)   # -0.0 ranked below +0.0
    order = np.lexsort((np.arange(n), -key))
    keep = np.sort(order[: min(k, n)])
    out = np.full(k, -1, dtype=np.int32); out[: keep.size] = keep
    return out


def _mut_attend_no_scale(q_t, keys, values, scale):
    return O.attend(q_t, keys, values, 1.0)


def _mut_attend_transposed(q_t, keys, values, scale):
    out, lse, p = O.attend(q_t, keys, values, scale)
    z = scale * (np.asarray(q_t) @ np.asarray(keys).T)
    p2 = np.exp(z - z.max(axis=0, keepdims=True))
    p2 = p2 / p2.sum(axis=0, keepdims=True)          # softmax over heads
    return p2 @ np.asarray(values), lse, p2


def _mut_sparse_mqa_v_offset(q, kv, v, idx, rows, scale, d_v):
    kv = np.asarray(kv)
    shifted = np.concatenate([kv[:, 1:], kv[:, :1]], axis=1)  # V = columns 1..d_v
    out, lse = O.sparse_mqa(q, kv, v, idx, rows, scale, d_v)
    out2, _ = O.sparse_mqa(q, shifted, v, idx, rows, scale, d_v)
    return out2, lse


def _mut_paged_slot(cache, table_row, ctx):
    cache = np.asarray(cache)
    n_pages = (ctx + cache.shape[1] - 1) // cache.shape[1]
    return cache[np.sort(np.asarray(table_row)[:n_pages])].reshape(-1, cache.shape[2])[:ctx]


def _mut_dequantize_divide(codes, scale):
    x = O.e4m3_decode(codes)
    s = np.asarray(scale, dtype=np.float64)
    return x / s.reshape(s.shape + (1,) * (x.ndim - s.ndim))


def _mut_kl_reversed(q_t, keys, scale, scores):
    p, r, _, g = O.indexer_kl_row(q_t, keys, scale, scores)
    return p, r, float(np.sum(r * (np.log(r) - np.log(p)))), g      # KL(r || p)


def _mut_kl_head_sum(q_t, keys, scale, scores):
    _, _, probs = O.attend(q_t, keys, np.asarray(keys)[:, :1], scale)
    p = probs.sum(axis=0)                                            # not averaged
    s = np.asarray(scores, dtype=np.float64)
    r = np.exp(s - s.max()); r /= r.sum()
    return p, r, float(np.sum(p * (np.log(p) - np.log(r)))), r - p


def _mut_kl_grad_sign(q_t, keys, scale, scores):
    p, r, kl, g = O.indexer_kl_row(q_t, keys, scale, scores)
    return p, r, kl, -g


def _mut_kl_softmax_over_heads(q_t, keys, scale, scores):
    z = scale * (np.asarray(q_t) @ np.asarray(keys).T)
    e = np.exp(z - z.max(axis=0, keepdims=True))
    p = (e / e.sum(axis=0, keepdims=True)).mean(axis=0)              # softmax across heads
    s = np.asarray(scores, dtype=np.float64)
    r = np.exp(s - s.max()); r /= r.sum()
    return p, r, float(np.sum(p * (np.log(p) - np.log(r)))), r - p


def _mut_bwd(no_delta=False, dk_scale=True, with_dv=True, dv_off=0):
    def bwd(q, kv, idx, rows, d_out, scale, d_v):
        q = np.asarray(q)
        kv = np.asarray(kv, dtype=np.float64)
        dq = np.zeros((len(rows),) + q.shape[1:])
        dkv = np.zeros(kv.shape)
        for r, row in enumerate(rows):
            sel = idx[r][idx[r] >= 0]
            if sel.size == 0:
                continue
            keys = kv[sel]
            vals = keys[:, :d_v]
            out, _, p = O.attend(q[row], keys, vals, scale)
            dp = d_out[r] @ vals.T
            delta = 0.0 if no_delta else np.sum(d_out[r] * out, axis=1, keepdims=True)
            dz = p * (dp - delta)
            dq[r] = scale * dz @ keys
            np.add.at(dkv, sel, (scale if dk_scale else 1.0) * dz.T @ q[row])
            if with_dv:
                np.add.at(dkv[:, dv_off:dv_off + d_v], sel, p.T @ d_out[r])
        return dq, dkv
    return bwd


PLANTED = [
    ("bwd no delta", lambda: check_bwd_finite_differences(_mut_bwd(no_delta=True))),
    ("bwd dk unscaled", lambda: check_bwd_finite_differences(_mut_bwd(dk_scale=False))),
    ("bwd value grad dropped", lambda: check_bwd_invariants(_mut_bwd(with_dv=False))),
    ("bwd value grad offset", lambda: check_bwd_vs_torch_autograd(_mut_bwd(dv_off=2))),
    ("kl reversed", lambda: check_kl_gradient_finite_differences(_mut_kl_reversed)),
    ("kl head sum", lambda: check_kl_zero_at_match(_mut_kl_head_sum)),
    ("kl grad sign", lambda: check_kl_gradient_finite_differences(_mut_kl_grad_sign)),
    ("kl softmax over heads", lambda: check_kl_one_head_is_softmax(_mut_kl_softmax_over_heads)),
    ("decode bias", lambda: check_e4m3_golden(_mut_decode_bias)),
    ("decode bias/torch", lambda: check_e4m3_vs_torch(_mut_decode_bias)),
    ("decode subnormal", lambda: check_e4m3_vs_torch(_mut_decode_subnormal)),
    ("dequant divide", lambda: check_dequantize_roundtrip(_mut_dequantize_divide)),
    ("indexer no relu", lambda: check_indexer_golden(_mut_indexer_no_relu)),
    ("indexer no relu/brute", lambda: check_indexer_bruteforce(_mut_indexer_no_relu)),
    ("indexer exclusive", lambda: check_indexer_golden(_mut_indexer_exclusive)),
    ("indexer relu after sum", lambda: check_indexer_golden(_mut_indexer_relu_after_sum)),
    ("topk higher index", lambda: check_topk_golden(_mut_topk_higher_index_wins)),
    ("topk exclusive", lambda: check_topk_golden(_mut_topk_exclusive)),
    ("topk signed zero", lambda: check_topk_golden(_mut_topk_signed_zero)),
    ("topk signed zero/brute", lambda: check_topk_bruteforce(_mut_topk_signed_zero)),
    ("attend no scale", lambda: check_attention_properties(_mut_attend_no_scale, O.sparse_mqa_row)
     or check_sparse_equals_dense(
         lambda q, kv, v, idx, rows, s, dv: O.sparse_mqa(q, kv, v, idx, rows, 1.0, dv),
         O.topk_row)),
    ("attend transposed", lambda: check_attention_golden(_mut_attend_transposed)),
    ("sparse V offset", lambda: check_sparse_equals_dense(_mut_sparse_mqa_v_offset, O.topk_row)),
    ("paged slot order", lambda: check_paged(_mut_paged_slot)),
]


@pytest.mark.parametrize("name,run", PLANTED, ids=[p[0] for p in PLANTED])
def test_pins_catch_planted_mistakes(name, run):
    with pytest.raises(AssertionError):
        run()
