"""Plain CPU oracle of the DeepSeek Sparse Attention (DSA) forward path.

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module; the library never does. It shares no
code, table or constant generator with the CUDA path.

Every step is the plain definition, in float64, with numpy library primitives
(matmul, sort) as the only building blocks:

  1. e4m3 decode and per-token dequantisation of the indexer inputs;
  2. the lightning indexer score I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s])
     over the causal prefix s <= t;
  3. fine-grained top-k selection: the min(k, t+1) best keys by
     (score descending, index ascending), emitted in ascending index order and
     padded with -1;
  4. MQA-mode attention of all query heads over the selected shared latent KV
     rows (V = the first d_v columns of the KV row), with the exact softmax and
     its log-sum-exp;
  5. dense causal attention, used to pin step 4 and as the dense baseline;
  6. the indexer's KL training signal over a key set;
  7. the gradient of step 4 with respect to the queries and the latent KV rows
     (the main model's sparse training over the same selection).

Sources (web pages on DeepSeek-V3.2 / V3.2-Exp):
  [53ai]  "DeepSeek-V3.2-Exp 技术报告解读" (53ai.com), section
          "创新架构：DeepSeek稀疏注意力的核心设计" (the core design of DSA) and
          its Figure 1 (DSA inside MLA).
  [juhe]  report read-through on juhe.plus, steps "第一步：Lightning Indexer"
          and "第二步：Fine-grained Token Selection".
  [pb]    paperbridge.wiki summary of arXiv 2512.02556, sections
          "密集注意力" (dense attention) and "DeepSeek Sparse Attention".
  [amaranth] engineering report on wiki-for-amaranth, section "DeepSeek
          Sparse Attention (DSA)" (indexer trained by a KL loss; stages A, B).
  [ocp]   OCP 8-bit floating point specification, E4M3 format (the pages only
          say "FP8"; the e4m3 variant and per-token scales are the workload's).

Parity unpinned: none of the functions below; every one has an independent
pin in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import numpy as np


# ---------------------------------------------------------------- step 1: FP8

def e4m3_decode(codes) -> np.ndarray:
    """Value of each e4m3 code [ocp]: bit 7 sign, bits 6..3 exponent (bias 7),
    bits 2..0 mantissa; exponent 0 is subnormal (m/8 * 2^-6); exponent 15 with
    mantissa 7 is NaN; there is no infinity (largest finite 448)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    subnormal = (m / 8.0) * 2.0 ** -6
    val = np.where(e == 0, subnormal, normal)
    val = np.where((e == 15) & ((c & 0x7) == 7), np.nan, val)
    return sign * val


def dequantize(codes, scale) -> np.ndarray:
    """x = decode(code) * scale[token] (one scale per leading index)."""
    x = e4m3_decode(codes)
    s = np.asarray(scale, dtype=np.float64)
    return x * s.reshape(s.shape + (1,) * (x.ndim - s.ndim))


# ------------------------------------------------------------ step 2: indexer

def indexer_row(q_t, k_prefix, w_t) -> np.ndarray:
    """Lightning-indexer scores of one query token against its prefix [53ai]
    [juhe]: for every key s of ``k_prefix`` ([n, d]),
    I[s] = sum_j w_t[j] * max(0, q_t[j] . k[s]) with q_t [H_I, d], w_t [H_I]."""
    q_t = np.asarray(q_t, dtype=np.float64)
    k_prefix = np.asarray(k_prefix, dtype=np.float64)
    w_t = np.asarray(w_t, dtype=np.float64)
    dots = q_t @ k_prefix.T                     # [H_I, n]  per-head score
    return w_t @ np.maximum(dots, 0.0)          # ReLU, then weighted head sum


def indexer_scores(q, k, w, rows, q_pos, n_cols) -> np.ndarray:
    """Score matrix for the query tokens ``rows`` (indices into q/w) whose
    positions are ``q_pos``: entry [r, s] for s <= q_pos[r], -inf after.
    ``q`` [n_q, H_I, d] and ``k`` [n_keys, d] are real-valued (dequantised)."""
    out = np.full((len(rows), n_cols), -np.inf, dtype=np.float64)
    for r, (row, pos) in enumerate(zip(rows, q_pos)):
        n = min(int(pos) + 1, n_cols)
        out[r, :n] = indexer_row(q[row], k[:n], w[row])
    return out


# -------------------------------------------------------------- step 3: top-k

def topk_row(scores, pos, k) -> np.ndarray:
    """Fine-grained token selection [juhe] [53ai] for one query at position
    ``pos``: among keys 0..pos keep the min(k, pos+1) with the largest score,
    ties to the lower index, -0.0 equal to +0.0, NaN below everything; return
    them in ascending index order padded with -1 to length k."""
    n = int(pos) + 1
    vals = np.asarray(scores, dtype=np.float64)[:n]
    nan = np.isnan(vals)
    vals = np.where(nan, -np.inf, vals) + 0.0   # +0.0 folds -0.0 into +0.0
    index = np.arange(n)
    # lexsort: last key is primary -> (not NaN first, value desc, index asc)
    order = np.lexsort((index, -vals, nan))
    keep = np.sort(order[: min(k, n)])
    out = np.full(k, -1, dtype=np.int32)
    out[: keep.size] = keep
    return out


# ---------------------------------------------------------- step 4: attention

def attend(q_t, keys, values, scale):
    """Softmax attention of all heads of one query token over the given key
    rows (MQA: every head reads the same rows) [53ai] [pb].
    q_t [H, d_qk], keys [n, d_qk], values [n, d_v].
    Returns (out [H, d_v], lse [H], probs [H, n])."""
    q_t = np.asarray(q_t, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    z = scale * (q_t @ keys.T)                  # [H, n] logits
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    out = p @ values
    lse = m[:, 0] + np.log(l[:, 0])
    return out, lse, p


def sparse_mqa_row(q_t, kv, v, idx_t, scale, d_v):
    """Sparse MQA attention for one query: the rows of ``kv`` named by the
    non-negative entries of ``idx_t`` serve as keys (all d_qk columns) and as
    values (the first d_v columns, or the rows of ``v`` when given)."""
    sel = np.asarray(idx_t)
    sel = sel[sel >= 0]
    keys = np.asarray(kv)[sel]
    values = np.asarray(v)[sel] if v is not None else keys[:, :d_v]
    out, lse, _ = attend(q_t, keys, values, scale)
    return out, lse


def sparse_mqa(q, kv, v, idx, rows, scale, d_v):
    """sparse_mqa_row for each query row in ``rows``; idx is [len(rows), k]."""
    H = np.asarray(q).shape[1]
    out = np.zeros((len(rows), H, d_v))
    lse = np.zeros((len(rows), H))
    for r, row in enumerate(rows):
        out[r], lse[r] = sparse_mqa_row(q[row], kv, v, idx[r], scale, d_v)
    return out, lse


# ------------------------------------------------------ step 5: dense causal

def dense_causal_attention(q, k, v, scale):
    """Dense causal attention [pb]: query t reads every key s <= t.
    q [L, H, d_qk], k [L, d_qk], v [L, d_v] -> (out [L, H, d_v], lse [L, H])."""
    L = np.asarray(q).shape[0]
    H = np.asarray(q).shape[1]
    d_v = np.asarray(v).shape[1]
    out = np.zeros((L, H, d_v))
    lse = np.zeros((L, H))
    for t in range(L):
        out[t], lse[t], _ = attend(q[t], k[: t + 1], v[: t + 1], scale)
    return out, lse


# ------------------------------------------- indexer KL training signal

def indexer_kl_row(q_t, keys, scale, scores):
    """Training signal of the lightning indexer for one query token over a key
    set (the selected keys in sparse training; every preceding key in the dense
    warm-up). [amaranth] section "DeepSeek Sparse Attention (DSA)" and [juhe]
    "阶段一：Dense Warm-up" / "阶段二：Sparse Training": the indexer learns to
    match the main attention's distribution through a KL-divergence loss;
    [53ai] "持续预训练：逐步优化稀疏机制" (continued pre-training): in sparse
    training the KL term is kept with only the top-k keys selected.

    The main attention distribution is every head's softmax over the keys,
    averaged over the heads (so it sums to 1); the indexer's is the softmax of
    its scores over the same keys. Returns (p, r, kl, grad): p the target, r
    the indexer distribution, kl = KL(p || r) = sum_i p_i (log p_i - log r_i),
    and grad = d kl / d scores = r - p (p taken as fixed).
    q_t [H, d_qk], keys [n, d_qk], scores [n]."""
    q_t = np.asarray(q_t, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    _, _, probs = attend(q_t, keys, keys[:, :1], scale)     # [H, n] per-head softmax
    p = probs.mean(axis=0)
    s = np.asarray(scores, dtype=np.float64)
    e = np.exp(s - s.max())
    r = e / e.sum()
    pos = p > 0
    kl = float(np.sum(p[pos] * (np.log(p[pos]) - np.log(r[pos]))))
    return p, r, kl, r - p


def indexer_kl_rows(q, kv, idx, rows, scale, sel_scores):
    """indexer_kl_row for each query row in ``rows`` over its selection
    idx[r] (entries < 0 skipped) with the indexer scores of those entries,
    sel_scores[r] (same positions as idx[r]). Returns (p, kl, grad) with p and
    grad laid out like idx (0 at skipped entries)."""
    idx = np.asarray(idx)
    p_out = np.zeros(idx.shape)
    g_out = np.zeros(idx.shape)
    kl = np.zeros(len(rows))
    for r, row in enumerate(rows):
        m = idx[r] >= 0
        keys = np.asarray(kv)[idx[r][m]]
        p, _, kl[r], g = indexer_kl_row(q[row], keys, scale, np.asarray(sel_scores)[r][m])
        p_out[r, m] = p
        g_out[r, m] = g
    return p_out, kl, g_out


# ------------------------------------------- gradient of the sparse attention

def attend_backward(q_t, keys, values, scale, d_out):
    """Gradient of attend() for one query token [amaranth] section "DeepSeek
    Sparse Attention (DSA)", stage B (sparse training: the main model is
    trained through the attention over the selected keys only; the indexer's
    input is detached, so no gradient reaches the selection). With
    z = scale * q K^T, P = softmax_rows(z), O = P V and an upstream gradient
    dO = d loss / d O, the chain rule gives
        dP = dO V^T,  dz = P * (dP - rowsum(dO * O)),
        dq = scale * dz K,  dK = scale * dz^T q,  dV = P^T dO
    (rowsum(dO * O) = sum_i P_i dP_i is the softmax Jacobian's correction).
    q_t [H, d_qk], keys [n, d_qk], values [n, d_v], d_out [H, d_v].
    Returns (dq [H, d_qk], dk [n, d_qk], dv [n, d_v])."""
    q_t = np.asarray(q_t, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    d_out = np.asarray(d_out, dtype=np.float64)
    out, _, p = attend(q_t, keys, values, scale)
    dp = d_out @ values.T                                  # [H, n]
    delta = np.sum(d_out * out, axis=1, keepdims=True)     # [H, 1]
    dz = p * (dp - delta)                                  # d loss / d z
    dq = scale * (dz @ keys)
    dk = scale * (dz.T @ q_t)
    dv = p.T @ d_out
    return dq, dk, dv


def sparse_mqa_backward(q, kv, idx, rows, d_out, scale, d_v):
    """Gradient of sparse_mqa (MQA mode, V = the first d_v columns of the
    selected latent rows) for the query rows ``rows`` with selections idx[r]
    (entries < 0 skipped) and upstream gradients d_out[r] [H, d_v].
    A latent row serves as key and as value, so its gradient is the sum of its
    key gradient and (in its first d_v columns) its value gradient, summed over
    every query that selected it.
    Returns (dq [len(rows), H, d_qk], dkv [n_kv, d_qk])."""
    q = np.asarray(q)
    kv = np.asarray(kv, dtype=np.float64)
    idx = np.asarray(idx)
    H, d_qk = q.shape[1], q.shape[2]
    dq = np.zeros((len(rows), H, d_qk))
    dkv = np.zeros(kv.shape)
    for r, row in enumerate(rows):
        sel = idx[r][idx[r] >= 0]
        if sel.size == 0:
            continue
        keys = kv[sel]
        dq[r], dk, dv = attend_backward(q[row], keys, keys[:, :d_v], scale, d_out[r])
        np.add.at(dkv, sel, dk)
        np.add.at(dkv[:, :d_v], sel, dv)
    return dq, dkv


# ------------------------------------------------------------- paged caches

def paged_rows(cache, block_table_row, ctx_len):
    """Logical rows 0..ctx_len-1 of one sequence stored in 64-token pages:
    logical row p lives in page block_table_row[p // P] at slot p % P."""
    cache = np.asarray(cache)
    P = cache.shape[1]
    n_pages = (int(ctx_len) + P - 1) // P
    pages = np.asarray(block_table_row)[:n_pages]
    return cache[pages].reshape((n_pages * P,) + cache.shape[2:])[: int(ctx_len)]


# ------------------------------------------------------------ whole forward

def forward_prefill_rows(q_idx, k_idx, w, q, kv, v, rows, k, scale, d_v):
    """indexer -> top-k -> sparse attention for the query rows ``rows`` of a
    prefill (query t at position t). Inputs are real-valued (dequantised).
    Returns (scores, idx, out, lse) for those rows."""
    L = np.asarray(k_idx).shape[0]
    scores = indexer_scores(q_idx, k_idx, w, rows, rows, L)
    idx = np.stack([topk_row(scores[r], rows[r], k) for r in range(len(rows))])
    out, lse = sparse_mqa(q, kv, v, idx, rows, scale, d_v)
    return scores, idx, out, lse
