"""Helpers shared by the GPU parity tests: run the library through its C ABI,
run the oracle on the same inputs (copied to the host), compare.

Tolerances (written here once, used by every parity test):
  indexer   |g - o| <= 1e-2 * max(|o|, 1e-2 * max_s |o[t, s]|)   (relative 1e-2,
            with a floor at 1% of the row's largest magnitude because mixed-sign
            head weights make scores cross zero)
  top-k     bit-exact, given the same float32 score array
  attention max |g - o| <= 2e-2 on bf16 outputs (oracle's indices); also
            relative RMS <= 1e-2 and |lse_g - lse_o| <= 2e-3
  fp32 tiny path: attention max-abs <= 1e-4 (relative RMS <= 1e-5, lse 1e-4);
            indexer relative 1e-4 with a floor at 1e-3 of the row's largest
            magnitude (fp32 sums against the float64 oracle)
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import dsa_oracle as O
from sparse_attention_long_tcgen05_b200 import dsa

IDX_REL = 1e-2
IDX_FLOOR = 1e-2
ATTN_MAX_ABS = 2e-2
ATTN_REL_RMS = 1e-2
LSE_ABS = 2e-3


def assert_indexer_close(g, o, rel=IDX_REL, floor=IDX_FLOOR):
    """g, o: [rows, cols] float arrays; -inf must match exactly."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    assert g.shape == o.shape
    assert np.array_equal(np.isneginf(g), np.isneginf(o)), "causal mask differs"
    fin = np.isfinite(o)
    assert np.all(np.isfinite(g[fin]))
    rowmax = np.max(np.where(fin, np.abs(o), 0.0), axis=1, keepdims=True)
    bound = rel * np.maximum(np.abs(o), floor * rowmax)
    err = np.abs(np.where(fin, g, 0.0) - np.where(fin, o, 0.0))
    bad = fin & (err > bound)
    assert not bad.any(), (f"{bad.sum()} indexer entries out of tolerance; worst "
                           f"{np.max(np.where(fin, err / np.maximum(bound, 1e-30), 0)):.3g}x bound")


def assert_attention_close(g_out, g_lse, o_out, o_lse, max_abs=ATTN_MAX_ABS,
                           rel_rms=ATTN_REL_RMS, lse_abs=LSE_ABS):
    g_out = np.asarray(g_out, dtype=np.float64)
    o_out = np.asarray(o_out, dtype=np.float64)
    err = np.abs(g_out - o_out)
    assert err.max() <= max_abs, f"attention max-abs {err.max():.3g}"
    rr = np.linalg.norm(g_out - o_out) / max(np.linalg.norm(o_out), 1e-30)
    assert rr <= rel_rms, f"attention relative RMS {rr:.3g}"
    if g_lse is not None:
        le = np.abs(np.asarray(g_lse, np.float64) - np.asarray(o_lse, np.float64))
        assert le.max() <= lse_abs, f"lse max-abs {le.max():.3g}"
    return float(err.max()), float(rr)


def topk_oracle_on(scores_rows: np.ndarray, pos: np.ndarray, k: int) -> np.ndarray:
    return np.stack([O.topk_row(scores_rows[r], int(pos[r]), k) for r in range(len(pos))])


# --------------------------------------------------------------------- prefill

def prefill_structs(inp, n_keys=None, q_offset_rows=None):
    """IndexerIn / AttnIn for a prefill PrefillInputs on the GPU."""
    wl = inp.wl
    ind = dsa.indexer_in(inp.q_idx, inp.k_idx, inp.w, inp.q_scale, inp.k_scale)
    att = dsa.attn_in(inp.q, inp.kv, wl.scale, wl.D_V, v=inp.v)
    return ind, att


def oracle_prefill_inputs(inp, rows):
    """Host float64 copies of what the oracle needs for the given query rows."""
    rows_t = torch.as_tensor(rows, dtype=torch.long, device=inp.q_idx.device)
    if inp.q_scale is not None:
        q_idx = O.dequantize(inp.q_idx[rows_t].cpu().numpy(), inp.q_scale[rows_t].cpu().numpy())
        k_idx = O.dequantize(inp.k_idx.cpu().numpy(), inp.k_scale.cpu().numpy())
    else:
        q_idx = inp.q_idx[rows_t].double().cpu().numpy()
        k_idx = inp.k_idx.double().cpu().numpy()
    w = inp.w[rows_t].double().cpu().numpy()
    q = inp.q[rows_t].double().cpu().numpy()
    return q_idx, k_idx, w, q


def oracle_key_side(inp):
    """Host float64 key side of the indexer (dequantised for FP8 inputs)."""
    if inp.q_scale is not None:
        return O.dequantize(inp.k_idx.cpu().numpy(), inp.k_scale.cpu().numpy())
    return inp.k_idx.double().cpu().numpy()


def oracle_query_side(inp, rows):
    """Host float64 copies of the indexer query side, w and q for these rows."""
    rows_t = torch.as_tensor(rows, dtype=torch.long, device=inp.q_idx.device)
    if inp.q_scale is not None:
        q_idx = O.dequantize(inp.q_idx[rows_t].cpu().numpy(), inp.q_scale[rows_t].cpu().numpy())
    else:
        q_idx = inp.q_idx[rows_t].double().cpu().numpy()
    return q_idx, inp.w[rows_t].double().cpu().numpy(), inp.q[rows_t].double().cpu().numpy()


def oracle_scores(q_idx_rows, k_idx, w_rows, pos, n_cols):
    local = list(range(len(pos)))
    return O.indexer_scores(q_idx_rows, k_idx, w_rows, local, list(pos), n_cols)


def oracle_attention(q_rows, kv_host, v_host, idx_rows, scale, d_v):
    return O.sparse_mqa(q_rows, kv_host, v_host, idx_rows, list(range(len(idx_rows))), scale,
                        d_v)


def gather_kv_rows(kv: torch.Tensor, idx_rows: np.ndarray):
    """Host float64 copy of only the KV rows the given selections name, and the
    selections re-indexed into it (keeps the copy small at 128K)."""
    uniq = np.unique(idx_rows[idx_rows >= 0])
    remap = np.full(int(uniq.max()) + 2 if uniq.size else 1, -1, dtype=np.int64)
    remap[uniq] = np.arange(uniq.size)
    sub = kv[torch.as_tensor(uniq, device=kv.device, dtype=torch.long)].double().cpu().numpy()
    idx_local = np.where(idx_rows >= 0, remap[np.maximum(idx_rows, 0)], -1)
    return sub, idx_local
