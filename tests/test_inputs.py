"""The seeded input generators that feed both the GPU path and the oracle
(CPU): shapes, dtypes, seeding, and the validity of the synthetic selections
that the attention tests use in place of the indexer's."""
import numpy as np
import torch

from sparse_attention_long_tcgen05_b200.inputs import make_grad_out, random_selection, sample_rows


def test_random_selection_is_a_valid_topk_output():
    """Every row: min(k, p+1) distinct keys of 0..p in ascending order, then
    -1 padding -- the format of the top-k's output -- for prefix and suffix
    query positions, k below and above the prefix lengths."""
    for n_q, n_keys, k in [(50, 50, 64), (300, 1000, 128), (64, 5000, 2048), (7, 7, 1)]:
        idx = random_selection(n_q, n_keys, k, seed=11).numpy()
        assert idx.shape == (n_q, k) and idx.dtype == np.int32
        for i in range(n_q):
            p = n_keys - n_q + i
            m = min(k, p + 1)
            row = idx[i]
            assert np.all(row[m:] == -1), (n_q, n_keys, k, i)
            sel = row[:m]
            assert sel.min() >= 0 and sel.max() <= p
            assert np.all(np.diff(sel) > 0)
            if p + 1 <= k:
                assert np.array_equal(sel, np.arange(p + 1))


def test_random_selection_spreads_over_the_prefix():
    """One key per stratum: for a long prefix the selection reaches both ends
    and no two keys share a stratum of width (p+1)/k."""
    n_keys, k = 40000, 2048
    idx = random_selection(1, n_keys, k, seed=3).numpy()[0]
    w = n_keys / k
    bounds = np.floor(np.arange(k) * w)              # stratum j: [floor(j w), floor((j+1) w))
    strata = np.searchsorted(bounds, idx, side="right") - 1
    assert np.array_equal(strata, np.arange(k))
    assert idx[0] < w and idx[-1] >= n_keys - w


def test_generators_are_seeded():
    a = random_selection(100, 300, 64, seed=5)
    b = random_selection(100, 300, 64, seed=5)
    c = random_selection(100, 300, 64, seed=6)
    assert torch.equal(a, b) and not torch.equal(a, c)
    g1 = make_grad_out(3, H=4, d_v=8, seed=9)
    g2 = make_grad_out(3, H=4, d_v=8, seed=9)
    assert g1.dtype == torch.bfloat16 and g1.shape == (3, 4, 8) and torch.equal(g1, g2)
    rows = sample_rows(131072, 512, seed=1)
    assert len(rows) == 512 and rows == sorted(set(rows))
    assert {0, 2047, 2048, 131071} <= set(rows)
