"""Pins for oracle.select: brute-force ranking, exact ties, closed forms, library pooling."""
import numpy as np
import pytest
import torch

from oracle import select as S
from oracle import masks as M


def test_top_k_matches_lexsort_and_rank_definition():
    rng = np.random.default_rng(0)
    for trial in range(50):
        n = int(rng.integers(1, 60))
        sc = np.round(rng.standard_normal(n) * 3, 1)  # rounding creates ties
        k = int(rng.integers(0, n + 1))
        got = S.top_k_indices(sc, range(n), k)
        order = np.lexsort((np.arange(n), -sc))  # library: primary -score, then index
        assert got == sorted(order[:k].tolist())
        # rank definition: j kept iff fewer than k candidates beat it
        beats = [sum((sc[i] > sc[j]) or (sc[i] == sc[j] and i < j) for i in range(n)) for j in range(n)]
        assert got == [j for j in range(n) if beats[j] < k]


def test_block_means_ragged_tail():
    x = np.arange(10, dtype=float)[:, None] * np.ones((1, 3))
    m = S.block_means(x, 4)
    np.testing.assert_array_equal(m[:, 0], [1.5, 5.5, 8.5])


def test_exact_ties_go_to_lower_index():
    # integer-valued Q/K constant per block: block means and scores are exact
    bs, nb, d = 4, 10, 2
    q = np.ones((bs * nb, d))
    kblk = np.array([3, 1, 3, 2, 3, 1, 2, 3, 0, 3], float)
    k = np.repeat(kblk, bs)[:, None] * np.ones((1, d))
    cls, sc = S.pooled_select(q, k, bs, bs, 0, [(0, nb, 3)], keep_text=False)
    for I in range(nb):
        assert list(np.nonzero(cls[I])[0]) == [0, 2, 4]  # the five 3s tie; lowest three kept


def test_pooled_select_structure():
    rng = np.random.default_rng(1)
    bs, n_text, N, d = 8, 12, 8 * 9 + 5, 4
    q, k = rng.standard_normal((2, N, d))
    ntb = 2
    nb = -(-N // bs)
    cls, _ = S.pooled_select(q, k, bs, bs, n_text, [(ntb, nb, 3)], keep_text=True)
    assert (cls[:ntb] == M.BLOCK_FULL).all()
    assert (cls[:, :ntb] == M.BLOCK_FULL).all()
    assert all(int((cls[I, ntb:] > 0).sum()) == 3 for I in range(ntb, nb))


def test_avgpool_rows_match_library_pooling_and_sum_to_inverse_block():
    rng = np.random.default_rng(2)
    N, d, bs = 64, 8, 16
    q, k = rng.standard_normal((2, N, d))
    bias = rng.standard_normal((N // bs, N // bs))
    scale = 0.4
    tq, tk = torch.from_numpy(q), torch.from_numpy(k)
    z = scale * tq @ tk.T + torch.from_numpy(np.repeat(np.repeat(bias, bs, 0), bs, 1))
    a = torch.softmax(z, dim=-1)
    pooled = torch.nn.functional.avg_pool2d(a[None, None], bs)[0, 0].numpy()
    for I in range(N // bs):
        row = S.avgpool_attention_rows(q, k, scale, bs, bs, I, bias)
        np.testing.assert_allclose(row, pooled[I], rtol=1e-12, atol=1e-15)
        assert abs(row.sum() - 1.0 / bs) < 1e-14


def test_zero_q_gives_uniform_scores_and_lowest_indices():
    rng = np.random.default_rng(3)
    N, d, bs = 128, 8, 16
    q = np.zeros((N, d))
    k = rng.standard_normal((N, d))
    cls, ap = S.full_score_select(q, k, 0.5, bs, bs, [(0, 6, 2), (6, 8, 1)])
    np.testing.assert_allclose(ap, 1.0 / N, rtol=1e-13)
    for I in range(N // bs):
        assert list(np.nonzero(cls[I])[0]) == [0, 1, 6]


def test_isolated_groups_are_cut_separately():
    # generation blocks with tiny scores still get their own quota
    sc = np.array([[5.0, 4.0, 3.0, 2.0, 0.1, 0.2]])
    cls = S.select_rows(sc, 6, [(0, 4, 2), (4, 6, 1)])
    assert list(np.nonzero(cls[0])[0]) == [0, 1, 5]
    merged = S.select_rows(sc, 6, [(0, 6, 3)])
    assert list(np.nonzero(merged[0])[0]) == [0, 1, 2]
