"""Pins for oracle.masks: closed-form counts, brute-force windows, special cases."""
import itertools

import numpy as np
import pytest

from oracle import masks as M


# --------------------------------------------------------------------------- arrow

def _arrow_count_closed_form(nb, ntb, w):
    """Kept blocks of one arrow head: text rows + text columns of image rows +
    image-image blocks within the band |I-J| <= w (counted by band length)."""
    n_img = nb - ntb
    band = n_img + 2 * sum(max(n_img - t, 0) for t in range(1, w + 1))
    return ntb * nb + n_img * ntb + band


@pytest.mark.parametrize("w", [0, 1, 2, 4, 7])
def test_arrow_counts_closed_form(w):
    c = M.arrow_block_classes(4352, 256, 64, M.HEAD_SPARSE, w)
    assert int((c > 0).sum()) == _arrow_count_closed_form(68, 4, w)
    assert not (c == M.BLOCK_PARTIAL).any()


def test_arrow_c2_counts():
    counts = {w: int((M.arrow_block_classes(4352, 256, 64, M.HEAD_SPARSE, w) > 0).sum())
              for w in (1, 2, 4)}
    assert counts == {1: 718, 2: 842, 4: 1084}


def test_arrow_c1_total():
    full = M.arrow_block_classes(512, 64, 64, M.HEAD_FULL, 0)
    arrow = M.arrow_block_classes(512, 64, 64, M.HEAD_SPARSE, 1)
    assert int((full > 0).sum()) + int((arrow > 0).sum()) == 98


def test_arrow_wide_window_is_full_and_skip_is_empty():
    c = M.arrow_block_classes(640, 100, 64, M.HEAD_SPARSE, 9)
    assert (c == M.BLOCK_FULL).all()
    assert (M.arrow_block_classes(640, 100, 64, M.HEAD_SKIP, 3) == 0).all()


def test_arrow_partial_text_block_is_text():
    # n_text = 70 with block 64: block 1 holds text tokens 64..69, so it is a text block
    c = M.arrow_block_classes(64 * 8, 70, 64, M.HEAD_SPARSE, 0)
    assert (c[:2] == M.BLOCK_FULL).all() and (c[:, :2] == M.BLOCK_FULL).all()
    assert c[5, 3] == 0 and c[5, 5] == M.BLOCK_FULL


# --------------------------------------------------------------------------- GNA windows

def _na_window_bruteforce(i, L, k):
    """Clamped neighborhood attention: among all length-k windows inside [0, L)
    that contain i, the one whose left part is closest to floor((k-1)/2) keys."""
    best = None
    for a in range(0, L - k + 1):
        if a <= i < a + k:
            key = abs((i - a) - (k - 1) // 2)
            if best is None or key < best[0]:
                best = (key, a)
    return best[1]


@pytest.mark.parametrize("L,k", [(10, 3), (10, 4), (7, 7), (13, 1), (16, 8), (80, 24)])
def test_stride_one_is_neighborhood_attention(L, k):
    for i in range(L):
        assert int(M.window_start(i, L, k, 1)) == _na_window_bruteforce(i, L, k)


@pytest.mark.parametrize("L,k,s", [(10, 4, 2), (12, 6, 3), (16, 8, 4), (48, 16, 8), (80, 24, 8),
                                   (9, 5, 5), (11, 4, 3)])
def test_stride_group_shares_window_and_contains_query(L, k, s):
    st = M.window_start(np.arange(L), L, k, s)
    for i in range(L):
        assert st[i] <= i < st[i] + k
        assert 0 <= st[i] <= L - k
        assert st[i] == st[s * (i // s)]


def test_translation_equivariance_away_from_border():
    L, k, s = 40, 9, 3
    st = M.window_start(np.arange(L), L, k, s)
    inner = [i for i in range(9, 30)]
    for i in inner:
        if i + s < 31:
            assert st[i + s] == st[i] + s


def _layouts():
    yield M.GnaLayout(0, (10,), (2,), (4,), (2,))
    yield M.GnaLayout(0, (10,), (4,), (3,), (1,))
    yield M.GnaLayout(4, (6, 7), (2, 4), (3, 4), (1, 2))
    yield M.GnaLayout(3, (4, 6, 5), (2, 2, 4), (2, 3, 3), (1, 1, 1))
    yield M.GnaLayout(8, (4, 6, 8), (2, 2, 2), (2, 4, 4), (2, 2, 2))
    yield M.GnaLayout(20, (4, 6), (2, 4), (3, 3), (1, 1))   # three text blocks, the last padded
    yield M.GnaLayout(16, (3, 5), (2, 4), (3, 2), (1, 2))   # text ends on a block edge


@pytest.mark.parametrize("lay", list(_layouts()))
def test_separable_classes_match_token_enumeration(lay):
    tm = M.gna_token_mask(lay)
    valid = lay.valid(np.arange(lay.N))
    enum = M.classify_blocks(tm, lay.bs, lay.bs, valid, valid)
    sep = M.gna_block_classes_separable(lay)
    np.testing.assert_array_equal(enum, sep)


def test_token_mask_matches_per_pair_brute_force():
    lay = M.GnaLayout(2, (4, 5), (2, 2), (3, 2), (1, 1))
    tm = M.gna_token_mask(lay)
    for i in range(lay.N):
        ki, ci = lay.coords(np.array([i]))
        for j in range(lay.N):
            kj, cj = lay.coords(np.array([j]))
            if ki[0] == 1 or kj[0] == 1:
                exp = False
            elif ki[0] == 0 or kj[0] == 0:
                exp = True
            else:
                exp = True
                for dim in range(3):
                    L, k = lay.grid[dim], lay.window[dim]
                    a = _na_window_bruteforce(int(ci[0, dim]), L, k)
                    exp &= a <= cj[0, dim] < a + k
            assert tm[i, j] == exp, (i, j)


def test_window_equal_grid_is_full():
    lay = M.GnaLayout(0, (4, 8), (2, 4), (4, 8), (1, 1))
    assert (M.gna_block_classes_separable(lay) == M.BLOCK_FULL).all()


def test_stride_equals_window_equals_tile_is_block_diagonal():
    lay = M.GnaLayout(16, (8, 8), (4, 4), (4, 4), (4, 4))
    c = M.gna_block_classes_separable(lay)
    nb = c.shape[0]
    for I in range(nb):
        for J in range(nb):
            if I == 0 or J == 0 or I == J:
                assert c[I, J] == M.BLOCK_FULL
            else:
                assert c[I, J] == M.BLOCK_NONE


def _one_dim_tile_classes(L, T, k, s):
    """1-D tile-pair classes by brute force over (query, key) positions."""
    nt = -(-L // T)
    out = np.zeros((nt, nt), int)
    for a in range(nt):
        for b in range(nt):
            qs = range(a * T, min(a * T + T, L))
            ks = range(b * T, min(b * T + T, L))
            ok = [_na_window_bruteforce(i, L, k) if s == 1 else None for i in qs]
            hits = 0
            for idx, i in enumerate(qs):
                st = ok[idx] if s == 1 else int(M.window_start(i, L, k, s))
                hits += sum(st <= j < st + k for j in ks)
            tot = len(qs) * len(ks)
            out[a, b] = 0 if hits == 0 else (1 if hits == tot else 2)
    return out


@pytest.mark.parametrize("stride", [(4, 8, 8), (1, 1, 1)])
def test_c5_tile_counts_from_one_dim_products(stride):
    grid, tile, win = (16, 48, 80), (4, 8, 8), (8, 16, 24)
    per = [_one_dim_tile_classes(grid[i], tile[i], win[i], stride[i]) for i in range(3)]
    full = int(np.prod([(p == 1).sum() for p in per]))
    touched = int(np.prod([(p > 0).sum() for p in per]))
    lay = M.GnaLayout(256, grid, tile, win, stride)
    c = M.gna_block_classes_separable(lay)[1:, 1:]
    assert int((c == M.BLOCK_FULL).sum()) == full
    assert int((c == M.BLOCK_PARTIAL).sum()) == touched - full
    if stride == (4, 8, 8):
        assert full == 240 * 12 and touched == full
        assert all(int((c[I] > 0).sum()) == 12 for I in range(240))
    else:
        assert (full, touched - full) == (768, 6272)


def test_gna_full_and_skip_heads():
    lay = M.GnaLayout(5, (6, 4), (2, 4), (3, 4), (1, 1))
    c = M.gna_block_classes_all(1, 3, lay, head_mode=[M.HEAD_FULL, M.HEAD_SPARSE, M.HEAD_SKIP])
    assert (c[0, 2] == 0).all()
    # text block holds 5 text tokens + 3 padding slots -> partial column for full heads
    assert (c[0, 0, :, 0] == M.BLOCK_PARTIAL).all() and (c[0, 0, :, 1:] == M.BLOCK_FULL).all()


def test_csr_roundtrip():
    rng = np.random.default_rng(3)
    cls = rng.integers(0, 3, (7, 11)).astype(np.uint8)
    cnt, idx, flag = M.to_csr(cls)
    back = np.zeros_like(cls)
    for I in range(7):
        assert list(idx[I, :cnt[I]]) == sorted(idx[I, :cnt[I]])
        assert (idx[I, cnt[I]:] == -1).all() and (flag[I, cnt[I]:] == 0).all()
        back[I, idx[I, :cnt[I]]] = flag[I, :cnt[I]]
    np.testing.assert_array_equal(back, cls)
