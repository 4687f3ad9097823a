"""Pins for oracle.permute: hand-listed tile orders, padding, round trips."""
import numpy as np

from oracle import masks as M
from oracle import permute as P


def test_2d_tile_order_hand_listed():
    # 4x4 grid, 2x2 tiles, 1 text token; raster video index r sits at position 1 + r
    lay = M.GnaLayout(1, (4, 4), (2, 2), (2, 2), (1, 1))
    src = P.tile_order_source(lay)
    # block size 4: text block = [text, pad, pad, pad]; then tiles (0,0),(0,1),(1,0),(1,1)
    expect = [0, -1, -1, -1,
              1 + 0, 1 + 1, 1 + 4, 1 + 5,
              1 + 2, 1 + 3, 1 + 6, 1 + 7,
              1 + 8, 1 + 9, 1 + 12, 1 + 13,
              1 + 10, 1 + 11, 1 + 14, 1 + 15]
    assert src.tolist() == expect


def test_padding_slots_in_ragged_grid():
    # 3x3 grid with 2x2 tiles: tiles grid 2x2, 7 padded slots
    lay = M.GnaLayout(0, (3, 3), (2, 2), (2, 2), (1, 1))
    src = P.tile_order_source(lay)
    expect = [0, 1, 3, 4,
              2, -1, 5, -1,
              6, 7, -1, -1,
              8, -1, -1, -1]
    assert src.tolist() == expect


def test_roundtrip_3d():
    lay = M.GnaLayout(5, (3, 5, 6), (2, 2, 4), (2, 3, 3), (1, 1, 1))
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, 3, 5 + 3 * 5 * 6, 4))
    y = P.permute_to_tiles(x, lay)
    assert y.shape[-2] == lay.N
    valid = lay.valid(np.arange(lay.N))
    assert np.all(y[..., ~valid, :] == 0)
    np.testing.assert_array_equal(P.unpermute_from_tiles(y, lay), x)


def test_c5_layout_has_no_padding():
    lay = M.GnaLayout(256, (16, 48, 80), (4, 8, 8), (8, 16, 24), (1, 1, 1))
    assert lay.N == 256 + 16 * 48 * 80 and lay.n_tiles == 240
    assert lay.valid(np.arange(lay.N)).all()
