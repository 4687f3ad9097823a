"""Workload shapes against the pages' printed token counts (tests/golden/token_counts.json)."""
import json
import os

import workloads as W

HERE = os.path.dirname(__file__)


def _rows():
    with open(os.path.join(HERE, "golden", "token_counts.json")) as f:
        return {r["model"]: r for r in json.load(f)["rows"]}


def test_token_formula_reproduces_printed_table():
    for r in _rows().values():
        t, h, w = r["latent"]
        pt, p = r["patch"]
        n = (t // pt) * (h // p) * (w // p)
        assert n == r["image_tokens"]
        assert n + r["text_tokens"] == r["sequence"]


def test_flux_2048_shape_is_the_printed_sequence():
    r = _rows()["FLUX.1 2048^2"]
    # the content-driven workload uses FLUX.1 2048^2's 128x128 token grid and 512 text tokens
    N = 512 + 128 * 128
    assert N == r["sequence"] == 16896


def test_sd3_image_token_grid():
    r = _rows()["SD3-medium 1024^2"]
    assert 64 * 64 == r["image_tokens"]


def test_mode_table_largest_remainder():
    modes, win = W.draw_mode_table(24, 1)
    assert sorted(modes.tolist()).count(W.HEAD_FULL) == 10
    assert sorted(modes.tolist()).count(W.HEAD_SPARSE) == 11
    assert sorted(modes.tolist()).count(W.HEAD_SKIP) == 3
    assert set(win[modes == W.HEAD_SPARSE].tolist()) <= {1, 2, 4}
    assert (win[modes != W.HEAD_SPARSE] == 0).all()


def test_topk_counts_are_ceil_of_rho():
    assert (30 * 128 + 99) // 100 == 39
    assert (30 * 240 + 99) // 100 == 72
    assert (30 * 16 + 99) // 100 == 5
