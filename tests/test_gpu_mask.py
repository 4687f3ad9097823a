"""GPU block-list builder vs the oracle: bit-exact classes and CSR lists."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import masks as OM
from parity_util import bsa, list_to_classes

pytestmark = pytest.mark.gpu


def _arrow_gpu(shape, modes, wins):
    m = bsa()
    blocks = m.BlockList.empty(shape.B, shape.H, shape.n_qb, shape.n_kb)
    dm = m.dims(shape.B, shape.H, shape.N, shape.d, shape.block_q, shape.block_k, shape.n_text)
    m.build_mask(dm, m.MASK_ARROW, blocks, head_mode=torch.from_numpy(modes).cuda(),
                 window=torch.from_numpy(wins).cuda())
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    return blocks


def _check_blocks(blocks, expect):
    got = list_to_classes(blocks, expect.shape[-1])
    np.testing.assert_array_equal(got, expect)
    np.testing.assert_array_equal(blocks.bitmap.cpu().numpy(), expect)


@pytest.mark.parametrize("case", ["c1", "c2"])
def test_arrow_mask_workloads(case):
    w = W.c1() if case == "c1" else W.c2()
    shp = w["shape"]
    blocks = _arrow_gpu(shp, w["head_mode"], w["window"])
    exp = OM.arrow_block_classes_all(shp, w["head_mode"], w["window"])
    _check_blocks(blocks, exp)
    if case == "c1":
        assert int(blocks.cnt.sum()) == 98


@pytest.mark.parametrize("N,n_text,bs", [(64 * 7 + 13, 70, 64), (128 * 5 + 1, 0, 128), (64, 64, 64)])
def test_arrow_mask_ragged(N, n_text, bs):
    rng = np.random.default_rng(N)
    H = 6
    modes = rng.integers(0, 3, H).astype(np.int32)
    wins = rng.integers(0, 4, H).astype(np.int32)
    shp = W.Shape(B=2, H=H, N=N, d=64, block_q=bs, block_k=bs, n_text=n_text)
    blocks = _arrow_gpu(shp, modes, wins)
    _check_blocks(blocks, OM.arrow_block_classes_all(shp, modes, wins))


def _gna_gpu(B, H, lay, grid, tile, window, stride, modes=None):
    m = bsa()
    nB = lay.N // lay.bs
    blocks = m.BlockList.empty(B, H, nB, nB)
    dm = m.dims(B, H, lay.N, 128, lay.bs, lay.bs, lay.n_text)
    g = m.GnaGeom.make(grid, tile, window, stride)
    m.build_mask(dm, m.MASK_GNA, blocks, head_mode=None if modes is None else torch.from_numpy(modes).cuda(),
                 gna=g)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    return blocks


@pytest.mark.parametrize("n_text,grid,tile,window,stride", [
    (0, (10,), (64,), (4,), (2,)),
    (5, (6, 7), (2, 32), (3, 4), (1, 2)),
    (3, (4, 6, 5), (2, 2, 16), (2, 3, 3), (1, 1, 1)),
    (64, (8, 12, 16), (2, 4, 8), (4, 6, 8), (2, 2, 4)),
    (100, (5, 9, 20), (2, 4, 8), (3, 5, 7), (1, 1, 1)),
])
def test_gna_mask_small(n_text, grid, tile, window, stride):
    lay = OM.GnaLayout(n_text, grid, tile, window, stride)
    modes = np.array([1, 0, 2, 1], np.int32)
    blocks = _gna_gpu(2, 4, lay, grid, tile, window, stride, modes)
    _check_blocks(blocks, OM.gna_block_classes_all(2, 4, lay, modes))


@pytest.mark.parametrize("stride", [(4, 8, 8), (1, 1, 1)])
def test_gna_mask_c5(stride):
    w = W.c5(stride=stride)
    g = w["geom"]
    lay = OM.GnaLayout(256, g.grid, g.tile, g.window, g.stride)
    blocks = _gna_gpu(1, 24, lay, g.grid, g.tile, g.window, g.stride)
    exp = OM.gna_block_classes_all(1, 24, lay)
    _check_blocks(blocks, exp)
    img = blocks.bitmap[0, 0, 1:, 1:].cpu().numpy()
    if stride == (4, 8, 8):
        assert int((img == 1).sum()) == 240 * 12 and int((img == 2).sum()) == 0
    else:
        assert int((img == 1).sum()) == 768 and int((img == 2).sum()) == 6272
