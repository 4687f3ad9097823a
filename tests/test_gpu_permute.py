"""GPU tile permutation vs the oracle: bit-exact, padding zeroed, round trip exact."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import masks as OM
from oracle import permute as OP
from parity_util import bsa

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_text,grid,tile,d", [
    (5, (3, 5, 6), (2, 2, 4), 64),
    (256, (16, 48, 80), (4, 8, 8), 128),
    (0, (7, 9), (4, 4), 8),
    (3, (10,), (4,), 16),
])
def test_permute_matches_oracle(n_text, grid, tile, d):
    m = bsa()
    B, H = 1, 2
    n_r = n_text + int(np.prod(grid))
    x = W.to_bf16(W.normal_f32((B, H, n_r, d), 17))
    y = W.to_bf16(W.normal_f32((B, H, n_r, d), 18))
    g = m.GnaGeom.make(grid, tile, tuple(1 for _ in grid), tuple(1 for _ in grid))
    lay = OM.GnaLayout(n_text, grid, tile, tuple(1 for _ in grid), tuple(1 for _ in grid))
    nt = m.gna_tiled_len(n_text, g)
    dm = m.dims(B, H, n_r, d, lay.bs, lay.bs, n_text)
    xt = torch.full((B, H, nt, d), 7.0, dtype=torch.bfloat16, device="cuda")
    yt = torch.full_like(xt, 7.0)
    m.permute_tiles(dm, g, [x.cuda(), y.cuda()], [xt, yt])
    exp = OP.permute_to_tiles(x.view(torch.int16).numpy(), lay)
    np.testing.assert_array_equal(xt.cpu().view(torch.int16).numpy(), exp)
    np.testing.assert_array_equal(yt.cpu().view(torch.int16).numpy(), OP.permute_to_tiles(y.view(torch.int16).numpy(), lay))
    back = torch.zeros_like(x, device="cuda")
    m.unpermute_tiles(dm, g, [xt], [back])
    torch.cuda.synchronize()
    assert torch.equal(back.cpu(), x)
