"""GPU bsa_jaccard against the schedule oracle (exact: both count integers;
the quotient is one float division on each side)."""
import numpy as np
import pytest
import torch

from oracle import schedule as OSc
from parity_util import bsa

pytestmark = pytest.mark.gpu


def _arrow_list(m, dm, H, nQB, nKB, window):
    modes = torch.full((H,), m.HEAD_SPARSE, dtype=torch.int32, device="cuda")
    wins = torch.full((H,), window, dtype=torch.int32, device="cuda")
    bl = m.BlockList.empty(dm.B, H, nQB, nKB, bitmap=False)
    m.build_mask(dm, m.MASK_ARROW, bl, head_mode=modes, window=wins)
    return bl


def _rows(bl):
    cnt = bl.cnt.cpu().numpy().reshape(-1)
    idx = bl.idx.cpu().numpy().reshape(cnt.size, -1)
    return [idx[r, :cnt[r]].tolist() for r in range(cnt.size)]


@pytest.mark.parametrize("wa,wb", [(1, 2), (4, 1), (2, 2)])
def test_jaccard_of_arrow_windows(wa, wb):
    m = bsa()
    B, H, N, bs, n_text = 2, 3, 4352, 64, 256
    dm = m.dims(B, H, N, 64, bs, bs, n_text)
    nQB = nKB = N // bs
    a = _arrow_list(m, dm, H, nQB, nKB, wa)
    b = _arrow_list(m, dm, H, nQB, nKB, wb)
    out = torch.full((B, H, nQB), float("nan"), dtype=torch.float32, device="cuda")
    m.jaccard(dm, a, b, out)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    exp = OSc.jaccard_rows(_rows(a), _rows(b)).astype(np.float32)
    np.testing.assert_allclose(out.cpu().numpy().reshape(-1), exp, rtol=1e-6)
    if wa == wb:
        assert torch.all(out == 1.0)


def test_jaccard_empty_rows_score_one():
    m = bsa()
    dm = m.dims(1, 1, 256, 64, 64, 64, 0)
    a = m.BlockList.empty(1, 1, 4, 4, bitmap=False)
    a.cnt.zero_()
    out = torch.zeros((1, 1, 4), dtype=torch.float32, device="cuda")
    m.jaccard(dm, a, a, out)
    torch.cuda.synchronize()
    assert torch.all(out == 1.0)
