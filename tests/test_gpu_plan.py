"""GPU bsa_rse vs the fp64 RSE oracle, and the plan pipeline on the C2 workload.

bsa_rse sums in fp64 over bf16 inputs; the oracle computes the same sums in
fp64 in another order, so they agree to ~1e-12 relative (tolerance 1e-9).
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import plan as OP
from parity_util import bsa, f64

pytestmark = pytest.mark.gpu


def _rse(dm, ym, yo):
    m = bsa()
    out = torch.empty(4 * dm.H, dtype=torch.float64, device="cuda")
    m.rse(dm, ym, yo, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("shape", [(1, 1, 8, 8), (2, 3, 129, 64), (1, 5, 1000, 128)])
def test_rse_random_matches_oracle(shape):
    m = bsa()
    B, H, N, d = shape
    yo = W.to_bf16(W.normal_f32(shape, 11))
    ym = W.to_bf16(W.normal_f32(shape, 12) * 0.3 + W.normal_f32(shape, 11))
    dm = m.dims(B, H, N, d, 64, 64, 0)
    got = _rse(dm, ym.cuda(), yo.cuda())
    i, num, den = OP.rse(f64(ym), f64(yo))
    np.testing.assert_allclose(got[:H], i, rtol=1e-9)
    np.testing.assert_allclose(got[H:].reshape(H, 3)[:, 0], num, rtol=1e-9)


def test_rse_exact_output_scores_zero():
    m = bsa()
    y = W.to_bf16(W.normal_f32((2, 4, 64, 64), 3)).cuda()
    got = _rse(m.dims(2, 4, 64, 64, 64, 64, 0), y, y)
    assert np.all(got[:4] == 0.0)


def _c2_outputs(w, mode, window=None):
    """C2 forward with every head in one mode (windows for arrow)."""
    m = bsa()
    shp = w["shape"]
    dm = m.dims(shp.B, shp.H, shp.N, shp.d, shp.block_q, shp.block_k, shp.n_text)
    q, k, v = (t.cuda() for t in (w["q"], w["k"], w["v"]))
    modes = torch.full((shp.H,), mode, dtype=torch.int32, device="cuda")
    wins = torch.full((shp.H,), window or 0, dtype=torch.int32, device="cuda")
    blocks = m.BlockList.empty(shp.B, shp.H, shp.n_qb, shp.n_kb, bitmap=False)
    m.build_mask(dm, m.MASK_ARROW, blocks, head_mode=modes, window=wins)
    o = torch.empty_like(q)
    cin = w["cache_f32"].cuda() if mode == m.HEAD_SKIP else None
    m.forward(dm, q, k, v, o, modes, blocks=blocks, cache_in=cin)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    per_head = blocks.cnt.sum(dim=(0, 2)).cpu().numpy().astype(np.int64) // shp.B  # blocks per (b, h)
    return dm, o, per_head


def test_plan_pipeline_on_c2():
    """Candidate methods per head (full, arrow w = 4/2/1, reuse of a drifted
    previous-step output), their RSE against the full output at full size,
    then the plan under the pages' budgets."""
    m = bsa()
    w = W.c2(1)
    shp = w["shape"]
    dm, y_full, _ = _c2_outputs(w, m.HEAD_FULL)
    # a previous step's output: the full output plus a small drift
    yf = y_full.float().cpu()
    w["cache_f32"] = yf + 0.05 * yf.std() * W.normal_f32(tuple(yf.shape), 21)
    cands = [(m.HEAD_FULL, None), (m.HEAD_SPARSE, 4), (m.HEAD_SPARSE, 2), (m.HEAD_SPARSE, 1), (m.HEAD_SKIP, None)]
    rse = np.zeros((shp.H, len(cands)))
    cost = np.zeros((shp.H, len(cands)), dtype=np.int64)
    for j, (mode, win) in enumerate(cands):
        if mode == m.HEAD_FULL:
            y, blocks = y_full, np.full(shp.H, shp.n_qb * shp.n_kb, dtype=np.int64)
        else:
            _, y, blocks = _c2_outputs(w, mode, win)
        got = _rse(dm, y, y_full)
        exp, _, _ = OP.rse(f64(y), f64(y_full))
        np.testing.assert_allclose(got[:shp.H], exp, rtol=1e-9, atol=1e-12)
        rse[:, j] = got[:shp.H]
        cost[:, j] = 0 if mode == m.HEAD_SKIP else blocks
    assert np.all(rse[:, 0] == 0.0)
    assert np.all(np.diff(cost[:, :4], axis=1) <= 0)  # narrower windows compute fewer blocks
    for delta in (0.2, 0.6):
        ch, total = m.plan_heads(rse, cost, delta, 1.5)
        assert OP.feasible(rse, ch, delta, 1.5)
        assert total == int(sum(cost[h, ch[h]] for h in range(shp.H)))
        assert total < int(cost[:, 0].sum())  # the budget buys some sparsity
