"""GPU bsa_select_topk vs the oracle: exact selections outside 1e-5-relative near-ties."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import masks as OM
from oracle import select as OS
from parity_util import bsa, check_full_score_rows, f64, list_to_classes, selection_matches

pytestmark = pytest.mark.gpu


def _select(shape, q, k, method, groups, keep_text, scale=1.0, bias=None):
    m = bsa()
    dm = m.dims(shape.B, shape.H, shape.N, shape.d, shape.block_q, shape.block_k, shape.n_text)
    sp = m.select_spec(method, groups, keep_text, scale)
    ws = torch.empty(m.select_workspace_size(dm, sp), dtype=torch.uint8, device="cuda")
    blocks = m.BlockList.empty(shape.B, shape.H, shape.n_qb, shape.n_kb)
    m.select_topk(dm, q.cuda(), k.cuda(), sp, blocks, ws, bias=None if bias is None else bias.cuda())
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    cls = list_to_classes(blocks, shape.n_kb)
    np.testing.assert_array_equal(cls, blocks.bitmap.cpu().numpy())
    return cls


def _check_pooled(shape, q, k, groups, keep_text, cls, max_amb_frac=0.02):
    ntq = -(-shape.n_text // shape.block_q) if keep_text else 0
    ntk = -(-shape.n_text // shape.block_k) if keep_text else 0
    amb = 0
    for b in range(shape.B):
        for h in range(shape.H):
            sc = OS.pooled_scores(f64(q[b, h]), f64(k[b, h]), shape.block_q, shape.block_k)
            for I in range(shape.n_qb):
                row = cls[b, h, I] > 0
                if I < ntq:
                    assert row.all()
                    continue
                fixed = np.zeros(shape.n_kb, bool)
                fixed[:ntk] = True
                assert row[:ntk].all()
                ok, a = selection_matches(row, sc[I], groups, fixed)
                assert ok, (b, h, I)
                amb += a
    assert amb <= max_amb_frac * shape.B * shape.H * shape.n_qb * 4 + 4


@pytest.mark.parametrize("N,bs,d", [(64 * 9 + 21, 64, 64), (128 * 7 + 100, 128, 128)])
def test_pooled_select_ragged(N, bs, d):
    B, H, n_text = 2, 3, bs + 10
    q, k, _ = W.qkv_normal(B, H, N, d, N)
    shape = W.Shape(B, H, N, d, bs, bs, n_text)
    nb = -(-N // bs)
    groups = [(2, nb, 3)]
    cls = _select(shape, q, k, bsa().SELECT_POOLED_QK, groups, True)
    _check_pooled(shape, q, k, groups, True, cls)


def test_pooled_select_exact_ties_lowest_index():
    bs, nb, d = 64, 10, 64
    N = bs * nb
    q = torch.ones(1, 1, N, d)
    kblk = torch.tensor([3, 1, 3, 2, 3, 1, 2, 3, 0, 3], dtype=torch.float32)
    k = kblk.repeat_interleave(bs)[None, None, :, None].expand(1, 1, N, d).contiguous()
    shape = W.Shape(1, 1, N, d, bs, bs, 0)
    cls = _select(shape, q.to(torch.bfloat16), k.to(torch.bfloat16), bsa().SELECT_POOLED_QK, [(0, nb, 3)], False)
    for I in range(nb):
        assert list(np.nonzero(cls[0, 0, I])[0]) == [0, 2, 4]


def test_pooled_select_c3_all_rows():
    w = W.c3()
    cls = _select(w["shape"], w["q"], w["k"], bsa().SELECT_POOLED_QK, w["groups"], True)
    _check_pooled(w["shape"], w["q"], w["k"], w["groups"], True, cls)
    kept = int((cls[0] > 0).sum())
    assert kept == 24 * (128 * (39 + 4) + 4 * 132)


def _check_full(shape, q, k, groups, bias, cls, rows_per_head=None, seed=0):
    rng = np.random.default_rng(seed)
    scale = shape.d ** -0.5
    for b in range(shape.B):
        for h in range(shape.H):
            Is = range(shape.n_qb) if rows_per_head is None else \
                np.sort(rng.choice(shape.n_qb, rows_per_head, replace=False))
            _, ap = OS.full_score_select(f64(q[b, h]), f64(k[b, h]), scale, shape.block_q, shape.block_k,
                                         groups, bias=None if bias is None else bias[h].numpy(), rows=Is)
            for r, I in enumerate(Is):
                ok, _ = selection_matches(cls[b, h, I] > 0, ap[r], groups, np.zeros(shape.n_kb, bool))
                assert ok, (b, h, I)


@pytest.mark.parametrize("N", [128 * 8, 128 * 9 + 50])
def test_full_score_select_small(N):
    B, H, d, bs = 1, 3, 128, 128
    q, k, _ = W.qkv_normal(B, H, N, d, N + 1)
    shape = W.Shape(B, H, N, d, bs, bs, 0)
    nb = -(-N // bs)
    groups = [(0, nb - 2, 3), (nb - 2, nb, 1)]
    bias, _ = W.dlm_bias(H, nb, nb - 2, seed=5, n_col_pre=2, n_col_gen=1, windows=(1, 2))
    cls = _select(shape, q, k, bsa().SELECT_FULL_SCORE, groups, False, d ** -0.5, bias)
    _check_full(shape, q, k, groups, bias, cls)


@pytest.mark.parametrize("N,bs,d", [(256 * 5 + 70, 256, 64), (384 * 3 + 200, 384, 128)])
def test_full_score_select_multi_tile_blocks(N, bs, d):
    """Blocks of two and three 128-token tiles: a query block's rows span several score CTAs, a
    key block several per-tile LSEs; ragged last blocks; every row against the oracle."""
    B, H = 1, 2
    q, k, _ = W.qkv_normal(B, H, N, d, N + 7)
    shape = W.Shape(B, H, N, d, bs, bs, 0)
    nb = -(-N // bs)
    groups = [(0, nb - 1, 2), (nb - 1, nb, 1)]
    bias, _ = W.dlm_bias(H, nb, nb - 1, seed=9, n_col_pre=1, n_col_gen=1, windows=(1,))
    cls = _select(shape, q, k, bsa().SELECT_FULL_SCORE, groups, False, d ** -0.5, bias)
    _check_full(shape, q, k, groups, bias, cls)


def test_full_score_select_zero_q_takes_lowest_indices():
    B, H, N, d, bs = 1, 1, 128 * 6, 128, 128
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
    _, k, _ = W.qkv_normal(B, H, N, d, 3)
    shape = W.Shape(B, H, N, d, bs, bs, 0)
    cls = _select(shape, q, k, bsa().SELECT_FULL_SCORE, [(0, 4, 2), (4, 6, 1)], False, d ** -0.5)
    for I in range(6):
        assert list(np.nonzero(cls[0, 0, I])[0]) == [0, 1, 4]


def c4_rows_plan(kinds, n_qb, n_full_heads=4, rows_per_head=16, seed=0):
    """Which query-block rows of each head the 32k check compares: every row of two 'column' and
    two 'slide-window' heads (or the first heads if one kind is missing), and a seeded 16 rows of
    every other head that always include the first row and the last one (a generation row)."""
    col = [h for h, kd in enumerate(kinds) if kd[0] == "column"]
    win = [h for h, kd in enumerate(kinds) if kd[0] != "column"]
    full = (col[:n_full_heads // 2] + win[:n_full_heads // 2])
    full += [h for h in range(len(kinds)) if h not in full][:n_full_heads - len(full)]
    rng = np.random.default_rng(seed)
    plan = {}
    for h in range(len(kinds)):
        if h in full:
            plan[h] = np.arange(n_qb)
        else:
            extra = rng.choice(np.arange(1, n_qb - 1), rows_per_head - 2, replace=False)
            plan[h] = np.unique(np.concatenate([[0, n_qb - 1], extra]))
    return plan


@pytest.mark.slow
def test_full_score_select_c4_rows():
    """SparseD-like 32k selection: every query-block row of four heads (both bias kinds) and 16
    rows of each of the other 28 heads against the oracle's A' (isolated prefill / generation
    top-rho%, ties within 1e-5 relative excluded)."""
    w = W.c4()
    shp = w["shape"]
    q, k, _ = W.dlm_step_qkv(shp, 3, 0)
    cls = _select(shp, q, k, bsa().SELECT_FULL_SCORE, w["groups"], False, shp.d ** -0.5, w["bias"])
    assert (cls[0] > 0).sum(axis=-1).min() == 77 and (cls[0] > 0).sum(axis=-1).max() == 77
    plan = c4_rows_plan(w["bias_kinds"], shp.n_qb)
    assert sum(len(r) == shp.n_qb for r in plan.values()) == 4
    assert all(len(r) >= 16 for r in plan.values())
    for h, rows in plan.items():
        check_full_score_rows(cls[0, h], f64(q[0, h]), f64(k[0, h]), shp.d ** -0.5, shp.block_q, shp.block_k,
                              w["groups"], rows, bias=w["bias"][h].numpy())
