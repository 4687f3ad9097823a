"""Full-size and capacity cases of the GPU forward against the fp64 oracle, on sampled rows.

They run after the quicker parity files: the SparseD-like 32k workload in the bench's launch
(selection on step 0, the forward of step 1 with the block bias) and the forward at the most
tokens a CTA's key schedule holds.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from parity_util import assert_close_out, bsa, check_full_score_rows, f64
from test_gpu_forward import _check_arrow, _dims, _run_arrow

pytestmark = pytest.mark.gpu


@pytest.mark.slow
def test_forward_c4_sampled_rows_with_gpu_selection():
    """SparseD-like DLM at 32k: the GPU full-score selection on step 0's Q/K, then the GPU forward
    of step 1 reusing it with the block bias (the bench's launch); oracle on 16 sampled rows of
    every head, each of whose selection rows is first checked against the oracle's A'."""
    m = bsa()
    w = W.c4()
    shp = w["shape"]
    dm = _dims(shp)
    bias = w["bias"]
    q0, k0, _ = W.dlm_step_qkv(shp, 3, 0)
    q1, k1, v1 = W.dlm_step_qkv(shp, 3, 1)
    sp = m.select_spec(m.SELECT_FULL_SCORE, w["groups"], False, shp.d ** -0.5)
    ws = torch.empty(m.select_workspace_size(dm, sp), dtype=torch.uint8, device="cuda")
    blocks = m.BlockList.empty(1, shp.H, shp.n_qb, shp.n_kb)
    bias_d = bias.cuda()
    m.select_topk(dm, q0.cuda(), k0.cuda(), sp, blocks, ws, bias=bias_d)
    q, k, v = (t.cuda() for t in (q1, k1, v1))
    o = torch.empty_like(q)
    m.forward(dm, q, k, v, o, torch.ones(shp.H, dtype=torch.int32, device="cuda"), blocks=blocks, bias=bias_d)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    bm = blocks.bitmap.cpu().numpy()
    bias_np = bias.numpy()
    rng = np.random.default_rng(1)
    for h in range(shp.H):
        rows = np.unique(np.concatenate([[0, shp.N - 1], rng.choice(shp.N, 14, replace=False)]))
        # the GPU selection rows these query rows use must first agree with the oracle's A' of step 0
        check_full_score_rows(bm[0, h], f64(q0[0, h]), f64(k0[0, h]), shp.d ** -0.5, shp.block_q, shp.block_k,
                              w["groups"], np.unique(rows // shp.block_q), bias=bias_np[h])
        fn = OA.block_mask_to_token_fn(bm[0, h], 128, 128, shp.N)
        bfn = OA.block_bias_fn(bias_np[h], 128, 128, shp.N)
        exp = OA.head_forward(f64(q1[0, h]), f64(k1[0, h]), f64(v1[0, h]), 1, fn, 128 ** -0.5, rows=rows,
                              bias_fn=bfn)
        assert_close_out(f64(o[0, h])[rows], exp, f"c4 h{h}")


@pytest.mark.slow
def test_forward_at_the_schedule_capacity():
    """N = 131072 tokens, the most a CTA's key schedule holds (2048 segments of 64 keys): one full
    head and one arrow head; sampled rows, the first and the last included, against the oracle."""
    w = W.arrow_case(B=1, H=2, n_text=256, grid_hw=(1, 131072 - 256), d=64, block=64, seed=13,
                     fracs=(0.5, 0.5, 0.0), with_cache=False)
    shp = w["shape"]
    assert shp.N == 131072 and sorted(int(x) for x in w["head_mode"]) == [W.HEAD_FULL, W.HEAD_SPARSE]
    o, _ = _run_arrow(w)
    rows = np.unique(np.concatenate([[0, shp.N - 1], np.random.default_rng(13).choice(shp.N, 22, replace=False)]))
    _check_arrow(w, o, rows=rows)
