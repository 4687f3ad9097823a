"""bsa_select_topk_static: the selection entry point for callers that cannot allocate.

Some callers plan every device buffer ahead (a fixed arena, no allocator on the
call path) or must not call cudaMalloc in a latency-critical loop, so they
cannot hand bsa_select_topk a workspace. bsa_select_topk_static runs the same
kernels on a fixed scratch array inside the library. Here it is called through
the C ABI twice in a row (the second call finds the first call's leftovers in
the shared scratch) and compared with bsa_select_topk on a caller workspace.
This file is collected last so that a stop-at-first-failure run has already
run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
from oracle import select as OS
from parity_util import bsa, check_full_score_rows, f64, list_to_classes, selection_matches

pytestmark = pytest.mark.gpu


def _with_workspace(m, dm, q, k, spec, nqb, nkb, bias=None):
    out = m.BlockList.empty(dm.B, dm.H, nqb, nkb)
    ws = torch.empty(m.select_workspace_size(dm, spec), dtype=torch.uint8, device="cuda")
    m.select_topk(dm, q, k, spec, out, ws, bias=bias)
    torch.cuda.synchronize()
    return out


def _static_via_c_abi(m, dm, q, k, spec, nqb, nkb, bias=None):
    out = m.BlockList.empty(dm.B, dm.H, nqb, nkb)
    lc = out.c()
    st = m.library().bsa_select_topk_static(
        ctypes.byref(dm), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.byref(spec),
        ctypes.c_void_p(bias.data_ptr()) if bias is not None else None, ctypes.byref(lc),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == m.OK, m.library().bsa_error_string(st)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    return out


def test_static_pooled_selection_matches_workspace_version_twice():
    m = bsa()
    B, H, N, d, bs, n_text = 1, 4, 128 * 20 + 50, 128, 128, 256
    w = W.content_case(B=B, H=H, n_text=n_text, grid_hw=(1, N - n_text), d=d, block=bs, seed=31)
    q, k = w["q"].cuda(), w["k"].cuda()
    nb = -(-N // bs)
    dm = m.dims(B, H, N, d, bs, bs, n_text)
    spec = m.select_spec(m.SELECT_POOLED_QK, [(2, nb, 6)], True)
    ref = _with_workspace(m, dm, q, k, spec, nb, nb)
    for _ in range(2):
        got = _static_via_c_abi(m, dm, q, k, spec, nb, nb)
        for name in ("cnt", "idx", "flag", "bitmap"):
            assert torch.equal(getattr(got, name), getattr(ref, name)), name


def test_static_full_score_selection_matches_workspace_version_twice():
    m = bsa()
    B, H, N, d, bs = 1, 3, 128 * 12 + 30, 128, 128
    q, k, _ = W.qkv_normal(B, H, N, d, 41)
    nb = -(-N // bs)
    groups = [(0, nb - 2, 4), (nb - 2, nb, 1)]
    bias, _ = W.dlm_bias(H, nb, nb - 2, seed=7, n_col_pre=3, n_col_gen=1, windows=(1, 2))
    dm = m.dims(B, H, N, d, bs, bs, 0)
    spec = m.select_spec(m.SELECT_FULL_SCORE, groups, False, d ** -0.5)
    qd, kd, bd = q.cuda(), k.cuda(), bias.cuda()
    ref = list_to_classes(_with_workspace(m, dm, qd, kd, spec, nb, nb, bd), nb)
    for _ in range(2):
        got = list_to_classes(_static_via_c_abi(m, dm, qd, kd, spec, nb, nb, bd), nb)
        for h in range(H):
            _, ap = OS.full_score_select(f64(q[0, h]), f64(k[0, h]), d ** -0.5, bs, bs, groups,
                                         bias=bias[h].numpy())
            for I in range(nb):
                if np.array_equal(got[0, h, I], ref[0, h, I]):
                    continue
                # fp32 atomics may order a near-tie differently; both must still be valid selections
                for row in (got[0, h, I], ref[0, h, I]):
                    ok, _ = selection_matches(row > 0, ap[I], groups, np.zeros(nb, bool))
                    assert ok, (h, I)


def test_static_one_pass_in_two_chunks_equals_one_chunk():
    """128 heads x 2048 tokens: the scratch holds the per-tile LSE slabs of 2032 of the 2048 query
    blocks, so the static entry runs the one-pass form in two chunks; a caller workspace of the
    reported size runs it in one. Every query block takes the same arithmetic either way: the
    block lists are identical."""
    m = bsa()
    B, H, N, d, bs = 1, 128, 2048, 128, 128
    q, k, _ = W.qkv_normal(B, H, N, d, 43)
    nb = N // bs
    dm = m.dims(B, H, N, d, bs, bs, 0)
    spec = m.select_spec(m.SELECT_FULL_SCORE, [(0, nb - 2, 5), (nb - 2, nb, 1)], False, d ** -0.5)
    qd, kd = q.cuda(), k.cuda()
    ref = _with_workspace(m, dm, qd, kd, spec, nb, nb)
    got = _static_via_c_abi(m, dm, qd, kd, spec, nb, nb)
    for name in ("cnt", "idx", "flag", "bitmap"):
        assert torch.equal(getattr(got, name), getattr(ref, name)), name


def test_static_two_pass_form_agrees_with_the_one_pass_form():
    """8 heads x 16384 tokens: too many slabs for the scratch's minimum chunk, so the static entry
    runs the two-pass form (row LSE, then block sums with atomics) while the caller workspace runs
    the one-pass form. Rows where the two differ must both be valid selections of the oracle's
    A' (near-ties only), and they must be rare."""
    m = bsa()
    B, H, N, d, bs = 1, 8, 16384, 128, 128
    q, k, _ = W.qkv_normal(B, H, N, d, 47)
    nb = N // bs
    groups = [(0, nb - 8, 38), (nb - 8, nb, 2)]
    bias, _ = W.dlm_bias(H, nb, nb - 8, seed=11, n_col_pre=6, n_col_gen=1, windows=(2, 4))
    dm = m.dims(B, H, N, d, bs, bs, 0)
    spec = m.select_spec(m.SELECT_FULL_SCORE, groups, False, d ** -0.5)
    qd, kd, bd = q.cuda(), k.cuda(), bias.cuda()
    ref = list_to_classes(_with_workspace(m, dm, qd, kd, spec, nb, nb, bd), nb)
    got = list_to_classes(_static_via_c_abi(m, dm, qd, kd, spec, nb, nb, bd), nb)
    diff = [(h, I) for h in range(H) for I in range(nb) if not np.array_equal(got[0, h, I], ref[0, h, I])]
    assert len(diff) <= H * nb // 50, len(diff)
    for h in sorted({h for h, _ in diff}):
        rows = np.array([I for hh, I in diff if hh == h])
        for cls in (got, ref):
            check_full_score_rows(cls[0, h], f64(q[0, h]), f64(k[0, h]), d ** -0.5, bs, bs, groups, rows,
                                  bias=bias[h].numpy())


def test_static_rejects_requests_beyond_its_scratch():
    m = bsa()
    B, H, N, d, bs = 1, 64, 32768, 128, 128  # full-score needs 24 MiB > 16 MiB
    dm = m.dims(B, H, N, d, bs, bs, 0)
    spec = m.select_spec(m.SELECT_FULL_SCORE, [(0, 240, 72), (240, 256, 5)], False, d ** -0.5)
    assert m.select_workspace_size(dm, spec) > m.STATIC_SCRATCH_BYTES
    p = ctypes.c_void_p(256)
    lst = m.BlockListC(p, p, p, None, 256)
    st = m.library().bsa_select_topk_static(ctypes.byref(dm), p, p, ctypes.byref(spec), None,
                                            ctypes.byref(lst), None)
    assert st == m.ERR_WORKSPACE
