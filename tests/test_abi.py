"""The C ABI library loads and exports every symbol include/bsa.h declares.

No kernel is launched here: only host-side argument checks (which return
before any CUDA call) and host-only helpers run.
"""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    from block_sparse_attention_37_b200 import build
    build.build()
    import block_sparse_attention_37_b200 as bsa
    return bsa, bsa.library()


def _declared():
    with open(os.path.join(ROOT, "include", "bsa.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    bsa, lib = _lib()
    names = _declared()
    assert "bsa_forward" in names and "bsa_select_topk" in names and "bsa_build_mask" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(bsa.EXPORTS) <= set(names)


def test_error_strings_and_version():
    bsa, lib = _lib()
    assert lib.bsa_error_string(0) == b"ok"
    assert lib.bsa_error_string(3) == b"workspace missing or too small"
    assert lib.bsa_version() >= 100


def test_host_argument_checks_return_before_launch():
    bsa, lib = _lib()
    # null dims / null tensors / bad head dim -> rejected on the host
    assert lib.bsa_forward(None, None, None, None, None, None, None, None, None, None, 1.0, None, None) \
        == bsa.ERR_INVALID_ARG
    dm = bsa.dims(1, 1, 128, 96, 64, 64, 0)
    p = ctypes.c_void_p(256)
    mode = ctypes.c_void_p(512)
    assert lib.bsa_forward(ctypes.byref(dm), p, p, p, None, mode, None, None, None, None, 1.0, p, None) \
        == bsa.ERR_UNSUPPORTED
    dm = bsa.dims(1, 1, 128, 64, 48, 64, 0)
    assert lib.bsa_forward(ctypes.byref(dm), p, p, p, None, mode, None, None, None, None, 1.0, p, None) \
        == bsa.ERR_UNSUPPORTED
    # the key schedule holds 2048 segments of 64 keys: N = 131072 is the largest sequence
    dm_max = bsa.dims(1, 1, 131073, 64, 64, 64, 0)
    assert lib.bsa_forward(ctypes.byref(dm_max), p, p, p, None, mode, None, None, None, None, 1.0, p, None) \
        == bsa.ERR_UNSUPPORTED
    bad = ctypes.c_void_p(257)  # not 16-byte aligned
    dm = bsa.dims(1, 1, 128, 64, 64, 64, 0)
    assert lib.bsa_forward(ctypes.byref(dm), bad, p, p, None, mode, None, None, None, None, 1.0, p, None) \
        == bsa.ERR_INVALID_ARG
    # list capacity below nKB
    lst = bsa.BlockListC(p, p, p, None, 1)
    spec = bsa.MaskSpec(bsa.MASK_ARROW, None, None, bsa.GnaGeom())
    assert lib.bsa_build_mask(ctypes.byref(dm), ctypes.byref(spec), ctypes.byref(lst), None) == bsa.ERR_INVALID_ARG
    # arrow needs equal block sizes
    dm2 = bsa.dims(1, 1, 256, 64, 64, 128, 0)
    lst2 = bsa.BlockListC(p, p, p, None, 8)
    assert lib.bsa_build_mask(ctypes.byref(dm2), ctypes.byref(spec), ctypes.byref(lst2), None) == bsa.ERR_UNSUPPORTED
    # workspace too small
    sp = bsa.select_spec(bsa.SELECT_POOLED_QK, [(0, 2, 1)], False)
    assert lib.bsa_select_topk(ctypes.byref(dm), p, p, ctypes.byref(sp), None, p, 16, ctypes.byref(lst2), None) \
        == bsa.ERR_WORKSPACE
    # the allocation-free selection runs the same argument checks before its scratch-size check:
    # an unsupported request that is also too large for the scratch reports UNSUPPORTED
    big_bad = bsa.dims(1, 64, 131072, 96, 128, 128, 0)
    lst_big = bsa.BlockListC(p, p, p, None, 1024)
    fs = bsa.select_spec(bsa.SELECT_FULL_SCORE, [(0, 1024, 8)], False, 0.1)
    assert lib.bsa_select_topk_static(ctypes.byref(big_bad), p, p, ctypes.byref(fs), None,
                                      ctypes.byref(lst_big), None) == bsa.ERR_UNSUPPORTED
    big_bs64 = bsa.dims(1, 64, 131072, 128, 64, 64, 0)
    lst_big64 = bsa.BlockListC(p, p, p, None, 2048)
    fs64 = bsa.select_spec(bsa.SELECT_FULL_SCORE, [(0, 2048, 8)], False, 0.1)
    assert lib.bsa_select_topk_static(ctypes.byref(big_bs64), p, p, ctypes.byref(fs64), None,
                                      ctypes.byref(lst_big64), None) == bsa.ERR_UNSUPPORTED
    assert lib.bsa_select_topk_static(ctypes.byref(big_bs64), bad, p, ctypes.byref(fs64), None,
                                      ctypes.byref(lst_big64), None) == bsa.ERR_INVALID_ARG
    # a valid request above the fixed scratch size is refused before any launch
    big_ok = bsa.dims(1, 64, 131072, 128, 128, 128, 0)
    assert bsa.select_workspace_size(big_ok, fs) > 16 << 20
    assert lib.bsa_select_topk_static(ctypes.byref(big_ok), p, p, ctypes.byref(fs), None,
                                      ctypes.byref(lst_big), None) == bsa.ERR_WORKSPACE
    # invalid GNA geometry (stride > window)
    g = bsa.GnaGeom.make((8,), (64,), (4,), (5,))
    n = ctypes.c_int32(0)
    assert lib.bsa_gna_tiled_len(0, ctypes.byref(g), ctypes.byref(n)) == bsa.ERR_INVALID_ARG
    # bsa_rse: null output, unaligned input, N*d not a multiple of 8
    assert lib.bsa_rse(ctypes.byref(dm), p, p, None, None) == bsa.ERR_INVALID_ARG
    assert lib.bsa_rse(ctypes.byref(dm), bad, p, p, None) == bsa.ERR_INVALID_ARG
    dm3 = bsa.dims(1, 1, 3, 4, 64, 64, 0)
    assert lib.bsa_rse(ctypes.byref(dm3), p, p, p, None) == bsa.ERR_UNSUPPORTED
    # bsa_jaccard: missing list or output
    assert lib.bsa_jaccard(ctypes.byref(dm), ctypes.byref(lst2), None, p, None) == bsa.ERR_INVALID_ARG
    assert lib.bsa_jaccard(ctypes.byref(dm), ctypes.byref(lst2), ctypes.byref(lst2), None, None) \
        == bsa.ERR_INVALID_ARG
    assert lib.bsa_error_string(bsa.ERR_INFEASIBLE) == b"no plan meets the error budget"
    # failure-detection settings: host-only, no launch
    assert lib.bsa_set_withheld_tile(-2) == bsa.ERR_INVALID_ARG
    assert lib.bsa_set_withheld_tile(-1) == bsa.OK
    assert lib.bsa_set_wait_limit_ns(0) == bsa.OK


@pytest.mark.parametrize("n_text,grid,tile", [(256, (16, 48, 80), (4, 8, 8)), (5, (3, 5, 6), (2, 2, 4)),
                                              (0, (10,), (4,)), (70, (6, 7), (4, 4))])
def test_tiled_len_matches_oracle_layout(n_text, grid, tile):
    bsa, lib = _lib()
    from oracle.masks import GnaLayout
    g = bsa.GnaGeom.make(grid, tile, tuple(1 for _ in grid), tuple(1 for _ in grid))
    assert bsa.gna_tiled_len(n_text, g) == GnaLayout(n_text, grid, tile, tuple(1 for _ in grid),
                                                    tuple(1 for _ in grid)).N


def test_workspace_sizes():
    bsa, lib = _lib()
    dm = bsa.dims(1, 24, 16896, 128, 128, 128, 512)
    sp = bsa.select_spec(bsa.SELECT_POOLED_QK, [(4, 132, 39)], True)
    assert bsa.select_workspace_size(dm, sp) >= 2 * 24 * 132 * 128 * 4
    sp2 = bsa.select_spec(bsa.SELECT_FULL_SCORE, [(0, 240, 72), (240, 256, 5)], False, 0.088)
    dm2 = bsa.dims(1, 32, 32768, 128, 128, 128, 0)
    assert bsa.select_workspace_size(dm2, sp2) >= 32 * 32768 * 4 + 32 * 256 * 256 * 4


def test_full_score_workspace_below_the_reported_size_is_refused():
    """bsa_select_topk's contract: at least bsa_select_workspace_size bytes. One 256-byte step
    less is refused before any CUDA call, although the two-pass form would fit in it."""
    bsa, lib = _lib()
    dm = bsa.dims(1, 32, 32768, 128, 128, 128, 0)
    sp = bsa.select_spec(bsa.SELECT_FULL_SCORE, [(0, 240, 72), (240, 256, 5)], False, 0.088)
    need = bsa.select_workspace_size(dm, sp)
    assert need > 32 * 32768 * 4 + 32 * 256 * 256 * 4  # the one-pass slabs are included
    p = ctypes.c_void_p(256)
    lst = bsa.BlockListC(p, p, p, None, 256)
    assert lib.bsa_select_topk(ctypes.byref(dm), p, p, ctypes.byref(sp), None, p, need - 256,
                               ctypes.byref(lst), None) == bsa.ERR_WORKSPACE


def test_cpu_tensors_are_rejected():
    bsa, lib = _lib()
    import torch
    dm = bsa.dims(1, 1, 128, 64, 64, 64, 0)
    t = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        bsa.forward(dm, t, t, t, t, torch.zeros(1, dtype=torch.int32))
