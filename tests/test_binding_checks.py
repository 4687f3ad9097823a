"""The Python binding refuses buffers smaller than the layouts include/bsa.h
states, before any pointer reaches the library (CPU tensors: nothing runs).

A too-small buffer must fail with the size message; a buffer of the right
size still on the CPU gets past the size check and stops at the device check.
"""
import pytest
import torch


def _m():
    from block_sparse_attention_37_b200 import build
    build.build()
    import block_sparse_attention_37_b200 as m
    return m


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


B, H, N, D, BS = 1, 2, 300, 64, 64      # 5 blocks, ragged tail
NB = 5


def _dims(m):
    return m.dims(B, H, N, D, BS, BS, 0)


def _blocks(m, rows_short=False, idx_short=False, bitmap_short=False):
    bl = m.BlockList.empty(B, H, NB, NB, device="cpu")
    if rows_short:
        bl.cnt = torch.zeros((B, H, NB - 1), dtype=torch.int32)
    if idx_short:
        bl.idx = torch.zeros((B, H, NB, NB - 1), dtype=torch.int32)
    if bitmap_short:
        bl.bitmap = torch.zeros((B, H, NB, NB - 1), dtype=torch.uint8)
    return bl


def test_forward_rejects_short_tensors():
    m = _m()
    dm = _dims(m)
    full = [_bf16(B, H, N, D) for _ in range(4)]
    mode = torch.zeros(H, dtype=torch.int32)
    for i, name in enumerate("QKVO"):
        args = list(full)
        args[i] = _bf16(B, H, N - 1, D)
        with pytest.raises(ValueError, match=f"{name} holds"):
            m.forward(dm, *args, mode)
    with pytest.raises(ValueError, match="head_mode holds"):
        m.forward(dm, *full, torch.zeros(H - 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="cache_in holds"):
        m.forward(dm, *full, mode, cache_in=torch.zeros((B, H, N, D - 1)))
    with pytest.raises(ValueError, match="bias holds"):
        m.forward(dm, *full, mode, bias=torch.zeros((H, NB, NB - 1)))
    for kw, name in (("rows_short", "cnt"), ("idx_short", "idx"), ("bitmap_short", "bitmap")):
        with pytest.raises(ValueError, match=f"{name} holds"):
            m.forward(dm, *full, mode, blocks=_blocks(m, **{kw: True}))
    # right sizes: past every size check, stopped by the device check
    with pytest.raises(ValueError, match="CUDA device"):
        m.forward(dm, *full, mode, blocks=_blocks(m), cache_in=torch.zeros((B, H, N, D)))


def test_mask_select_and_stats_reject_short_tensors():
    m = _m()
    dm = _dims(m)
    with pytest.raises(ValueError, match="window holds"):
        m.build_mask(dm, m.MASK_ARROW, _blocks(m), window=torch.zeros(H - 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="cnt holds"):
        m.build_mask(dm, m.MASK_ARROW, _blocks(m, rows_short=True))
    spec = m.select_spec(m.SELECT_POOLED_QK, [(0, NB, 2)], keep_text=False)
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="K holds"):
        m.select_topk(dm, _bf16(B, H, N, D), _bf16(B, H, N // 2, D), spec, _blocks(m), ws)
    with pytest.raises(ValueError, match="Q holds"):
        m.select_topk_static(dm, _bf16(1), _bf16(B, H, N, D), spec, _blocks(m))
    with pytest.raises(ValueError, match="y_o holds"):
        m.rse(dm, _bf16(B, H, N, D), _bf16(B, H, N, D // 2), torch.zeros(4 * H, dtype=torch.float64))
    with pytest.raises(ValueError, match="out holds"):
        m.rse(dm, _bf16(B, H, N, D), _bf16(B, H, N, D), torch.zeros(4 * H - 1, dtype=torch.float64))
    with pytest.raises(TypeError, match="float64"):
        m.rse(dm, _bf16(B, H, N, D), _bf16(B, H, N, D), torch.zeros(4 * H, dtype=torch.float32))
    with pytest.raises(ValueError, match="out holds"):
        m.jaccard(dm, _blocks(m), _blocks(m), torch.zeros((B, H, NB - 1)))
    with pytest.raises(ValueError, match="CUDA device"):
        m.jaccard(dm, _blocks(m), _blocks(m), torch.zeros((B, H, NB)))


def test_permute_sizes_follow_the_tile_layout():
    m = _m()
    n_text, grid, tile = 5, (3, 5, 6), (2, 2, 4)
    g = m.GnaGeom.make(grid, tile, (1, 1, 1), (1, 1, 1))
    n_r = n_text + 3 * 5 * 6
    n_t = m.gna_tiled_len(n_text, g)
    assert n_t > n_r                              # text and ragged tiles are padded
    dm = m.dims(B, H, n_r, D, 16, 16, n_text)
    raster, tiled = _bf16(B, H, n_r, D), _bf16(B, H, n_t, D)
    with pytest.raises(ValueError, match=r"out\[0\] holds"):
        m.permute_tiles(dm, g, [raster], [_bf16(B, H, n_r, D)])   # raster-sized output is too small
    with pytest.raises(ValueError, match=r"in\[0\] holds"):
        m.unpermute_tiles(dm, g, [raster], [raster])               # the inverse reads the tiled length
    with pytest.raises(ValueError, match="as many outputs"):
        m.permute_tiles(dm, g, [raster, raster], [tiled])
    with pytest.raises(ValueError, match="CUDA device"):
        m.permute_tiles(dm, g, [raster], [tiled])
    with pytest.raises(ValueError, match="CUDA device"):
        m.unpermute_tiles(dm, g, [tiled], [raster])
