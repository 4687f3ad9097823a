"""The Python binding refuses buffers smaller than the layouts include/bsa.h
states, before any pointer reaches the library (CPU tensors: nothing runs).

A too-small buffer must fail with the size message; a buffer of the right
size still on the CPU gets past the size check and stops at the device check.
Over a recording stand-in for the library, every wrapper must pass each
buffer's address at its position in the header's argument list.
"""
import ctypes

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


class _Recorder:
    """Stands in for the library: records each call's arguments, returns OK.
    Host-only helpers go to the real library."""

    def __init__(self, real):
        self.real, self.calls = real, {}

    def __getattr__(self, name):
        if name in ("bsa_gna_tiled_len", "bsa_error_string"):
            return getattr(self.real, name)

        def call(*args):
            self.calls[name] = args
            return 0
        return call


@pytest.fixture
def recorded(monkeypatch):
    """The binding over a recording library, with the device check dropped
    (CPU tensors stand in for device ones; nothing is dereferenced)."""
    m = _m()
    rec = _Recorder(m.library())
    monkeypatch.setattr(m, "_lib", lambda: rec)

    def host_ptr(t, dtype=None, name="tensor", numel=None):
        if t is None:
            return None
        m._check_buffer(t, dtype, name, numel)
        return ctypes.c_void_p(t.data_ptr())
    monkeypatch.setattr(m, "_ptr", host_ptr)
    return m, rec


def _addr(a):
    return a.value if isinstance(a, ctypes.c_void_p) else a


def _list_addrs(bl_c):
    return [bl_c.cnt, bl_c.idx, bl_c.flag, bl_c.bitmap, bl_c.max_k]


def _expect_list(bl):
    return [bl.cnt.data_ptr(), bl.idx.data_ptr(), bl.flag.data_ptr(),
            bl.bitmap.data_ptr() if bl.bitmap is not None else None, bl.max_k]


def test_forward_passes_buffers_in_abi_order(recorded):
    m, rec = recorded
    dm = _dims(m)
    q, k, v, o = (_bf16(B, H, N, D) for _ in range(4))
    mode = torch.ones(H, dtype=torch.int32)
    cin, cout = torch.zeros((B, H, N, D)), torch.zeros((B, H, N, D))
    bias = torch.zeros((H, NB, NB))
    bl = _blocks(m)
    g = m.GnaGeom.make((4, 4), (2, 2), (3, 3), (1, 1))
    m.forward(dm, q, k, v, o, mode, blocks=bl, gna=g, cache_in=cin, cache_out=cout, bias=bias, scale=0.25,
              stream=0)
    a = rec.calls["bsa_forward"]
    # bsa_forward(dims, Q, K, V, list, head_mode, gna, cache_in, cache_out, block_bias, scale, O, stream)
    assert a[0]._obj is dm
    assert [_addr(x) for x in (a[1], a[2], a[3])] == [q.data_ptr(), k.data_ptr(), v.data_ptr()]
    assert _list_addrs(a[4]._obj) == _expect_list(bl)
    assert _addr(a[5]) == mode.data_ptr() and a[6]._obj is g
    assert [_addr(x) for x in (a[7], a[8], a[9])] == [cin.data_ptr(), cout.data_ptr(), bias.data_ptr()]
    assert a[10] == 0.25 and _addr(a[11]) == o.data_ptr() and _addr(a[12]) in (0, None)
    m.forward(dm, q, k, v, o, mode, stream=0)
    a = rec.calls["bsa_forward"]
    assert a[4] is None and a[6] is None and a[7] is None and a[8] is None and a[9] is None
    assert a[10] == pytest.approx(D ** -0.5)


def test_mask_and_select_pass_buffers_in_abi_order(recorded):
    m, rec = recorded
    dm = _dims(m)
    bl = _blocks(m)
    mode, win = torch.ones(H, dtype=torch.int32), torch.full((H,), 2, dtype=torch.int32)
    m.build_mask(dm, m.MASK_ARROW, bl, head_mode=mode, window=win, stream=0)
    a = rec.calls["bsa_build_mask"]
    spec = a[1]._obj
    assert spec.kind == m.MASK_ARROW and spec.head_mode == mode.data_ptr() and spec.window == win.data_ptr()
    assert _list_addrs(a[2]._obj) == _expect_list(bl)

    q, k = _bf16(B, H, N, D), _bf16(B, H, N, D)
    sp = m.select_spec(m.SELECT_FULL_SCORE, [(0, NB, 2)], keep_text=False, scale=0.125)
    ws = torch.zeros(4096, dtype=torch.float32)
    bias = torch.zeros((H, NB, NB))
    m.select_topk(dm, q, k, sp, bl, ws, bias=bias, stream=0)
    a = rec.calls["bsa_select_topk"]
    # bsa_select_topk(dims, Q, K, spec, block_bias, workspace, workspace_bytes, list, stream)
    assert [_addr(a[1]), _addr(a[2])] == [q.data_ptr(), k.data_ptr()] and a[3]._obj is sp
    assert _addr(a[4]) == bias.data_ptr() and _addr(a[5]) == ws.data_ptr() and a[6] == 4096 * 4
    assert _list_addrs(a[7]._obj) == _expect_list(bl)
    m.select_topk_static(dm, q, k, sp, bl, stream=0)
    a = rec.calls["bsa_select_topk_static"]
    # bsa_select_topk_static(dims, Q, K, spec, block_bias, list, stream)
    assert [_addr(a[1]), _addr(a[2])] == [q.data_ptr(), k.data_ptr()] and a[4] is None
    assert _list_addrs(a[5]._obj) == _expect_list(bl)


def test_stats_and_permute_pass_buffers_in_abi_order(recorded):
    m, rec = recorded
    dm = _dims(m)
    ym, yo, out = _bf16(B, H, N, D), _bf16(B, H, N, D), torch.zeros(4 * H, dtype=torch.float64)
    m.rse(dm, ym, yo, out, stream=0)
    a = rec.calls["bsa_rse"]
    assert [_addr(x) for x in a[1:4]] == [ym.data_ptr(), yo.data_ptr(), out.data_ptr()]

    la, lb = _blocks(m), _blocks(m)
    jo = torch.zeros((B, H, NB))
    m.jaccard(dm, la, lb, jo, stream=0)
    a = rec.calls["bsa_jaccard"]
    assert _list_addrs(a[1]._obj) == _expect_list(la) and _list_addrs(a[2]._obj) == _expect_list(lb)
    assert _addr(a[3]) == jo.data_ptr()

    n_text, grid, tile = 5, (3, 5, 6), (2, 2, 4)
    g = m.GnaGeom.make(grid, tile, (1, 1, 1), (1, 1, 1))
    n_r, n_t = n_text + 90, m.gna_tiled_len(n_text, g)
    pd = m.dims(B, H, n_r, D, 16, 16, n_text)
    ins = [_bf16(B, H, n_r, D) for _ in range(3)]
    outs = [_bf16(B, H, n_t, D) for _ in range(3)]
    m.permute_tiles(pd, g, ins, outs, stream=0)
    a = rec.calls["bsa_permute_tiles"]
    assert a[2] == 3
    assert list(a[3]) == [t.data_ptr() for t in ins] and list(a[4]) == [t.data_ptr() for t in outs]
    m.unpermute_tiles(pd, g, outs[:1], ins[:1], stream=0)
    a = rec.calls["bsa_unpermute_tiles"]
    assert a[2] == 1 and list(a[3]) == [outs[0].data_ptr()] and list(a[4]) == [ins[0].data_ptr()]
