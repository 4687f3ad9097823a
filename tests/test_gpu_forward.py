"""GPU bsa_forward vs the fp64 oracle (max-abs 2e-2, mean-abs 5e-3 on bf16 outputs)."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from oracle import masks as OM
from oracle import permute as OP
from oracle import select as OS
from parity_util import arrow_expected, assert_close_out, bsa, check_pooled_rows, f64

pytestmark = pytest.mark.gpu


def _dims(shp):
    return bsa().dims(shp.B, shp.H, shp.N, shp.d, shp.block_q, shp.block_k, shp.n_text)


def _run_arrow(w, cache_out=False, bias=None):
    m = bsa()
    shp = w["shape"]
    dm = _dims(shp)
    q, k, v = (t.cuda() for t in (w["q"], w["k"], w["v"]))
    modes = torch.from_numpy(w["head_mode"]).cuda()
    wins = torch.from_numpy(w["window"]).cuda()
    blocks = m.BlockList.empty(shp.B, shp.H, shp.n_qb, shp.n_kb, bitmap=False)
    m.build_mask(dm, m.MASK_ARROW, blocks, head_mode=modes, window=wins)
    o = torch.empty_like(q)
    cin = w.get("cache")
    cin = cin.cuda() if cin is not None else None
    cout = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda") if cache_out else None
    b = bias.cuda() if bias is not None else None
    m.forward(dm, q, k, v, o, modes, blocks=blocks, cache_in=cin, cache_out=cout, bias=b)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    return o, cout


def _check_arrow(w, o, rows=None, cout=None, bias=None, heads=None):
    shp = w["shape"]
    worst = 0.0
    for b in range(shp.B):
        for h in (range(shp.H) if heads is None else heads):
            exp = arrow_expected(w["q"], w["k"], w["v"], shp, w["head_mode"], w["window"], b, h, rows=rows,
                                 cache=w.get("cache"), bias=bias)
            got = f64(o[b, h]) if rows is None else f64(o[b, h])[rows]
            if int(w["head_mode"][h]) == W.HEAD_SKIP:
                np.testing.assert_array_equal(got, exp)  # bit-exact bf16 of the cache
                if cout is not None:
                    assert torch.isnan(cout[b, h]).all(), "SKIP heads must not write cache_out"
                continue
            mx, _ = assert_close_out(got, exp, f"b{b} h{h} mode{w['head_mode'][h]}")
            worst = max(worst, mx)
            if cout is not None:
                gc = cout[b, h].double().cpu().numpy()
                gc = gc if rows is None else gc[rows]
                assert np.abs(gc - exp).max() <= 5e-3
    return worst


def test_forward_c1_all_rows():
    w = W.c1()
    o, _ = _run_arrow(w)
    _check_arrow(w, o)


def test_forward_c2_all_rows():
    """The benchmarked workload, every output row of every (b, h)."""
    w = W.c2()
    o, cout = _run_arrow(w, cache_out=True)
    _check_arrow(w, o, cout=cout)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [64, 128, 256])
def test_forward_arrow_ragged(d, bs):
    """Ragged N (tail block), partial text block, all three modes, fp32 cache_out."""
    N = bs * 4 + 77
    w = W.arrow_case(B=1, H=6, n_text=70, grid_hw=(1, N - 70), d=d, block=bs, seed=d + bs,
                     fracs=(0.34, 0.5, 0.16))
    o, cout = _run_arrow(w, cache_out=True)
    _check_arrow(w, o, cout=cout)


def test_forward_block_bias():
    N, bs = 128 * 6 + 40, 128
    w = W.arrow_case(B=1, H=4, n_text=128, grid_hw=(1, N - 128), d=128, block=bs, seed=11,
                     fracs=(0.5, 0.5, 0.0))
    nb = -(-N // bs)
    bias = torch.from_numpy(np.random.default_rng(3).normal(0, 2, (4, nb, nb)).astype(np.float32))
    o, _ = _run_arrow(w, bias=bias)
    _check_arrow(w, o, bias=bias.numpy())


def test_forward_dense_matches_library_sdpa():
    """All heads FULL = plain attention; cross-checked with torch's fp64 SDPA as well."""
    B, H, N, d = 1, 2, 600, 64
    q, k, v = W.qkv_normal(B, H, N, d, 21)
    w = dict(shape=W.Shape(B, H, N, d, 64, 64, 0), q=q, k=k, v=v,
             head_mode=np.zeros(H, np.int32), window=np.zeros(H, np.int32))
    o, _ = _run_arrow(w)
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double())
    assert_close_out(f64(o), ref.numpy(), "dense vs sdpa")


def test_forward_empty_rows_are_zero():
    m = bsa()
    B, H, N, d, bs = 1, 1, 512, 64, 64
    q, k, v = (t.cuda() for t in W.qkv_normal(B, H, N, d, 5))
    nb = N // bs
    blocks = m.BlockList.empty(B, H, nb, nb, bitmap=False)
    cnt = torch.tensor([[[2, 0, 1, 0, 3, 0, 0, 1]]], dtype=torch.int32)
    idx = torch.full((B, H, nb, nb), -1, dtype=torch.int32)
    lists = {0: [0, 5], 2: [7], 4: [1, 2, 3], 7: [7]}
    for I, js in lists.items():
        idx[0, 0, I, :len(js)] = torch.tensor(js)
    blocks.cnt.copy_(cnt)
    blocks.idx.copy_(idx)
    blocks.flag.copy_((idx >= 0).to(torch.uint8))
    o = torch.empty_like(q)
    modes = torch.ones(H, dtype=torch.int32, device="cuda")
    m.forward(m.dims(B, H, N, d, bs, bs, 0), q, k, v, o, modes, blocks=blocks)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    cls = np.zeros((nb, nb), np.uint8)
    for I, js in lists.items():
        cls[I, js] = 1
    fn = OA.block_mask_to_token_fn(cls, bs, bs, N)
    exp = OA.head_forward(f64(q[0, 0]), f64(k[0, 0]), f64(v[0, 0]), 1, fn, 1 / 8.0)
    assert_close_out(f64(o[0, 0]), exp)
    for I in (1, 3, 5, 6):
        assert torch.all(o[0, 0, I * bs:(I + 1) * bs] == 0)


def test_forward_selected_blocks_from_oracle_selection():
    """Irregular per-row lists: the oracle's pooled top-k selection fed to the GPU forward."""
    m = bsa()
    w = W.content_case(B=1, H=3, n_text=256, grid_hw=(32, 32), d=128, block=128, seed=9)
    shp = w["shape"]
    ntb = 2
    groups = [(ntb, shp.n_kb, 3)]
    blocks = m.BlockList.empty(1, 3, shp.n_qb, shp.n_kb, bitmap=False)
    cls_all = np.zeros((1, 3, shp.n_qb, shp.n_kb), np.uint8)
    for h in range(3):
        cls_all[0, h], _ = OS.pooled_select(f64(w["q"][0, h]), f64(w["k"][0, h]), 128, 128, 256, groups, True)
    cnt, idx, flag = zip(*[OM.to_csr(cls_all[0, h]) for h in range(3)])
    blocks.cnt.copy_(torch.from_numpy(np.stack(cnt))[None])
    blocks.idx.copy_(torch.from_numpy(np.stack(idx))[None])
    blocks.flag.copy_(torch.from_numpy(np.stack(flag))[None])
    q, k, v = (t.cuda() for t in (w["q"], w["k"], w["v"]))
    o = torch.empty_like(q)
    m.forward(_dims(shp), q, k, v, o, torch.ones(3, dtype=torch.int32, device="cuda"), blocks=blocks)
    torch.cuda.synchronize()
    for h in range(3):
        fn = OA.block_mask_to_token_fn(cls_all[0, h], 128, 128, shp.N)
        exp = OA.head_forward(f64(w["q"][0, h]), f64(w["k"][0, h]), f64(w["v"][0, h]), 1, fn, 128 ** -0.5)
        assert_close_out(f64(o[0, h]), exp, f"h{h}")


def _tile_rows(lay, tiles):
    """Tile-order positions of every token of the listed tiles (tile coordinates per dim; None is
    the text tile)."""
    out = []
    for t in tiles:
        if t is None:
            out.append(np.arange(lay.text_span))
            continue
        lin = 0
        for c, n in zip(t, lay.tiles):
            assert 0 <= c < n
            lin = lin * n + c
        start = lay.text_span + lin * lay.vol
        out.append(np.arange(start, start + lay.vol))
    return np.concatenate(out)


def _gna_forward(B, H, n_text, grid, tile, window, stride, d, seed, modes, rows_per_head=None,
                 all_rows_tiles=(), all_rows_heads=()):
    """Raster inputs -> GPU permute -> mask -> forward -> unpermute; oracle on sampled rows.

    Heads in ``all_rows_heads`` also compare every row of the tiles in ``all_rows_tiles``."""
    m = bsa()
    wl = W.video_case(B, H, n_text, grid, tile, window, stride, d, seed)
    lay = OM.GnaLayout(n_text, grid, tile, window, stride)
    g = m.GnaGeom.make(grid, tile, window, stride)
    nt = m.gna_tiled_len(n_text, g)
    assert nt == lay.N
    dm_r = m.dims(B, H, wl["shape"].N, d, lay.bs, lay.bs, n_text)
    dm = m.dims(B, H, nt, d, lay.bs, lay.bs, n_text)
    raster = [t.cuda() for t in (wl["q"], wl["k"], wl["v"])]
    tiled = [torch.empty((B, H, nt, d), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    m.permute_tiles(dm_r, g, raster, tiled)
    nb = nt // lay.bs
    blocks = m.BlockList.empty(B, H, nb, nb, bitmap=False)
    mt = torch.from_numpy(np.asarray(modes, np.int32)).cuda()
    m.build_mask(dm, m.MASK_GNA, blocks, head_mode=mt, gna=g)
    o_t = torch.empty_like(tiled[0])
    m.forward(dm, *tiled, o_t, mt, blocks=blocks, gna=g)
    o = torch.empty_like(raster[0])
    m.unpermute_tiles(dm_r, g, [o_t], [o])
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    src = OP.tile_order_source(lay)
    valid = lay.valid(np.arange(nt))
    rng = np.random.default_rng(seed)
    for b in range(B):
        for h in range(H):
            qt, kt, vt = (OP.permute_to_tiles(f64(t[b, h]), lay) for t in (wl["q"], wl["k"], wl["v"]))
            cand = np.nonzero(valid)[0]
            rows = cand if rows_per_head is None else np.sort(rng.choice(cand, rows_per_head, replace=False))
            if h in all_rows_heads and rows_per_head is not None:
                extra = _tile_rows(lay, all_rows_tiles)
                rows = np.unique(np.concatenate([rows, extra[valid[extra]]]))
            mode = int(modes[h])
            if mode == OM.HEAD_FULL:
                fn = lambda r: valid[np.asarray(r)][:, None] & valid[None, :]
            else:
                fn = lambda r: OM.gna_token_mask(lay, r)
            exp = OA.head_forward(qt, kt, vt, mode, fn, d ** -0.5, rows=rows)
            got = f64(o[b, h])[src[rows]]
            assert_close_out(got, exp, f"gna b{b} h{h}")


@pytest.mark.parametrize("n_text,grid,tile,window,stride", [
    (64, (4, 8, 16), (2, 4, 8), (3, 5, 7), (1, 1, 1)),      # partial tiles everywhere
    (50, (5, 9, 20), (2, 4, 8), (3, 5, 7), (1, 2, 2)),      # padding in grid and text
    (0, (300,), (64,), (97,), (5,)),                          # 1-D, padded last tile
    (128, (8, 256), (1, 128), (3, 48), (1, 16)),              # x tile wider than a segment
    # one-slice layouts (each 64-key segment in one y-x slice of a tile), with padding: the
    # forward's instantiation for them, and the per-group narrowing of partial segments
    (128, (4, 12, 20), (2, 8, 8), (3, 9, 11), (1, 1, 1)),
    (128, (4, 12, 20), (2, 8, 8), (3, 9, 11), (1, 3, 2)),
    (40, (3, 20, 10), (1, 16, 4), (3, 7, 5), (1, 2, 1)),      # block 64, padded text
])
def test_forward_gna_small(n_text, grid, tile, window, stride):
    _gna_forward(1, 3, n_text, grid, tile, window, stride, 128, 7, modes=[1, 0, 1])


# Tiles of the 4 x 6 x 10 tile grid of the video workload where windows clamp: two opposite
# corners, a corner on the other diagonal, and one tile on a face of each dimension; None is the
# text tile (full rows).
C5_EDGE_TILES = ((0, 0, 0), (3, 5, 9), (3, 5, 0), (0, 2, 4), (2, 0, 5), (1, 4, 9), None)


@pytest.mark.slow
@pytest.mark.parametrize("stride", [(4, 8, 8), (1, 1, 1)])
def test_forward_c5_sampled_rows(stride):
    """24 sampled rows of every head, plus every row of the corner and face tiles on three heads."""
    _gna_forward(1, 24, 256, (16, 48, 80), (4, 8, 8), (8, 16, 24), stride, 128, 4, modes=[1] * 24,
                 rows_per_head=24, all_rows_tiles=C5_EDGE_TILES, all_rows_heads=(0, 11, 23))


def test_forward_c3_sampled_rows_with_gpu_selection():
    """FLUX-2048-like: GPU pooled selection, then the GPU forward; 16 sampled rows of every head.

    Each sampled row's block row of the GPU selection is first checked against the oracle's
    pooled scores; only a row that passes becomes the oracle forward's mask."""
    m = bsa()
    w = W.c3()
    shp = w["shape"]
    dm = _dims(shp)
    q, k, v = (t.cuda() for t in (w["q"], w["k"], w["v"]))
    sp = m.select_spec(m.SELECT_POOLED_QK, w["groups"], True)
    ws = torch.empty(m.select_workspace_size(dm, sp), dtype=torch.uint8, device="cuda")
    blocks = m.BlockList.empty(1, shp.H, shp.n_qb, shp.n_kb)
    m.select_topk(dm, q, k, sp, blocks, ws)
    o = torch.empty_like(q)
    m.forward(dm, q, k, v, o, torch.ones(shp.H, dtype=torch.int32, device="cuda"), blocks=blocks)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    bm = blocks.bitmap.cpu().numpy()
    rng = np.random.default_rng(0)
    for h in range(shp.H):
        rows = np.unique(np.concatenate([[0, shp.N - 1], rng.choice(shp.N, 14, replace=False)]))
        qh, kh = f64(w["q"][0, h]), f64(w["k"][0, h])
        check_pooled_rows(bm[0, h], qh, kh, shp.block_q, shp.block_k, shp.n_text, w["groups"],
                          np.unique(rows // shp.block_q))
        fn = OA.block_mask_to_token_fn(bm[0, h], 128, 128, shp.N)
        exp = OA.head_forward(qh, kh, f64(w["v"][0, h]), 1, fn, 128 ** -0.5, rows=rows)
        assert_close_out(f64(o[0, h])[rows], exp, f"c3 h{h}")
