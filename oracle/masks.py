"""Token-level masks and their block classification (fp64 oracle, test use only).

Readings of the pages used here (each is the plainest one the text supports):

* Sequence order: text tokens first, then the image/video tokens.
* Arrow attention (DiTFastAttnV2, "Head-wise Arrow Attention"): the joint map
  splits into visual-visual, visual-text, text-visual and text-text regions;
  the three regions that touch text stay full and the visual-visual region
  keeps only blocks near the diagonal. Mixed blocks are made dense ("Fused
  Kernel": blocks are converted to dense blocks), so the arrow pattern is
  block-granular: block (I, J) is kept iff I or J holds a text token or
  |I - J| <= w, w in blocks. Needs block_q == block_k.
* GNA (jsqmd.com GNA article, section 1.1): per dimension of length L with
  window k and stride s, query i reads the keys
  [start(i), start(i) + k) with
  start(i) = clamp(s*floor(i/s) - s*floor((k-s)/(2s)), 0, L-k).
  At s = 1 this is clamped neighborhood attention; every query in a stride
  group shares one window; with tile-aligned strides the pattern is
  "perfectly block-sparse". A token pair is allowed iff the key is inside the
  window in every dimension. Text tokens are full rows and columns.
* Block classes: a (Q block, KV block) pair is FULL when every pair of real
  tokens is allowed and the KV block holds no padding, NONE when no pair is
  allowed, PARTIAL otherwise ("dynamic mask": the fine mask runs only on
  partially covered KV tiles).
"""
from __future__ import annotations

import numpy as np

HEAD_FULL, HEAD_SPARSE, HEAD_SKIP = 0, 1, 2
BLOCK_NONE, BLOCK_FULL, BLOCK_PARTIAL = 0, 1, 2


def n_blocks(n: int, bs: int) -> int:
    return -(-n // bs)


# ----------------------------------------------------------------------------
# arrow


def arrow_token_mask(N, n_text, bs, mode, window, rows=None):
    """bool [len(rows), N]: may query i attend key j under the arrow pattern.

    DiTFastAttnV2, "Head-wise Arrow Attention" and "Fused Kernel" (mixed
    blocks densified). FULL heads allow everything, SKIP heads nothing.
    A block holding any text token is a text block.
    """
    rows = np.arange(N) if rows is None else np.asarray(rows)
    if mode == HEAD_FULL:
        return np.ones((len(rows), N), dtype=bool)
    if mode == HEAD_SKIP:
        return np.zeros((len(rows), N), dtype=bool)
    ntb = n_blocks(n_text, bs)
    bq = rows // bs
    bk = np.arange(N) // bs
    text_q = bq < ntb
    text_k = bk < ntb
    near = np.abs(bq[:, None] - bk[None, :]) <= window
    return text_q[:, None] | text_k[None, :] | near


# ----------------------------------------------------------------------------
# GNA


def _pad3(v, fill=1):
    v = tuple(int(x) for x in v)
    return (fill,) * (3 - len(v)) + v


class GnaLayout:
    """Tile-order token layout for GNA over a text prefix plus a 1..3-D grid.

    Positions [0, n_text) are text, [n_text, ntb*bs) are zero padding, then
    the video tiles follow in raster order of the tile grid, each tile's
    tokens in raster order inside the tile. Tiles at the far edge of a grid
    whose length is not a tile multiple are padded; padded tokens are not
    valid keys. Block size bs equals the tile volume.
    (jsqmd.com GNA article, section 1.1 multi-dimensional tiling and 2.2
    token permutation.)
    """

    def __init__(self, n_text, grid, tile, window, stride):
        self.n_text = int(n_text)
        self.grid = _pad3(grid)
        self.tile = _pad3(tile)
        self.window = _pad3(window)
        self.stride = _pad3(stride)
        for L, T, k, s in zip(self.grid, self.tile, self.window, self.stride):
            if not (1 <= s <= k <= L) or T < 1:
                raise ValueError("need 1 <= stride <= window <= grid and tile >= 1")
        self.vol = int(np.prod(self.tile))
        self.bs = self.vol
        self.ntb = n_blocks(self.n_text, self.bs)
        self.tiles = tuple(n_blocks(L, T) for L, T in zip(self.grid, self.tile))
        self.n_tiles = int(np.prod(self.tiles))
        self.text_span = self.ntb * self.bs
        self.N = self.text_span + self.n_tiles * self.vol

    def coords(self, pos):
        """(kind, coords[...,3]) for positions: kind 0 text, 1 padding, 2 video."""
        pos = np.asarray(pos, dtype=np.int64)
        kind = np.where(pos < self.n_text, 0, np.where(pos < self.text_span, 1, 2))
        v = np.maximum(pos - self.text_span, 0)
        tile_id = v // self.vol
        local = v % self.vol
        Gt, Gy, Gx = self.tiles
        Tt, Ty, Tx = self.tile
        tt, ty, tx = tile_id // (Gy * Gx), (tile_id // Gx) % Gy, tile_id % Gx
        lt, ly, lx = local // (Ty * Tx), (local // Tx) % Ty, local % Tx
        c = np.stack([tt * Tt + lt, ty * Ty + ly, tx * Tx + lx], axis=-1)
        inside = np.all(c < np.array(self.grid), axis=-1)
        kind = np.where((kind == 2) & ~inside, 1, kind)
        return kind, c

    def valid(self, pos):
        kind, _ = self.coords(pos)
        return kind != 1


def window_start(i, L, k, s):
    """First key of query i's window in one dimension (reading stated above)."""
    i = np.asarray(i, dtype=np.int64)
    start = s * (i // s) - s * ((k - s) // (2 * s))
    return np.clip(start, 0, L - k)


def gna_token_mask(lay: GnaLayout, rows=None, cols=None):
    """bool [len(rows), len(cols)] over tile-order positions.

    jsqmd.com GNA article, section 1.1: key inside the query's window in every
    dimension; text rows and columns full; padded tokens never allowed.
    """
    rows = np.arange(lay.N) if rows is None else np.asarray(rows)
    cols = np.arange(lay.N) if cols is None else np.asarray(cols)
    kq, cq = lay.coords(rows)
    kk, ck = lay.coords(cols)
    ok = (kq != 1)[:, None] & (kk != 1)[None, :]
    text = (kq == 0)[:, None] | (kk == 0)[None, :]
    win = np.ones((len(rows), len(cols)), dtype=bool)
    for dim in range(3):
        st = window_start(cq[:, dim], lay.grid[dim], lay.window[dim], lay.stride[dim])
        c = ck[:, dim]
        win &= (c[None, :] >= st[:, None]) & (c[None, :] < st[:, None] + lay.window[dim])
    vid = (kq == 2)[:, None] & (kk == 2)[None, :]
    return ok & (text | (vid & win))


def _interval_overlap_count(q_lo, q_hi, k_lo, k_hi, L, k, s):
    """sum over i in [q_lo,q_hi) of |[start(i), start(i)+k) intersect [k_lo,k_hi)|."""
    i = np.arange(q_lo, q_hi)
    st = window_start(i, L, k, s)
    lo = np.maximum(st, k_lo)
    hi = np.minimum(st + k, k_hi)
    return int(np.maximum(hi - lo, 0).sum())


def gna_block_classes_separable(lay: GnaLayout):
    """uint8 [nB, nB] tile classes from per-dimension pair counts.

    The window is a product of per-dimension intervals, so the number of
    allowed (query, key) pairs between two tiles is the product of the
    one-dimensional counts; FULL needs that product to equal all real pairs
    and the KV tile to hold no padding.
    """
    nB = lay.ntb + lay.n_tiles
    out = np.zeros((nB, nB), dtype=np.uint8)
    # only a text block reaching past n_text holds padding slots
    text_pad = [(J + 1) * lay.bs > lay.n_text for J in range(lay.ntb)]
    tiles = [np.unravel_index(t, lay.tiles) for t in range(lay.n_tiles)]
    rng = []
    for tc in tiles:
        r = []
        for dim in range(3):
            lo = tc[dim] * lay.tile[dim]
            hi = min(lo + lay.tile[dim], lay.grid[dim])
            r.append((lo, hi))
        rng.append(r)
    padded_tile = [any(hi - lo < lay.tile[d] for d, (lo, hi) in enumerate(r)) for r in rng]
    for I in range(nB):
        for J in range(nB):
            if I < lay.ntb or J < lay.ntb:
                k_pad = text_pad[J] if J < lay.ntb else padded_tile[J - lay.ntb]
                out[I, J] = BLOCK_PARTIAL if k_pad else BLOCK_FULL
                continue
            rq, rk = rng[I - lay.ntb], rng[J - lay.ntb]
            allowed, total = 1, 1
            for dim in range(3):
                c = _interval_overlap_count(rq[dim][0], rq[dim][1], rk[dim][0], rk[dim][1],
                                            lay.grid[dim], lay.window[dim], lay.stride[dim])
                allowed *= c
                total *= (rq[dim][1] - rq[dim][0]) * (rk[dim][1] - rk[dim][0])
            if allowed == 0:
                out[I, J] = BLOCK_NONE
            elif allowed == total and not padded_tile[J - lay.ntb]:
                out[I, J] = BLOCK_FULL
            else:
                out[I, J] = BLOCK_PARTIAL
    return out


# ----------------------------------------------------------------------------
# generic classification and CSR


def classify_blocks(token_mask, bq, bk, q_valid=None, k_valid=None):
    """uint8 [nQB, nKB] classes of a dense token mask by counting pairs.

    Only real tokens count (``q_valid``/``k_valid``, default all). A KV block
    holding an invalid key can be FULL only if it has no allowed pair at all
    (then it is NONE); otherwise it is PARTIAL.
    """
    Nq, Nk = token_mask.shape
    q_valid = np.ones(Nq, bool) if q_valid is None else np.asarray(q_valid)
    k_valid = np.ones(Nk, bool) if k_valid is None else np.asarray(k_valid)
    nQB, nKB = n_blocks(Nq, bq), n_blocks(Nk, bk)
    out = np.zeros((nQB, nKB), dtype=np.uint8)
    for I in range(nQB):
        qs = slice(I * bq, min((I + 1) * bq, Nq))
        for J in range(nKB):
            ks = slice(J * bk, min((J + 1) * bk, Nk))
            sub = token_mask[qs, ks] & q_valid[qs][:, None] & k_valid[ks][None, :]
            n_ok = int(sub.sum())
            n_all = int(q_valid[qs].sum()) * (ks.stop - ks.start)
            if n_ok == 0:
                out[I, J] = BLOCK_NONE
            elif n_ok == n_all and bool(k_valid[ks].all()):
                out[I, J] = BLOCK_FULL
            else:
                out[I, J] = BLOCK_PARTIAL
    return out


def to_csr(classes, max_k=None):
    """(cnt [nQB], idx [nQB, max_k], flag [nQB, max_k]) in ascending KV order.

    idx is padded with -1 and flag with 0; flag holds the block class.
    """
    nQB, nKB = classes.shape
    max_k = nKB if max_k is None else max_k
    cnt = np.zeros(nQB, np.int32)
    idx = np.full((nQB, max_k), -1, np.int32)
    flag = np.zeros((nQB, max_k), np.uint8)
    for I in range(nQB):
        js = np.nonzero(classes[I])[0]
        cnt[I] = len(js)
        idx[I, :len(js)] = js
        flag[I, :len(js)] = classes[I, js]
    return cnt, idx, flag


def arrow_block_classes(N, n_text, bs, mode, window):
    """Arrow classes straight from the token mask (every kept block FULL)."""
    tm = arrow_token_mask(N, n_text, bs, mode, window)
    return classify_blocks(tm, bs, bs)


def arrow_block_classes_all(shape, head_mode, window):
    """uint8 [B, H, nQB, nKB] for a mode table shared across the batch."""
    out = np.zeros((shape.B, shape.H, shape.n_qb, shape.n_kb), np.uint8)
    for h in range(shape.H):
        c = arrow_block_classes(shape.N, shape.n_text, shape.block_q, int(head_mode[h]),
                                int(window[h]))
        out[:, h] = c
    return out


def gna_block_classes_all(B, H, lay: GnaLayout, head_mode=None):
    """uint8 [B, H, nB, nB]; FULL heads keep every block, SKIP heads none."""
    base = gna_block_classes_separable(lay)
    nB = base.shape[0]
    out = np.zeros((B, H, nB, nB), np.uint8)
    kvalid = np.array([bool(lay.valid(np.arange(J * lay.bs, (J + 1) * lay.bs)).all())
                       for J in range(nB)])
    full_row = np.where(kvalid, BLOCK_FULL, BLOCK_PARTIAL).astype(np.uint8)
    for h in range(H):
        m = HEAD_SPARSE if head_mode is None else int(head_mode[h])
        if m == HEAD_SPARSE:
            out[:, h] = base
        elif m == HEAD_FULL:
            out[:, h] = full_row[None, :]
    return out
