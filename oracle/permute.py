"""Raster <-> tile-order token permutation (fp64 oracle, test use only).

jsqmd.com GNA article, section 2.2: tokens are permuted from raster order into
tile order before the kernel and back afterwards; the planned dedicated kernel
fuses the permutation with padding. The layout is the one of
``masks.GnaLayout``: text first, zero padding up to a block multiple, then the
tiles of the (padded) grid in raster order, each tile's tokens in raster order.
"""
from __future__ import annotations

import numpy as np

from .masks import GnaLayout


def tile_order_source(lay: GnaLayout):
    """int64 [lay.N]: raster position feeding each tile-order slot, -1 = padding."""
    src = np.full(lay.N, -1, dtype=np.int64)
    src[:lay.n_text] = np.arange(lay.n_text)
    kind, c = lay.coords(np.arange(lay.text_span, lay.N))
    L = lay.grid
    raster = lay.n_text + (c[:, 0] * L[1] + c[:, 1]) * L[2] + c[:, 2]
    src[lay.text_span:] = np.where(kind == 2, raster, -1)
    return src


def permute_to_tiles(x, lay: GnaLayout):
    """x [..., n_text + prod(grid), d] raster -> [..., lay.N, d] tile order, zero padded."""
    x = np.asarray(x)
    src = tile_order_source(lay)
    out = np.zeros(x.shape[:-2] + (lay.N, x.shape[-1]), dtype=x.dtype)
    ok = src >= 0
    out[..., ok, :] = x[..., src[ok], :]
    return out


def unpermute_from_tiles(y, lay: GnaLayout):
    """Inverse of ``permute_to_tiles`` (padding slots are dropped)."""
    y = np.asarray(y)
    src = tile_order_source(lay)
    n_raster = lay.n_text + int(np.prod(lay.grid))
    out = np.zeros(y.shape[:-2] + (n_raster, y.shape[-1]), dtype=y.dtype)
    ok = src >= 0
    out[..., src[ok], :] = y[..., ok, :]
    return out
