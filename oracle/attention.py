"""Masked softmax attention in fp64 (oracle, test use only).

The block-sparse forward is exact masked attention, not an approximation:
lmnt.cn BSA post, section 3.1 (FlashAttention-style tiles with online softmax
over the selected blocks only), DiTFastAttnV2 "Fused Kernel" (per head: full,
arrow, or skip with the cached output of the previous step), jsqmd.com GNA
article section 2.1 (fine mask only on partially covered tiles).

So the oracle is the plain definition, row by row:

    z_ij = scale * q_i . k_j + bias(i, j)       for allowed j
    p_ij = exp(z_ij - max_j z_ij) / sum_j exp(z_ij - max_j z_ij)
    o_i  = sum_j p_ij v_j

A row with no allowed key gives o_i = 0 (reading: empty rows are zero).
SKIP heads return the caller's fp32 cache rounded to bf16 (round to nearest,
ties to even).
"""
from __future__ import annotations

import numpy as np

from .masks import HEAD_SKIP


def bf16_round(x):
    """Round fp32 values to the nearest bf16 (ties to even), returned as fp64.

    Written from the IEEE-754 definition on the fp32 bit pattern: keep the top
    16 bits, rounding on the 16 dropped bits with ties to even. NaN is kept
    quiet.
    """
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    nan = np.isnan(f)
    r = np.where(nan, (u.astype(np.uint32) | 0x00400000) & 0xFFFF0000, r).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


def masked_attention_rows(q, k, v, allowed, scale, bias=None):
    """fp64 [R, d] outputs for R query rows.

    q [R, d], k [N, d], v [N, d], allowed bool [R, N], bias None or [R, N].
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    z = scale * (q @ k.T)
    if bias is not None:
        z = z + bias
    z = np.where(allowed, z, -np.inf)
    m = z.max(axis=1, keepdims=True)
    empty = ~np.isfinite(m[:, 0])
    m = np.where(np.isfinite(m), m, 0.0)
    p = np.exp(z - m)
    s = p.sum(axis=1, keepdims=True)
    s = np.where(s > 0, s, 1.0)
    o = (p / s) @ v
    o[empty] = 0.0
    return o


def attention_probs_rows(q, k, allowed, scale, bias=None):
    """fp64 [R, N] softmax probabilities of the allowed keys (0 elsewhere)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    z = scale * (q @ k.T)
    if bias is not None:
        z = z + bias
    z = np.where(allowed, z, -np.inf)
    m = z.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    p = np.exp(z - m)
    s = p.sum(axis=1, keepdims=True)
    return p / np.where(s > 0, s, 1.0)


def head_forward(q, k, v, mode, allowed_fn, scale, rows=None, bias_fn=None, cache=None,
                 chunk=1024):
    """fp64 [len(rows), d] output of one (b, h).

    allowed_fn(rows) -> bool [len(rows), N]; bias_fn(rows) -> [len(rows), N].
    """
    N = k.shape[0]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    if mode == HEAD_SKIP:
        return bf16_round(np.asarray(cache, np.float32)[rows])
    out = np.zeros((len(rows), v.shape[1]))
    for c0 in range(0, len(rows), chunk):
        r = rows[c0:c0 + chunk]
        b = None if bias_fn is None else bias_fn(r)
        out[c0:c0 + len(r)] = masked_attention_rows(np.asarray(q)[r], k, v, allowed_fn(r), scale, b)
    return out


def block_mask_to_token_fn(classes_bh, bq, bk, N, fine_fn=None):
    """allowed_fn from block classes: FULL blocks allowed, PARTIAL via fine_fn.

    Used for selected-block masks (pooled / full-score selection), where the
    token-level mask is by definition the union of the kept blocks.
    """
    cls = np.asarray(classes_bh)

    def fn(rows):
        rows = np.asarray(rows)
        c = cls[rows // bq][:, np.arange(N) // bk]
        out = c == 1
        if fine_fn is not None and (c == 2).any():
            out |= (c == 2) & fine_fn(rows)
        return out
    return fn


def block_bias_fn(bias_h, bq, bk, N):
    """bias_fn for a block-constant logit offset table [nQB, nKB]."""
    b = np.asarray(bias_h, np.float64)

    def fn(rows):
        rows = np.asarray(rows)
        return b[rows // bq][:, np.arange(N) // bk]
    return fn
