"""Content-driven block selection (fp64 oracle, test use only).

Two scorers, one selection rule.

* Pooled Q/K scoring: lmnt.cn BSA post, section 2.2 (mean-pool every block to
  one vector, score query block against key block, keep the top-k key
  blocks) and section 2.3 (image-to-image is selected; blocks touching text
  stay dense). The learnable projection of that post needs trained weights
  and is left out, so the score is the plain dot product of the block means.
* SparseD, "Isolated Selection": A is the softmax attention map, A' =
  avgpool(A, block_size), and each query block keeps the top rho% of the
  prefill key blocks and, separately, the top rho% of the generation key
  blocks: S_i = S_i^pre union S_i^gen.

Selection rule (readings): k = ceil(rho * n) in integers; candidates are
ranked by descending score with ties going to the lower block index; the kept
set is reported in ascending block order. The ranking decision is taken on
scores rounded to fp32, the precision the GPU path computes them in.
"""
from __future__ import annotations

import numpy as np

from .masks import BLOCK_FULL, n_blocks


def block_means(x, bs):
    """fp64 [nB, d]: mean over the real tokens of each block of x [N, d]."""
    x = np.asarray(x, dtype=np.float64)
    N = x.shape[0]
    nb = n_blocks(N, bs)
    out = np.zeros((nb, x.shape[1]))
    for I in range(nb):
        out[I] = x[I * bs:min((I + 1) * bs, N)].mean(axis=0)
    return out


def pooled_scores(q, k, bq, bk):
    """fp64 [nQB, nKB]: score(I, J) = mean(Q_I) . mean(K_J) (no scale)."""
    return block_means(q, bq) @ block_means(k, bk).T


def top_k_indices(scores, candidates, k):
    """The k candidates with the largest score, ties to the lower index.

    Implemented as a full sort on the key (-score, index); returned ascending.
    """
    cand = [int(c) for c in candidates]
    ranked = sorted(cand, key=lambda j: (-float(scores[j]), j))
    return sorted(ranked[:k])


def select_rows(scores, n_kb, groups, keep_text_blocks=0, full_rows=0):
    """uint8 classes [nQB, nKB] from a score matrix.

    ``groups``: (begin, end, k) ranges of key blocks, each cut separately.
    The first ``keep_text_blocks`` key blocks are always kept; the first
    ``full_rows`` query rows keep every block.
    """
    s32 = np.asarray(scores, dtype=np.float64).astype(np.float32)
    nqb = s32.shape[0]
    out = np.zeros((nqb, n_kb), np.uint8)
    for I in range(nqb):
        if I < full_rows:
            out[I, :] = BLOCK_FULL
            continue
        out[I, :keep_text_blocks] = BLOCK_FULL
        for (b, e, k) in groups:
            for J in top_k_indices(s32[I], range(b, e), min(k, e - b)):
                out[I, J] = BLOCK_FULL
    return out


def pooled_select(q, k, bq, bk, n_text, groups, keep_text):
    """Classes [nQB, nKB] for one (b, h) under pooled Q/K scoring."""
    N = q.shape[0]
    sc = pooled_scores(q, k, bq, bk)
    ntq = n_blocks(n_text, bq) if keep_text else 0
    ntk = n_blocks(n_text, bk) if keep_text else 0
    return select_rows(sc, n_blocks(N, bk), groups, keep_text_blocks=ntk, full_rows=ntq), sc


def avgpool_attention_rows(q, k, scale, bq, bk, I, bias=None):
    """fp64 [nKB]: row I of A' = avgpool(softmax(scale*Q K^T + bias), block).

    ``bias`` (optional, fp64 [nQB, nKB]) is a block-constant logit offset.
    Only query block I is materialised (SparseD chunks Q the same way).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    N = k.shape[0]
    nkb = n_blocks(N, bk)
    rows = q[I * bq:min((I + 1) * bq, q.shape[0])]
    z = scale * (rows @ k.T)
    if bias is not None:
        z = z + np.repeat(np.asarray(bias, np.float64)[I], bk)[:N][None, :]
    z = z - z.max(axis=1, keepdims=True)
    a = np.exp(z)
    a = a / a.sum(axis=1, keepdims=True)
    out = np.zeros(nkb)
    for J in range(nkb):
        blk = a[:, J * bk:min((J + 1) * bk, N)]
        out[J] = blk.mean()
    return out


def full_score_select(q, k, scale, bq, bk, groups, bias=None, rows=None):
    """(classes [len(rows), nKB], A' rows) for one (b, h), SparseD selection."""
    N = q.shape[0]
    nqb = n_blocks(N, bq)
    rows = range(nqb) if rows is None else rows
    ap = np.stack([avgpool_attention_rows(q, k, scale, bq, bk, I, bias) for I in rows])
    return select_rows(ap, n_blocks(N, bk), groups), ap
