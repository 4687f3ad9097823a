"""Shared helpers of the GPU parity tests: run the library, ask the oracle, compare."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

from oracle import attention as OA
from oracle import masks as OM
from oracle import select as OS

MAX_ABS = 2e-2   # spec tolerance for bf16 outputs
MEAN_ABS = 5e-3
TIE_REL = 1e-5   # selections: scores this close to the cut are ties


def bsa():
    import block_sparse_attention_37_b200 as m
    return m


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close_out(got: np.ndarray, exp: np.ndarray, what: str = ""):
    err = np.abs(got - exp)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def arrow_expected(q, k, v, shape, head_mode, window, b, h, rows=None, cache=None, bias=None):
    """Oracle output of one (b, h) for an arrow / full / skip head."""
    N = shape.N
    mode = int(head_mode[h])
    qn, kn, vn = f64(q[b, h]), f64(k[b, h]), f64(v[b, h])
    fn = lambda r: OM.arrow_token_mask(N, shape.n_text, shape.block_q, mode, int(window[h]), r)
    bfn = None if bias is None else OA.block_bias_fn(bias[h], shape.block_q, shape.block_k, N)
    c = None if cache is None else cache[b, h].numpy()
    return OA.head_forward(qn, kn, vn, mode, fn, 1.0 / np.sqrt(shape.d), rows=rows, bias_fn=bfn, cache=c)


def list_to_classes(blocks, nKB):
    """Decode a GPU block list into dense classes [B,H,nQB,nKB] (and check its invariants)."""
    cnt = blocks.cnt.cpu().numpy()
    idx = blocks.idx.cpu().numpy()
    flag = blocks.flag.cpu().numpy()
    B, H, nQB = cnt.shape
    out = np.zeros((B, H, nQB, nKB), np.uint8)
    for b in range(B):
        for h in range(H):
            for I in range(nQB):
                n = int(cnt[b, h, I])
                js = idx[b, h, I, :n]
                assert np.all(np.diff(js) > 0), "idx must be strictly ascending"
                assert np.all(idx[b, h, I, n:] == -1) and np.all(flag[b, h, I, n:] == 0)
                out[b, h, I, js] = flag[b, h, I, :n]
    return out


def selection_matches(got_row: np.ndarray, scores: np.ndarray, groups, fixed_keep: np.ndarray):
    """True iff a GPU selection row agrees with the oracle's scores outside near-ties.

    got_row: bool [nKB]; scores: fp64 [nKB]; fixed_keep: bool [nKB] blocks kept regardless.
    Returns (ok, n_ambiguous)."""
    amb_total = 0
    rest = got_row.copy()
    rest[fixed_keep] = False
    for (b, e, k) in groups:
        k = min(k, e - b)
        cand = np.arange(b, e)
        s = scores[b:e]
        g = got_row[b:e]
        if int(g.sum()) != k:
            return False, amb_total
        order = sorted(range(len(cand)), key=lambda i: (-s[i], cand[i]))
        exp = np.zeros(len(cand), bool)
        exp[order[:k]] = True
        amb = np.zeros(len(cand), bool)
        if 0 < k < len(cand):
            sk, sk1 = s[order[k - 1]], s[order[k]]
            tol = TIE_REL * max(abs(sk), abs(sk1))
            if sk - sk1 <= tol:
                amb = (np.abs(s - sk) <= tol) | (np.abs(s - sk1) <= tol)
        amb_total += int(amb.sum())
        if np.any(g[~amb] != exp[~amb]):
            return False, amb_total
        rest[b:e] = False
    return (not rest.any()), amb_total


def oracle_workers() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def full_score_rows(q, k, scale, bq, bk, rows, bias=None):
    """fp64 [len(rows), nKB]: the oracle's A' rows for the given query blocks of one (b, h).

    The rows are independent, so they are spread over a thread pool (numpy releases the GIL in
    its matmul and exp); each row is the oracle's own avgpool_attention_rows."""
    rows = [int(I) for I in rows]
    with ThreadPoolExecutor(oracle_workers()) as ex:
        out = list(ex.map(lambda I: OS.avgpool_attention_rows(q, k, scale, bq, bk, I, bias), rows))
    return np.stack(out)


def check_full_score_rows(cls_bh, q, k, scale, bq, bk, groups, rows, bias=None):
    """Every listed query-block row of a GPU full-score selection of one (b, h) agrees with the
    oracle's A' outside near-ties. Returns the oracle's A' rows."""
    ap = full_score_rows(q, k, scale, bq, bk, rows, bias)
    nkb = cls_bh.shape[-1]
    for r, I in enumerate(rows):
        ok, _ = selection_matches(cls_bh[I] > 0, ap[r], groups, np.zeros(nkb, bool))
        assert ok, f"query block {I}"
    return ap


def check_pooled_rows(cls_bh, q, k, bq, bk, n_text, groups, rows):
    """Every listed query-block row of a GPU pooled selection of one (b, h) agrees with the
    oracle's pooled scores (text rows full, text key blocks kept, groups cut outside near-ties)."""
    sc = OS.pooled_scores(q, k, bq, bk)
    ntq, ntk = -(-n_text // bq), -(-n_text // bk)
    nkb = cls_bh.shape[-1]
    for I in rows:
        row = cls_bh[I] > 0
        if I < ntq:
            assert row.all(), f"text query block {I} must be full"
            continue
        fixed = np.zeros(nkb, bool)
        fixed[:ntk] = True
        assert row[:ntk].all(), f"query block {I} must keep the text key blocks"
        ok, _ = selection_matches(row, sc[I], groups, fixed)
        assert ok, f"query block {I}"
