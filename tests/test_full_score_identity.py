"""The identity the one-pass full-score selection computes A' by, checked in fp64 on the CPU.

The score kernel never holds a row of A. Per row i and 128-key tile t it keeps
x[i, t] = log2 sum_{j in t} 2^(z[i, j]) (z = scale * q.k + bias, in log2 units), carries the
row's LSE, lse_i = log2 sum_t 2^(x[i, t]), and at the end forms the block sums
sum_{i in I} sum_{t in J} 2^(x[i, t] - lse_i); the selection divides them by the block's real
query and key counts. Written here step by step in numpy, the result must equal the oracle's
avgpool(softmax) rows: the same quantity up to rounding, on ragged sizes, several tiles per
block, and a block-constant bias.
"""
import numpy as np
import pytest

from oracle import select as OS

LOG2E = 1.4426950408889634


def _one_pass_ap(q, k, scale, bs, bias=None):
    N = q.shape[0]
    nb = -(-N // bs)
    T = -(-N // 128)
    z = scale * (q @ k.T) * LOG2E                      # log2 units
    if bias is not None:
        z = z + (np.repeat(np.repeat(bias, bs, axis=0), bs, axis=1)[:N, :N] * LOG2E)
    x = np.full((N, T), -np.inf)
    for t in range(T):
        zt = z[:, 128 * t:min(128 * t + 128, N)]
        mx = zt.max(axis=1)
        x[:, t] = mx + np.log2(np.exp2(zt - mx[:, None]).sum(axis=1))
    m = x.max(axis=1)
    lse = m + np.log2(np.exp2(x - m[:, None]).sum(axis=1))
    tpk = bs // 128
    ap = np.zeros((nb, nb))
    for I in range(nb):
        rows = slice(I * bs, min(I * bs + bs, N))
        nq = rows.stop - rows.start
        for J in range(nb):
            ts = slice(J * tpk, min(J * tpk + tpk, T))
            nk = min(J * bs + bs, N) - J * bs
            ap[I, J] = np.exp2(x[rows, ts] - lse[rows, None]).sum() / (nq * nk)
    return ap


@pytest.mark.parametrize("N,bs,d,with_bias", [(128 * 5 + 37, 128, 64, False), (128 * 7, 128, 128, True),
                                              (256 * 3 + 90, 256, 64, True), (384 * 2 + 5, 384, 32, False)])
def test_tile_lse_pooling_equals_the_avgpooled_softmax(N, bs, d, with_bias):
    rng = np.random.default_rng(N + bs)
    q = rng.standard_normal((N, d)) * 1.5
    k = rng.standard_normal((N, d)) * 1.5
    nb = -(-N // bs)
    bias = rng.uniform(-2.0, 2.0, (nb, nb)) if with_bias else None
    scale = d ** -0.5
    got = _one_pass_ap(q, k, scale, bs, bias)
    _, exp = OS.full_score_select(q, k, scale, bs, bs, [(0, nb, 1)], bias=bias)
    np.testing.assert_allclose(got, exp, rtol=1e-12, atol=1e-300)
    # softmax rows sum to one: a row of A' weighted by its key blocks' sizes sums to one
    kcounts = np.array([min(J * bs + bs, N) - J * bs for J in range(nb)], dtype=float)
    np.testing.assert_allclose((got * kcounts[None, :]).sum(axis=1), 1.0, rtol=1e-12)
