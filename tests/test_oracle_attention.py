"""Pins for oracle.attention: independent library routines, closed forms, invariants."""
import numpy as np
import pytest
import torch

from oracle import attention as A


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, mask=None, scale=None, float_mask=None):
    """torch's fp64 CPU scaled_dot_product_attention as an independent routine."""
    tq, tk, tv = (torch.from_numpy(np.asarray(x, np.float64))[None, None] for x in (q, k, v))
    am = None
    if mask is not None:
        am = torch.from_numpy(mask)[None, None]
    if float_mask is not None:
        am = torch.from_numpy(float_mask)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=am, scale=scale)
    return o[0, 0].numpy()


@pytest.mark.parametrize("N,d", [(17, 8), (64, 16), (130, 32)])
def test_dense_matches_library_sdpa(N, d):
    q, k, v = _rand((N, d), 1), _rand((N, d), 2), _rand((N, d), 3)
    allowed = np.ones((N, N), bool)
    o = A.masked_attention_rows(q, k, v, allowed, 1 / np.sqrt(d))
    np.testing.assert_allclose(o, _sdpa(q, k, v), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_mask_matches_library_sdpa(seed):
    N, d = 96, 16
    rng = np.random.default_rng(seed)
    q, k, v = rng.standard_normal((3, N, d))
    allowed = rng.random((N, N)) < 0.3
    allowed[np.arange(N), rng.integers(0, N, N)] = True  # every row non-empty
    o = A.masked_attention_rows(q, k, v, allowed, 0.37)
    np.testing.assert_allclose(o, _sdpa(q, k, v, mask=allowed, scale=0.37), rtol=1e-12, atol=1e-12)


def test_bias_matches_library_float_mask():
    N, d = 48, 8
    rng = np.random.default_rng(5)
    q, k, v = rng.standard_normal((3, N, d))
    bias = rng.standard_normal((N, N))
    allowed = np.ones((N, N), bool)
    o = A.masked_attention_rows(q, k, v, allowed, 0.5, bias)
    np.testing.assert_allclose(o, _sdpa(q, k, v, scale=0.5, float_mask=bias), rtol=1e-12, atol=1e-12)


def test_row_constant_bias_is_invariant():
    N, d = 40, 8
    rng = np.random.default_rng(6)
    q, k, v = rng.standard_normal((3, N, d))
    allowed = rng.random((N, N)) < 0.5
    allowed[:, 0] = True
    b = np.repeat(rng.standard_normal((N, 1)) * 5, N, axis=1)
    np.testing.assert_allclose(A.masked_attention_rows(q, k, v, allowed, 0.3, b),
                               A.masked_attention_rows(q, k, v, allowed, 0.3), rtol=1e-12, atol=1e-12)


def test_constant_v_gives_constant_output():
    N, d = 70, 8
    rng = np.random.default_rng(7)
    q, k = rng.standard_normal((2, N, d))
    v = np.full((N, d), 2.5)
    allowed = rng.random((N, N)) < 0.2
    allowed[:, -1] = True
    o = A.masked_attention_rows(q, k, v, allowed, 1.0)
    np.testing.assert_allclose(o, 2.5, rtol=0, atol=1e-13)


def test_zero_q_gives_mean_of_allowed_values():
    N, d = 50, 6
    rng = np.random.default_rng(8)
    k, v = rng.standard_normal((2, N, d))
    q = np.zeros((N, d))
    allowed = rng.random((N, N)) < 0.4
    allowed[:, 3] = True
    o = A.masked_attention_rows(q, k, v, allowed, 1.0)
    expect = np.stack([v[allowed[i]].mean(axis=0) for i in range(N)])
    np.testing.assert_allclose(o, expect, rtol=1e-12, atol=1e-13)


def test_one_hot_v_recovers_probabilities_and_rows_sum_to_one():
    N = 24
    rng = np.random.default_rng(9)
    q, k = rng.standard_normal((2, N, 5))
    v = np.eye(N)
    allowed = rng.random((N, N)) < 0.6
    allowed[:, 0] = True
    p = A.masked_attention_rows(q, k, v, allowed, 0.8)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(p[~allowed] == 0)
    np.testing.assert_allclose(p, A.attention_probs_rows(q, k, allowed, 0.8), rtol=1e-12, atol=1e-14)


def test_block_diagonal_equals_independent_blocks():
    N, d, bs = 96, 8, 32
    rng = np.random.default_rng(10)
    q, k, v = rng.standard_normal((3, N, d))
    blk = np.arange(N) // bs
    allowed = blk[:, None] == blk[None, :]
    o = A.masked_attention_rows(q, k, v, allowed, 0.25)
    for b in range(N // bs):
        s = slice(b * bs, (b + 1) * bs)
        np.testing.assert_allclose(o[s], _sdpa(q[s], k[s], v[s], scale=0.25), rtol=1e-12, atol=1e-12)


def test_empty_row_is_zero():
    N, d = 10, 4
    rng = np.random.default_rng(11)
    q, k, v = rng.standard_normal((3, N, d))
    allowed = np.ones((N, N), bool)
    allowed[3] = False
    o = A.masked_attention_rows(q, k, v, allowed, 1.0)
    assert np.all(o[3] == 0)
    assert np.all(np.isfinite(o))


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(12)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 10,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0, 3.4e38,
                                  1e-40, -1e-40, np.inf, -np.inf], np.float32)])
    # exact ties: mantissa tail 0x8000 with even and odd kept bit
    ties = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x40408000], np.uint32).view(np.float32)
    x = np.concatenate([x, ties])
    ours = A.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_skip_head_returns_rounded_cache():
    N, d = 12, 4
    cache = np.random.default_rng(13).standard_normal((N, d)).astype(np.float32)
    o = A.head_forward(np.zeros((N, d)), np.zeros((N, d)), np.zeros((N, d)), 2, None, 1.0,
                       cache=cache)
    ref = torch.from_numpy(cache).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(o, ref)
