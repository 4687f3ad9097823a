"""bsa_plan_heads (host-only, no GPU) against the brute-force plan oracle.

The library solves the plan exactly with a dynamic program over the total
cost; the oracle enumerates every assignment. Several plans can be optimal,
so the test compares what is unique (the minimum cost, and the least total
error at that cost) and checks that the library's plan meets the
constraints.
"""
import numpy as np
import pytest

from oracle import plan as OP


def _bsa():
    from block_sparse_attention_37_b200 import build
    build.build()
    import block_sparse_attention_37_b200 as bsa
    return bsa


def _instance(rng, H, M):
    r = np.zeros((H, M))
    cost = np.zeros((H, M), dtype=np.int64)
    for h in range(H):
        r[h, 0] = 0.0  # method 0 is exact (full attention)
        r[h, 1:] = np.sort(rng.uniform(0.0, 0.4, M - 1))
        cost[h, 0] = 100
        cost[h, 1:] = np.sort(rng.integers(0, 100, M - 1))[::-1]  # cheaper methods err more
    return r, cost


@pytest.mark.parametrize("seed", range(40))
def test_plan_matches_bruteforce(seed):
    bsa = _bsa()
    rng = np.random.default_rng(seed)
    H, M = int(rng.integers(1, 6)), int(rng.integers(2, 5))
    r, cost = _instance(rng, H, M)
    delta = float(rng.uniform(0.0, 0.8))
    c = float(rng.choice([1.0, 1.5, 2.0, 10.0]))
    best, ch_o = OP.plan_bruteforce(r, cost, delta, c)
    assert best is not None  # the exact method always fits
    ch, total = bsa.plan_heads(r, cost, delta, c)
    assert total == best
    assert int(sum(cost[h, ch[h]] for h in range(H))) == best
    assert OP.feasible(r, ch, delta, c)
    err = sum(r[h, ch[h]] for h in range(H))
    err_o = sum(r[h, ch_o[h]] for h in range(H))
    assert err == pytest.approx(err_o, abs=1e-15)


def test_plan_cap_and_budget_by_hand():
    bsa = _bsa()
    r = np.array([[0.0, 0.5], [0.0, 0.2], [0.0, 0.2]])
    cost = np.array([[100, 0], [100, 50], [100, 50]])
    ch, total = bsa.plan_heads(r, cost, 0.6, 1.5)
    assert list(ch) == [0, 1, 1] and total == 200


def test_plan_infeasible_and_bad_arguments():
    bsa = _bsa()
    with pytest.raises(bsa.BsaError) as e:
        bsa.plan_heads(np.array([[0.5, 0.6]]), np.array([[1, 0]]), 0.1, 1.5)
    assert e.value.status == bsa.ERR_INFEASIBLE
    with pytest.raises(bsa.BsaError) as e:
        bsa.plan_heads(np.array([[0.0, 0.1]]), np.array([[1, -1]]), 0.1, 1.5)
    assert e.value.status == bsa.ERR_INVALID_ARG
    with pytest.raises(bsa.BsaError) as e:
        bsa.plan_heads(np.array([[0.0]]), np.array([[1]]), float("nan"), 1.5)
    assert e.value.status == bsa.ERR_INVALID_ARG
    with pytest.raises(bsa.BsaError) as e:  # tables too large: coarser cost units needed
        bsa.plan_heads(np.zeros((4, 2)), np.array([[1 << 27, 0]] * 4), 0.1, 1.5)
    assert e.value.status == bsa.ERR_UNSUPPORTED


def test_plan_at_c2_scale_is_feasible_and_locally_optimal():
    """24 heads x 5 methods with block-count costs: too large to enumerate;
    the plan meets the constraints and no single head can switch to a
    cheaper method without breaking them."""
    bsa = _bsa()
    rng = np.random.default_rng(7)
    H, M = 24, 5
    cost = np.array([[4624, 1084, 842, 718, 0]] * H, dtype=np.int64)  # full, arrow w=4/2/1, skip
    base = rng.uniform(0.002, 0.05, H)
    r = np.stack([np.zeros(H), base, 2 * base, 4 * base, rng.uniform(0.01, 0.2, H)], axis=1)
    for delta in (0.2, 0.6):
        ch, total = bsa.plan_heads(r, cost, delta, 1.5)
        assert OP.feasible(r, ch, delta, 1.5)
        assert total == int(sum(cost[h, ch[h]] for h in range(H)))
        for h in range(H):
            for m in range(M):
                if cost[h, m] < cost[h, ch[h]]:
                    alt = ch.copy()
                    alt[h] = m
                    assert not OP.feasible(r, alt, delta, 1.5)
