"""Pins for the plan oracle (DiTFastAttnV2, "efficient compression plan search").

The RSE pins are closed forms of the definition; the plan pins are small
cases whose optimum follows by hand.
"""
import numpy as np
import pytest

from oracle import plan as OP


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_rse_exact_method_scores_zero():
    y = _rand((2, 3, 17, 8), 1)
    i, num, den = OP.rse(y, y)
    assert np.all(i == 0.0) and np.all(num == 0.0) and np.all(den > 0)


def test_rse_predicting_the_mean_scores_one():
    y = _rand((2, 3, 17, 8), 2)
    ym = np.broadcast_to(y.mean(axis=(0, 2, 3), keepdims=True), y.shape)
    i, _, _ = OP.rse(ym, y)
    assert np.allclose(i, 1.0, rtol=1e-12)


@pytest.mark.parametrize("k", [0.5, 2.0, -3.0])
def test_rse_scaled_deviation_scores_k_squared(k):
    # y_m = y_o + k (y_o - mean): error sum = k^2 * variance sum
    y = _rand((1, 4, 33, 16), 3)
    mu = y.mean(axis=(0, 2, 3), keepdims=True)
    i, _, _ = OP.rse(y + k * (y - mu), y)
    assert np.allclose(i, k * k, rtol=1e-12)


def test_rse_is_per_head():
    y = _rand((2, 2, 9, 4), 4)
    ym = y.copy()
    ym[:, 1] += 1.0  # only head 1 changes
    i, num, den = OP.rse(ym, y)
    assert i[0] == 0.0
    assert np.isclose(num[1], 2 * 9 * 4)  # B * N * d unit errors
    assert np.isclose(den[1], np.sum((y[:, 1] - y[:, 1].mean()) ** 2))


def test_plan_all_full_when_budget_is_zero():
    r = np.array([[0.0, 0.1, 0.3]] * 3)
    cost = np.array([[100, 40, 0]] * 3)
    c, ch = OP.plan_bruteforce(r, cost, delta=0.0)
    assert c == 300 and list(ch) == [0, 0, 0]


def test_plan_cap_limits_one_head():
    # one head could take all the budget by itself; the cap c*delta/n stops it
    r = np.array([[0.0, 0.5], [0.0, 0.2], [0.0, 0.2]])
    cost = np.array([[100, 0], [100, 50], [100, 50]])
    delta = 0.6  # cap = 1.5 * 0.6 / 3 = 0.3: head 0's 0.5 is out
    c, ch = OP.plan_bruteforce(r, cost, delta)
    assert c == 200 and list(ch) == [0, 1, 1]
    # without a binding cap (c large) head 0 alone is the cheapest way down
    c2, ch2 = OP.plan_bruteforce(r, cost, delta, c=10.0)
    assert c2 == 200 and OP.feasible(r, ch2, delta, 10.0)
    c3, _ = OP.plan_bruteforce(r, cost, 0.9, c=10.0)
    assert c3 == 100  # 0.5 + 0.2 + 0.2 = 0.9 fits: costs 0 + 50 + 50


def test_plan_prefers_cheaper_at_equal_budget():
    r = np.array([[0.0, 0.1, 0.1], [0.0, 0.1, 0.1]])
    cost = np.array([[10, 7, 5], [10, 7, 5]])
    c, ch = OP.plan_bruteforce(r, cost, delta=0.2)
    assert c == 10 and list(ch) == [2, 2]


def test_plan_infeasible_without_an_exact_method():
    r = np.array([[0.5, 0.6]])
    cost = np.array([[1, 0]])
    assert OP.plan_bruteforce(r, cost, delta=0.1) == (None, None)
