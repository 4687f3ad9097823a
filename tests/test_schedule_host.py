"""Host-only schedule routines of the library against the schedule oracle
(exact integer equality; no GPU)."""
import random

import pytest

from oracle import schedule as OSc


def _bsa():
    from block_sparse_attention_37_b200 import build
    build.build()
    import block_sparse_attention_37_b200 as bsa
    return bsa


def test_full_steps_and_actions_match_oracle():
    bsa = _bsa()
    for T in list(range(1, 40)) + [128, 1024]:
        for skip in (0, 1, 7, 20, 33, 50, 99, 100):
            n = bsa.schedule_full_steps(T, skip)
            assert n == OSc.n_full_steps(T, skip), (T, skip)
            for s in range(T):
                assert bsa.step_action(s, T, n) == OSc.step_action(s, T, n)
    assert bsa.STEP_FULL == OSc.FULL and bsa.STEP_SELECT == OSc.SELECT and bsa.STEP_REUSE == OSc.REUSE


def test_keep_pct_matches_oracle():
    bsa = _bsa()
    rng = random.Random(3)
    for _ in range(60):
        L, T = rng.randint(1, 40), rng.randint(1, 60)
        hi, lo = rng.randint(0, 100), rng.randint(0, 100)
        for l in range(0, L, max(1, L // 7)):
            for s in range(0, T, max(1, T // 9)):
                assert bsa.keep_pct(l, L, s, T, hi, lo) == OSc.keep_pct(l, L, s, T, hi, lo), (l, L, s, T, hi, lo)


def test_schedule_argument_checks():
    bsa = _bsa()
    for args in ((0, 20), (10, -1), (10, 101)):
        with pytest.raises(bsa.BsaError):
            bsa.schedule_full_steps(*args)
    for args in ((5, 5, 1), (-1, 5, 1), (0, 5, 6)):
        with pytest.raises(bsa.BsaError):
            bsa.step_action(*args)
    with pytest.raises(bsa.BsaError):
        bsa.keep_pct(3, 3, 0, 5, 30, 10)
