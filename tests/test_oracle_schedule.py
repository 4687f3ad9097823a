"""Pins for the step-schedule oracle (SparseD "overall framework" and
"sparse reuse"; GNA article image results; lmnt.cn BSA post section 3.3)."""
import numpy as np

from oracle import schedule as OSc


def test_sparsed_default_split():
    # 20% of 128 steps = 25.6 -> 26 full steps, selection at step 26
    n = OSc.n_full_steps(128, 20)
    assert n == 26
    acts = [OSc.step_action(s, 128, n) for s in range(128)]
    assert acts[:26] == [OSc.FULL] * 26 and acts[26] == OSc.SELECT
    assert acts[27:] == [OSc.REUSE] * 101
    assert OSc.n_full_steps(1024, 20) == 205  # 204.8
    assert OSc.n_full_steps(100, 20) == 20    # exact


def test_gna_split_nine_of_twenty_eight():
    acts = [OSc.step_action(s, 28, 9) for s in range(28)]
    assert acts.count(OSc.FULL) == 9 and acts[9] == OSc.SELECT and acts.count(OSc.REUSE) == 18


def test_no_skip_selects_first():
    assert OSc.step_action(0, 10, 0) == OSc.SELECT


def test_jaccard_closed_forms():
    j = OSc.jaccard_rows([[1, 2, 3], [], [0, 5], [4]], [[1, 2, 3], [], [5, 6, 7], [9]])
    assert np.allclose(j, [1.0, 1.0, 1 / 4, 0.0])


def test_keep_pct_ends_and_middle():
    assert OSc.keep_pct(0, 24, 0, 28, 30, 10) == 30     # shallow layer, first step
    assert OSc.keep_pct(23, 24, 27, 28, 30, 10) == 10   # deepest layer, last step
    assert OSc.keep_pct(23, 24, 0, 28, 30, 10) == 20    # halfway in the mean
    assert OSc.keep_pct(0, 1, 0, 1, 30, 10) == 30       # single layer and step
    # monotone non-increasing along layers and steps
    v = [[OSc.keep_pct(l, 12, s, 20, 30, 12) for s in range(20)] for l in range(12)]
    v = np.array(v)
    assert np.all(np.diff(v, axis=0) <= 0) and np.all(np.diff(v, axis=1) <= 0)
