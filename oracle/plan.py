"""Head-wise compression plan (fp64 oracle, test use only).

DiTFastAttnV2, "efficient compression plan search":

* The single-layer relative squared error of a compression method m is
  I(m) = sum (y_m - y_o)^2 / sum (y_o - mean(y_o))^2, where y_o is the
  layer's uncompressed attention output and y_m the output under m. The
  printed numerator subtracts mean(y_o); the reading taken here is the plain
  difference y_m - y_o (with mean(y_o) there, an exact method would not score
  0). It is taken per head: the sums run over that head's outputs for every
  batch item, token and channel.
* The plan picks one method per head to minimise latency under an RSE
  budget delta, with the per-head cap I(h, m) <= (c / n) * delta for n heads
  (c = 1.5 by default). Reading: the heads' errors add up,
  sum_h I(h, m_h) <= delta, and latency is the number of computed blocks.

This module holds the definitions only: `rse` is the formula, and
`plan_bruteforce` enumerates every assignment, so it is usable on tiny
cases only.
"""
from __future__ import annotations

import itertools

import numpy as np


def rse(y_m, y_o):
    """fp64 [H]: I(h) for outputs [B, H, N, d] (any float dtype).

    Also returns the numerator and denominator per head.
    """
    ym = np.asarray(y_m, dtype=np.float64)
    yo = np.asarray(y_o, dtype=np.float64)
    H = yo.shape[1]
    num = np.empty(H)
    den = np.empty(H)
    for h in range(H):
        a = ym[:, h]
        o = yo[:, h]
        num[h] = np.sum((a - o) ** 2)
        den[h] = np.sum((o - o.mean()) ** 2)
    return num / den, num, den


def feasible(rse_hm, choice, delta, c):
    """Does `choice` [H] meet the per-head caps and the total budget?"""
    rse_hm = np.asarray(rse_hm, dtype=np.float64)
    H = rse_hm.shape[0]
    vals = np.array([rse_hm[h, choice[h]] for h in range(H)])
    return bool(np.all(vals <= c * delta / H) and vals.sum() <= delta)


def plan_bruteforce(rse_hm, cost_hm, delta, c=1.5):
    """Minimum total cost over every assignment that meets the constraints.

    rse_hm, cost_hm: [H, M]. Returns (min_cost, one optimal choice [H]) or
    (None, None) when no assignment is feasible. Among optimal assignments the
    one with the least total error, then the lexicographically smallest, is
    returned (several can be optimal; only the cost is unique).
    """
    rse_hm = np.asarray(rse_hm, dtype=np.float64)
    cost_hm = np.asarray(cost_hm, dtype=np.int64)
    H, M = rse_hm.shape
    best = None
    for choice in itertools.product(range(M), repeat=H):
        if not feasible(rse_hm, choice, delta, c):
            continue
        key = (int(sum(cost_hm[h, choice[h]] for h in range(H))),
               float(sum(rse_hm[h, choice[h]] for h in range(H))), choice)
        if best is None or key < best:
            best = key
    if best is None:
        return None, None
    return best[0], np.array(best[2], dtype=np.int32)
