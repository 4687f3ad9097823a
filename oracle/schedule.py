"""Step schedule of the sparse path (plain Python oracle, test use only).

* SparseD, "overall framework": the first T x skip% denoising steps run full
  attention; at that step the head-specific pattern M_S is selected once
  (full scores, block pooling, isolated top-rho%), and every later step
  reuses it. The GNA article's image results use the same split with a
  step count (full attention for the first 9 of 28 steps, GNA after).
  Reading: the number of full steps is ceil(T * skip / 100) in integers,
  "the first skip% of the steps" taken as at least that share.
* SparseD, "sparse reuse": the stability of M_S is the Jaccard similarity
  |A n B| / |A u B| of the block sets selected for the same query-block row,
  averaged over rows and heads. Reading: two empty rows are identical (1).
* lmnt.cn BSA post, section 3.3: shallow layers and early steps keep more
  blocks (about 30%), deep layers and late steps fewer (10-15%). The post
  gives no formula; reading: the kept percentage falls linearly from `hi` to
  `lo` with the mean of the layer fraction l / (L - 1) and the step fraction
  s / (T - 1) (a fraction is 0 when there is a single layer or step),
  rounded to the nearest integer percent, halves up.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

FULL, SELECT, REUSE = 0, 1, 2


def n_full_steps(n_steps: int, skip_pct: int) -> int:
    """ceil(T * skip / 100): the full-attention steps before selection."""
    return -(-n_steps * skip_pct // 100)


def step_action(step: int, n_steps: int, n_full: int) -> int:
    """FULL before the selection step, SELECT at it, REUSE after it."""
    if step < n_full:
        return FULL
    return SELECT if step == n_full else REUSE


def jaccard_rows(a_sets, b_sets):
    """Per-row Jaccard similarity of two lists of block-index sets."""
    out = []
    for a, b in zip(a_sets, b_sets):
        a, b = set(a), set(b)
        out.append(1.0 if not a and not b else len(a & b) / len(a | b))
    return np.array(out)


def keep_pct(layer: int, n_layers: int, step: int, n_steps: int, hi: int, lo: int) -> int:
    """The kept percentage for (layer, step), exact rational arithmetic."""
    fl = Fraction(layer, n_layers - 1) if n_layers > 1 else Fraction(0)
    fs = Fraction(step, n_steps - 1) if n_steps > 1 else Fraction(0)
    v = Fraction(hi) - (Fraction(hi) - Fraction(lo)) * (fl + fs) / 2
    return int(v + Fraction(1, 2)) if v >= 0 else -int(-v + Fraction(1, 2))
