"""fp64 CPU oracle for block-sparse attention in diffusion transformers.

TEST INFRASTRUCTURE ONLY. Nothing in the library imports this package; only
the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
(and its ``--impl reference`` arm) may use it. It shares no code with the CUDA
path: the two meet only at the seeded inputs from ``workloads``.

Each function states, in its docstring, the passage it follows (page title and
section). Everything is written as the plain definition: token-level masks,
rank-and-cut selection by a full sort, row-wise softmax attention in fp64.

Modules
-------
masks      arrow (DiTFastAttnV2) and GNA window+stride token predicates,
           tile classification (none / full / partial), CSR block lists.
select     mean-pooled Q/K block scoring with top-k (lmnt.cn BSA post) and
           the SparseD full-score avg-pooled isolated top-rho selection.
attention  masked softmax attention in fp64, per-head modes (full / sparse /
           skip with cached output), bf16 round-to-nearest-even.
permute    raster <-> tile-order token permutation with padding (GNA).

Parity status: every function here is pinned by tests under ``tests/`` that
do not reuse the function's own formula (brute force, closed forms, library
routines, invariants), except where a docstring says "parity unpinned".
"""
from . import masks, select, attention, permute  # noqa: F401
