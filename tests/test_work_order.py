"""The forward's grid order (longest first), as a host transcription.

fwd_kernel maps blockIdx.x onto a (b, h, query pair) item: every FULL head,
then pair 0 of every sparse head, then the other sparse pairs in chunks of
(b, head) units whose K and V fit in 32 MiB (pair by pair within a chunk),
then the SKIP heads. This file restates that formula (keep it in step with
map_item in csrc/forward.cu) and checks it is a bijection with the intended
order; the GPU parity tests check every output row of the kernel itself.
"""
import random

import pytest

FULL, SPARSE, SKIP = 0, 1, 2


def map_item(B, H, N, d, modes, k):
    nQP = (N + 255) // 256
    nF = sum(1 for m in modes if m == FULL)
    nK = sum(1 for m in modes if m == SKIP)
    nS = H - nF - nK
    perF, perS = B * nF * nQP, B * nS * nQP
    if k < perF:
        cls, pair, b, m = FULL, k % nQP, (k // nQP) // nF, (k // nQP) % nF
    elif k < perF + perS:
        r, units, cls = k - perF, B * nS, SPARSE
        if r < units:
            pair, u = 0, r
        else:
            r -= units
            np_ = nQP - 1
            fit = (32 << 20) // (4 * N * d)
            G = max(1, min(units, fit))
            c = r // (G * np_)
            gsz = min(G, units - c * G)
            rr = r - c * G * np_
            u, pair = c * G + rr % gsz, 1 + rr // gsz
        b, m = u // nS, u % nS
    else:
        r, cls = k - perF - perS, SKIP
        pair, b, m = r % nQP, (r // nQP) // nK, (r // nQP) % nK
    heads = [h for h in range(H) if (modes[h] == cls if cls != SPARSE else modes[h] not in (FULL, SKIP))]
    return b, heads[m], pair


def _check(B, H, N, d, modes):
    nQP = (N + 255) // 256
    items = [map_item(B, H, N, d, modes, k) for k in range(B * H * nQP)]
    assert len(set(items)) == len(items) == B * H * nQP
    cls = [FULL if modes[h] == FULL else SKIP if modes[h] == SKIP else SPARSE for (_, h, _) in items]
    # FULL items first, SKIP items last
    assert cls == sorted(cls, key=lambda c: {FULL: 0, SPARSE: 1, SKIP: 2}[c])
    # among sparse items, every pair-0 item comes before any other pair
    sp = [p for (_, h, p), c in zip(items, cls) if c == SPARSE]
    n0 = sum(1 for p in sp if p == 0)
    assert all(p == 0 for p in sp[:n0])


@pytest.mark.parametrize("B,H,N,d,counts", [
    (1, 2, 512, 64, (1, 1, 0)),        # tiny arrow
    (2, 24, 4352, 64, (10, 11, 3)),    # SD3-1024-like
    (1, 24, 16896, 128, (0, 24, 0)),   # FLUX-2048-like
    (1, 32, 32768, 128, (0, 32, 0)),   # SparseD-like DLM
    (1, 24, 61952, 128, (0, 24, 0)),   # GNA video (tile order)
])
def test_workload_orders(B, H, N, d, counts):
    modes = [FULL] * counts[0] + [SPARSE] * counts[1] + [SKIP] * counts[2]
    random.Random(H).shuffle(modes)
    _check(B, H, N, d, modes)


def test_random_orders():
    rng = random.Random(5)
    for _ in range(300):
        B, H = rng.randint(1, 3), rng.randint(1, 40)
        N, d = rng.choice([256, 300, 4352, 32768, 100000]), rng.choice([64, 128])
        modes = [rng.choice([FULL, SPARSE, SKIP, 7]) for _ in range(H)]
        _check(B, H, N, d, modes)
