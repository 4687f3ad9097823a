"""Host-side index arithmetic of the one-pass full-score selection, on the CPU.

The one-pass form writes, per 128-row query tile, a [T][128] slab of per-tile row LSEs and a
partial row of A', and runs over the query blocks in chunks that the workspace holds. These tests
mirror the library's chunk sizes (the reported workspace size pins the mirror to the library)
and walk every index the score kernel (KIND_TLSE) and the selection kernels form for each chunk:
every (b, h, query tile) is computed exactly once, every slab access stays inside the chunk's
slabs and reads what the same row wrote, every partial row of A' is written exactly once, and the
selection reads exactly the partial rows of its query block that were written.
"""
import pytest

import block_sparse_attention_37_b200 as bsa

CAP = 1 << 30
MIN_CTAS = 1024
STATIC = 16 << 20


def cdiv(a, b):
    return -(-a // b)


def a256(x):
    return (x + 255) & ~255


def geom(B, H, N, bs):
    nqb = cdiv(N, bs)
    units = B * H * nqb
    m = bs // 128
    T = cdiv(N, 128)
    unit_bytes = m * T * 128 * 4
    return units, m, T, unit_bytes, min(units, cdiv(MIN_CTAS, m))


def apool_bytes(B, H, N, bs):
    units, m, _, _, _ = geom(B, H, N, bs)
    return a256(units * m * cdiv(N, bs) * 4)  # block_q / 128 partial rows per query block


def reported(B, H, N, bs):
    units, m, T, ub, mn = geom(B, H, N, bs)
    chunk = min(units, max(max(1, CAP // ub), mn))
    return apool_bytes(B, H, N, bs) + chunk * ub, chunk


def for_bytes(B, H, N, bs, nbytes):
    """(form, chunk, total) of the layout a workspace of nbytes runs."""
    units, m, T, ub, mn = geom(B, H, N, bs)
    nqb = cdiv(N, bs)
    base = apool_bytes(B, H, N, bs)
    if nbytes > base:
        chunk = min(units, (nbytes - base) // ub)
        if chunk >= mn:
            return "one", chunk, base + chunk * ub
    return "two", 0, a256(B * H * N * 4) + a256(B * H * nqb * nqb * 4)


CASES = [(1, 3, 128 * 12 + 30, 128), (1, 32, 32768, 128), (2, 3, 256 * 5 + 70, 256), (1, 2, 384 * 3 + 200, 384),
         (1, 128, 2048, 128), (1, 8, 16384, 128), (1, 64, 131072, 128), (1, 4, 131072, 1024)]


@pytest.mark.parametrize("B,H,N,bs", CASES)
def test_reported_size_matches_the_library(B, H, N, bs):
    dm = bsa.dims(B, H, N, 128, bs, bs, 0)
    nkb = cdiv(N, bs)
    sp = bsa.select_spec(bsa.SELECT_FULL_SCORE, [(0, nkb, 1)], False, 0.1)
    total, chunk = reported(B, H, N, bs)
    assert bsa.select_workspace_size(dm, sp) == total
    # the reported size always runs the one-pass form, its slabs bounded by the cap or one chunk's minimum
    form, c, t = for_bytes(B, H, N, bs, total)
    assert form == "one" and c == chunk and t == total
    units, m, T, ub, mn = geom(B, H, N, bs)
    assert chunk * ub <= max(CAP, mn * ub)


def _walk(B, H, N, bs, chunk):
    """Emulate every chunk's launch; return the multiset of computed (bh, qt) and partial rows."""
    units, m, T, ub, _ = geom(B, H, N, bs)
    nqb, nqt, nkb = cdiv(N, bs), cdiv(N, 128), cdiv(N, bs)
    slab_floats = chunk * ub // 4
    computed, written = {}, {}
    u0 = 0
    while u0 < units:
        n = min(chunk, units - u0)
        # score kernel, KIND_TLSE: grid n * m
        for c in range(n * m):
            u = u0 + c // m
            bh, qt = u // nqb, (u % nqb) * m + c % m
            if qt >= nqt:
                continue  # the CTA returns before any setup
            assert 0 <= bh < B * H
            computed[(bh, qt)] = computed.get((bh, qt), 0) + 1
            for t in (0, T - 1):
                for r in (0, 127):
                    if qt * 128 + r < N:
                        off = c * T * 128 + t * 128 + r  # written, then read back by row r alone
                        assert 0 <= off < slab_floats
            prow = u0 * m + c  # the CTA's partial row of A'
            assert prow == u * m + c % m
            assert (prow + 1) * nkb <= units * m * nkb
            written[prow] = written.get(prow, 0) + 1
        u0 += n
    # selection: query block row = bh * nqb + I reads its partial rows row * m + j, j < np
    for row in range(B * H * nqb):
        I = row % nqb
        np_ = min(m, nqt - I * m)
        assert np_ >= 1
        for j in range(np_):
            assert written.get(row * m + j) == 1, (row, j)
    return computed, written


@pytest.mark.parametrize("B,H,N,bs", CASES[:6])
@pytest.mark.parametrize("which", ["reported", "static", "small"])
def test_chunks_cover_every_tile_once(B, H, N, bs, which):
    units, m, T, ub, mn = geom(B, H, N, bs)
    if which == "reported":
        chunk = reported(B, H, N, bs)[1]
    elif which == "static":
        form, chunk, total = for_bytes(B, H, N, bs, STATIC)
        if form != "one":
            pytest.skip("two-pass form in the static scratch")
        assert total <= STATIC
    else:
        chunk = max(1, units // 3)  # more chunks than either entry point uses, with a ragged last one
    computed, written = _walk(B, H, N, bs, chunk)
    nqb, nqt = cdiv(N, bs), cdiv(N, 128)
    assert set(computed) == {(bh, qt) for bh in range(B * H) for qt in range(nqt)}
    assert set(computed.values()) == {1}
    assert len(written) == B * H * nqt and set(written.values()) == {1}


def test_static_scratch_forms():
    # the static entry runs the one-pass form in two chunks here ...
    form, chunk, _ = for_bytes(1, 128, 2048, 128, STATIC)
    assert form == "one" and 0 < 2048 - chunk < chunk
    # ... the two-pass form here, as for the 32-head 32k DLM workload ...
    assert for_bytes(1, 8, 16384, 128, STATIC)[0] == "two"
    assert for_bytes(1, 32, 32768, 128, STATIC)[0] == "two"
    # ... and neither fits at 64 heads x 32k (the request is refused)
    assert for_bytes(1, 64, 32768, 128, STATIC)[2] > STATIC
