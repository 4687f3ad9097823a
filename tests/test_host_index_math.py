"""The kernels' GNA index arithmetic, compiled for the host from the library's own
sources, against the oracle (no GPU).

The forward's fine mask of a PARTIAL tile (gna_query_window + gna_segment_bits),
the mask builder's tile classes (gna_class) and the permutation's row map
(tile_source_row) are host-callable functions of csrc/. A small harness that
includes the library's single translation unit exposes them; every bit, class
and row index must equal what the oracle's token-level GNA mask, its block
classes and its tile order give.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import masks as OM
from oracle import permute as OP

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_attention_37_b200", "csrc")

HARNESS = r'''
#include "bsa_lib.cu"
extern "C" int h_segbits_row(int n_text, const bsa_gna_geom* geom, int pq, unsigned long long* out, int nseg) {
  bsa::GnaDev g;
  const int st = bsa::make_gna(geom, n_text, &g);
  if (st) return st;
  const bsa::QWin q = bsa::gna_query_window(g, pq, true);
  for (int s = 0; s < nseg; ++s) out[s] = bsa::gna_segment_bits(g, s, q);
  return 0;
}
extern "C" int h_segbits_geo_row(int n_text, const bsa_gna_geom* geom, int pq, unsigned long long* out, int nseg) {
  bsa::GnaDev g;
  const int st = bsa::make_gna(geom, n_text, &g);
  if (st) return st;
  if (!g.seg_one_slice) return -1;
  const bsa::QBox b = bsa::gna_query_box(g, bsa::gna_query_window(g, pq, true));
  for (int s = 0; s < nseg; ++s) out[s] = bsa::gna_segment_bits_geo(g, s, bsa::gna_segment_geo(g, s), b);
  return 0;
}
extern "C" int h_gna_classes(int n_text, const bsa_gna_geom* geom, unsigned char* out, int nb) {
  bsa::GnaDev g;
  const int st = bsa::make_gna(geom, n_text, &g);
  if (st) return st;
  for (int I = 0; I < nb; ++I)
    for (int J = 0; J < nb; ++J) out[I * nb + J] = (unsigned char)bsa::gna_class(g, I, J);
  return 0;
}
extern "C" int h_group_meets(int n_text, const bsa_gna_geom* geom, unsigned char* out, int nseg) {
  bsa::GnaDev g;
  const int st = bsa::make_gna(geom, n_text, &g);
  if (st) return st;
  if (!g.seg_one_slice) return -1;
  for (int q = 0; q < nseg; ++q) {
    const bsa::GroupWin w = bsa::gna_group_window(g, q);
    for (int s = 0; s < nseg; ++s) out[q * nseg + s] = bsa::gna_segment_meets(g, bsa::gna_segment_geo(g, s), w);
  }
  return 0;
}
extern "C" void h_fdiv_many(int d, const int* n, long long* out, int count) {
  const bsa::FastDiv f = bsa::make_fastdiv(d);
  for (int i = 0; i < count; ++i) out[i] = bsa::fdiv(n[i], f);
}
extern "C" int h_tile_sources(int n_text, const bsa_gna_geom* geom, int* out, int n) {
  bsa::GnaDev g;
  const int st = bsa::make_gna(geom, n_text, &g);
  if (st) return st;
  for (int pos = 0; pos < n; ++pos) out[pos] = bsa::tile_source_row(g, pos);
  return 0;
}
'''


@pytest.fixture(scope="module")
def host_lib(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found: the harness is compiled from the library's CUDA sources")
    d = tmp_path_factory.mktemp("host_index_math")
    src = d / "harness.cu"
    src.write_text(HARNESS)
    so = d / "harness.so"
    cmd = [nvcc, "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-Xcompiler", "-fPIC",
           "-shared", "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-o", str(so), str(src)]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lib = ctypes.CDLL(str(so))
    lib.h_segbits_row.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int]
    lib.h_tile_sources.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.h_gna_classes.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.h_fdiv_many.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.h_segbits_geo_row.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int]
    lib.h_group_meets.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    return lib


def test_division_by_invariant_integers_is_exact(host_lib):
    """The fine mask divides by launch invariants with a multiply-high and a shift (Granlund and
    Montgomery, N = 31): exact floor division for every divisor up to 4096 over all dividends
    below 2^20, and for large dividends up to 2^31 - 1 (also with large divisors)."""
    rng = np.random.default_rng(0)
    dense = np.arange(0, 1 << 20, dtype=np.int32)
    big = np.concatenate([rng.integers(0, 2 ** 31 - 1, 20000),
                          np.arange(2 ** 31 - 2048, 2 ** 31, dtype=np.int64)]).astype(np.int32)
    out = np.empty(len(dense), dtype=np.int64)
    divisors = list(range(1, 4097)) + [65535, 65536, 100003, 1 << 20, (1 << 30) + 7, 2 ** 31 - 1]
    for d in divisors:
        for n in ((dense, big) if d <= 256 else (dense[::61], big)):
            n = np.ascontiguousarray(n)
            host_lib.h_fdiv_many(d, n.ctypes.data, out.ctypes.data, len(n))
            assert np.array_equal(out[:len(n)], n.astype(np.int64) // d), d


class Geom(ctypes.Structure):  # bsa_gna_geom
    _fields_ = [("ndim", ctypes.c_int32), ("grid", ctypes.c_int32 * 3), ("tile", ctypes.c_int32 * 3),
                ("window", ctypes.c_int32 * 3), ("stride", ctypes.c_int32 * 3)]


def _geom(grid, tile, window, stride):
    g = Geom()
    g.ndim = len(grid)
    for i in range(len(grid)):
        g.grid[i], g.tile[i], g.window[i], g.stride[i] = grid[i], tile[i], window[i], stride[i]
    return g


CASES = [
    (64, (4, 8, 16), (2, 4, 8), (3, 5, 7), (1, 1, 1)),        # partial tiles everywhere
    (50, (5, 9, 20), (2, 4, 8), (3, 5, 7), (1, 2, 2)),        # padding in the grid and the text
    (0, (300,), (64,), (97,), (5,)),                            # 1-D, padded last tile
    (128, (8, 256), (1, 128), (3, 48), (1, 16)),                # tile x extent wider than a segment
    (17, (6, 10, 12), (2, 2, 16), (4, 5, 6), (2, 1, 3)),        # mixed strides, ragged text
    (256, (16, 48, 80), (4, 8, 8), (8, 16, 24), (1, 1, 1)),     # the video workload, stride 1
    (256, (16, 48, 80), (4, 8, 8), (8, 16, 24), (4, 8, 8)),     # the video workload, stride 4x8x8
    (33, (3, 37, 21), (1, 16, 8), (2, 9, 11), (1, 2, 3)),       # segments in one t-slice, two per slice
    (0, (40, 50), (8, 8), (7, 9), (1, 1)),                      # 2-D, one segment per tile, padded y
    (128, (4, 12, 20), (2, 8, 8), (3, 9, 11), (1, 1, 1)),       # one-slice, padded y and x
    (128, (4, 12, 20), (2, 8, 8), (3, 9, 11), (1, 3, 2)),       # the same, strided
    (40, (3, 20, 10), (1, 16, 4), (3, 7, 5), (1, 2, 1)),        # one-slice, block 64, padded text
]


@pytest.mark.parametrize("n_text,grid,tile,window,stride", CASES)
def test_fine_mask_bits_equal_the_token_mask(host_lib, n_text, grid, tile, window, stride):
    lay = OM.GnaLayout(n_text, grid, tile, window, stride)
    g = _geom(grid, tile, window, stride)
    nseg = -(-lay.N // 64)
    rows = np.arange(lay.N)
    if lay.N > 4096:
        rows = np.sort(np.random.default_rng(lay.N).choice(lay.N, 256, replace=False))
    rows = rows[lay.valid(rows)]
    out = np.zeros(nseg, dtype=np.uint64)
    shifts = np.arange(64, dtype=np.uint64)
    for pq in rows:
        assert host_lib.h_segbits_row(n_text, ctypes.byref(g), int(pq), out.ctypes.data, nseg) == 0
        got = ((out[:, None] >> shifts[None, :]) & np.uint64(1)).astype(bool).reshape(-1)[:lay.N]
        exp = OM.gna_token_mask(lay, [int(pq)])[0]
        assert np.array_equal(got, exp), (grid, int(pq), np.nonzero(got != exp)[0][:5])


@pytest.mark.parametrize("n_text,grid,tile,window,stride", CASES)
def test_precomputed_geometry_bits_equal_the_token_mask(host_lib, n_text, grid, tile, window, stride):
    """The forward's fast path for layouts whose segments lie in one t-slice: the segment's grid
    position computed once (schedule build) and each query's clamped window once give the same
    bits as the token mask."""
    lay = OM.GnaLayout(n_text, grid, tile, window, stride)
    g = _geom(grid, tile, window, stride)
    nseg = -(-lay.N // 64)
    rows = np.arange(lay.N)
    if lay.N > 4096:
        rows = np.sort(np.random.default_rng(lay.N + 1).choice(lay.N, 256, replace=False))
    rows = rows[lay.valid(rows)]
    out = np.zeros(nseg, dtype=np.uint64)
    shifts = np.arange(64, dtype=np.uint64)
    for pq in rows:
        st = host_lib.h_segbits_geo_row(n_text, ctypes.byref(g), int(pq), out.ctypes.data, nseg)
        if st == -1:
            pytest.skip("segments span several t-slices: the forward keeps the general path")
        assert st == 0
        got = ((out[:, None] >> shifts[None, :]) & np.uint64(1)).astype(bool).reshape(-1)[:lay.N]
        exp = OM.gna_token_mask(lay, [int(pq)])[0]
        assert np.array_equal(got, exp), (grid, int(pq), np.nonzero(got != exp)[0][:5])


@pytest.mark.parametrize("n_text,grid,tile,window,stride", CASES)
def test_group_window_never_drops_a_visible_key(host_lib, n_text, grid, tile, window, stride):
    """The schedule leaves a partial key segment out of a 64-row query group when it misses the
    group's window (bounding box of its rows' windows). Wherever it does, the token mask of those
    64 rows and 64 keys must be all false; for the video workload the test finds every empty pair
    of an image group (the bound is tight for a box of rows)."""
    lay = OM.GnaLayout(n_text, grid, tile, window, stride)
    g = _geom(grid, tile, window, stride)
    nseg = -(-lay.N // 64)
    meets = np.zeros((nseg, nseg), dtype=np.uint8)
    st = host_lib.h_group_meets(n_text, ctypes.byref(g), meets.ctypes.data, nseg)
    if st == -1:
        pytest.skip("segments span several t-slices: the schedule is not narrowed")
    assert st == 0
    qs = np.arange(nseg)
    if nseg > 96:
        qs = np.sort(np.random.default_rng(nseg).choice(nseg, 96, replace=False))
    missed = dropped = 0
    for q in qs:
        rows = np.arange(64 * q, min(64 * q + 64, lay.N))
        tm = OM.gna_token_mask(lay, rows)
        seen = np.array([tm[:, 64 * s:64 * s + 64].any() for s in range(nseg)])
        assert not (seen & (meets[q] == 0)).any(), (q, np.nonzero(seen & (meets[q] == 0))[0][:5])
        dropped += int((meets[q] == 0).sum())
        if lay.valid(rows).all() and rows[0] >= lay.text_span:
            missed += int((~seen & (meets[q] == 1)).sum())
    if (n_text, grid, tile, window, stride) == CASES[5]:
        assert dropped > 0 and missed == 0


@pytest.mark.parametrize("n_text,grid,tile,window,stride", CASES)
def test_permutation_row_map_equals_the_tile_order(host_lib, n_text, grid, tile, window, stride):
    lay = OM.GnaLayout(n_text, grid, tile, window, stride)
    g = _geom(grid, tile, window, stride)
    out = np.empty(lay.N, dtype=np.int32)
    assert host_lib.h_tile_sources(n_text, ctypes.byref(g), out.ctypes.data, lay.N) == 0
    np.testing.assert_array_equal(out, OP.tile_order_source(lay))


@pytest.mark.parametrize("n_text,grid,tile,window,stride", CASES)
def test_tile_classes_equal_the_oracle(host_lib, n_text, grid, tile, window, stride):
    lay = OM.GnaLayout(n_text, grid, tile, window, stride)
    g = _geom(grid, tile, window, stride)
    nb = lay.N // lay.bs
    out = np.empty(nb * nb, dtype=np.uint8)
    assert host_lib.h_gna_classes(n_text, ctypes.byref(g), out.ctypes.data, nb) == 0
    got = out.reshape(nb, nb)
    if lay.N <= 4096:  # against the classes counted from the token-level mask
        valid = lay.valid(np.arange(lay.N))
        exp = OM.classify_blocks(OM.gna_token_mask(lay), lay.bs, lay.bs, valid, valid)
    else:              # the separable counts (pinned to token enumeration on small layouts)
        exp = OM.gna_block_classes_separable(lay)
    np.testing.assert_array_equal(got, exp)
