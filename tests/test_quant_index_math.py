"""The e4m3 quantiser's memory accesses, emulated on the CPU from the kernels' own index arithmetic
(csrc/quant.cu): every vector load and store is aligned to its width and inside its buffer, every
output byte is written exactly once, and the transposed V store puts key k of channel c at
c * Nt + k. No GPU.

The kernels' index expressions are restated here line by line (the grid, the thread's chunk and
the shared staging pitch); a change to one must change the other.
"""
import numpy as np
import pytest

ST_PITCH = 136  # kStPitch in csrc/quant.cu


def _rows_kernel(BH, N):
    """quant_rows_kernel: grid (nS, BH, 2), 256 threads; returns the byte offsets of every 16-byte
    load (bf16 source) and every 8-byte store (u8 codes), per tensor."""
    nS = -(-N // 64)
    loads, stores = [], []
    for blk in range(nS):
        for bh in range(BH):
            base = (bh * N + blk * 64) * 128
            rows = min(64, N - blk * 64)
            n16 = rows * 16
            for tid in range(256):
                for u in range(4):
                    c = tid + 256 * u
                    if c < n16:
                        loads.append(base * 2 + 16 * c)
                        stores.append(base + 8 * c)
    return np.array(loads), np.array(stores)


def _vt_kernel(BH, N):
    """quant_vt_kernel: grid (ceil(N / 128), BH), 256 threads; the 16-byte loads of V, the 8-byte
    shared stores of the staged codes, and the 16-byte transposed global stores with the keys each
    one carries."""
    Nt = (N + 15) // 16 * 16
    loads, sh_stores, g_stores = [], [], []
    for tile in range(-(-N // 128)):
        key0 = tile * 128
        keys = min(128, N - key0)
        for bh in range(BH):
            for half in range(2):
                for tid in range(256):
                    for u in range(4):
                        i = tid + 256 * u
                        key = half * 64 + (i >> 4)
                        if key < keys:
                            loads.append(((bh * N + key0) * 128 + key * 128 + (i & 15) * 8) * 2)
                        sh_stores.append((tile, bh, key * ST_PITCH + (i & 15) * 8))
            for tid in range(256):
                for u in range(4):
                    j = tid + 256 * u
                    c, g = j >> 3, j & 7
                    k0 = key0 + g * 16
                    if k0 >= Nt:
                        continue
                    g_stores.append((bh * 128 * Nt + c * Nt + k0, c, k0))
    return np.array(loads), sh_stores, g_stores, Nt


@pytest.mark.parametrize("BH,N", [(1, 300), (2, 128), (3, 453), (1, 64), (2, 1000)])
def test_quant_accesses_are_aligned_in_bounds_and_cover_every_byte(BH, N):
    loads, stores = _rows_kernel(BH, N)
    assert np.all(loads % 16 == 0) and np.all(stores % 8 == 0)
    assert loads.max() + 16 <= BH * N * 128 * 2 and stores.max() + 8 <= BH * N * 128
    cover = np.zeros(BH * N * 128, np.int64)
    for s in stores:
        cover[s:s + 8] += 1
    assert np.all(cover == 1)

    vl, sh, gs, Nt = _vt_kernel(BH, N)
    assert np.all(vl % 16 == 0) and vl.max() + 16 <= BH * N * 128 * 2
    offs = np.array([o for (_, _, o) in sh])
    assert np.all(offs % 8 == 0) and offs.max() + 8 <= 128 * ST_PITCH
    addr = np.array([a for (a, _, _) in gs])
    assert np.all(addr % 16 == 0) and addr.max() + 16 <= BH * 128 * Nt
    vcover = np.zeros(BH * 128 * Nt, np.int64)
    for a, c, k0 in gs:
        assert (a % Nt) == k0 and ((a // Nt) % 128) == c  # channel row c, keys k0 .. k0 + 15
        vcover[a:a + 16] += 1
    assert np.all(vcover == 1)
