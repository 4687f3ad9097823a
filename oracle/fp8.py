"""FP8 (e4m3) operands of the forward (fp64 oracle, test use only).

The GNA article (Blackwell adaptation, "mixed precision") computes in
FP16/BF16 and offers FP8 for more throughput (1.7 against 1.2 PFLOP/s on
B200, +40% at equal visual quality). It gives no scheme; readings:

* e4m3 is the OCP 8-bit float with 1 sign, 4 exponent (bias 7) and 3
  mantissa bits, no infinities, largest finite 448, subnormals down to 2^-9.
  Conversion rounds to nearest, ties to even, and saturates at +-448 (the
  hardware's satfinite conversion).
* Q, K and V are scaled per (b, h, 64-token block): s = amax / 448 over the
  block's tokens and channels (s = 1 for an all-zero block), stored as
  e4m3(x / s), read back as e4m3 * s.
* The FP8 forward is the attention of the same heads on the dequantised
  operands; how the kernel rounds P is the kernel's business, as with bf16.
* Where fp arithmetic decides a code, the decision is taken in the kernel's
  precision (quantize_fp32): r = fl32(448 / amax) once per block, then
  e4m3(fl32(x * r)); the scale is fl32(amax / 448). It differs from
  quantize() only where fl32(x * r) and x / s straddle a rounding boundary.
* Codes are stored as OCP e4m3 bytes (encode_e4m3): sign in bit 7, biased
  exponent in bits 3..6, mantissa in bits 0..2; exponent field 0 holds the
  subnormals m/8 * 2^-6.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def round_e4m3(x):
    """fp64 array: x rounded to the nearest e4m3 value (ties to even), saturated."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # exponent of the binade; below the normal range the step stays 2^-9
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    step = np.exp2(e - 3.0)
    q = np.round(a / step) * step          # exact: step is a power of two
    q = np.minimum(q, E4M3_MAX)
    q = np.where(a > 0, q, 0.0)
    return np.copysign(q, x)


def e4m3_values():
    """All 253 finite e4m3 values that differ as numbers (+0 once), fp64, sorted."""
    vals = {0.0}
    for e in range(-6, 9):
        for m in range(8):
            v = (1 + m / 8) * 2.0 ** e
            if v <= E4M3_MAX:
                vals.add(v)
                vals.add(-v)
    for m in range(1, 8):  # subnormals
        vals.add(m / 8 * 2.0 ** -6)
        vals.add(-m / 8 * 2.0 ** -6)
    return np.array(sorted(vals))


def block_scales(x, bs=64):
    """fp64 [nB]: amax / 448 per bs-token block of x [N, d] (1 for zero blocks)."""
    x = np.asarray(x, dtype=np.float64)
    N = x.shape[0]
    nb = -(-N // bs)
    s = np.empty(nb)
    for b in range(nb):
        m = np.max(np.abs(x[b * bs:(b + 1) * bs]))
        s[b] = m / E4M3_MAX if m > 0 else 1.0
    return s


def quantize(x, bs=64):
    """(codes as e4m3 values fp64 [N, d], scales [nB]) for x [N, d]."""
    x = np.asarray(x, dtype=np.float64)
    s = block_scales(x, bs)
    rows = np.repeat(s, bs)[: x.shape[0]][:, None]
    return round_e4m3(x / rows), s


def dequantize(q, s, bs=64):
    rows = np.repeat(np.asarray(s), bs)[: q.shape[0]][:, None]
    return np.asarray(q) * rows


def quantize_fp32(x, bs=64):
    """(codes as e4m3 values fp64 [N, d], scales [nB]) for x [N, d], the code decision in fp32."""
    x = np.asarray(x, dtype=np.float32)
    N = x.shape[0]
    nb = -(-N // bs)
    codes = np.empty(x.shape, dtype=np.float64)
    s = np.empty(nb)
    for b in range(nb):
        blk = x[b * bs:(b + 1) * bs]
        m = np.float32(np.max(np.abs(blk)))
        r = np.float32(np.float32(E4M3_MAX) / m) if m > 0 else np.float32(1.0)
        codes[b * bs:(b + 1) * bs] = round_e4m3((blk * r).astype(np.float32).astype(np.float64))
        s[b] = float(np.float32(m / np.float32(E4M3_MAX))) if m > 0 else 1.0
    return codes, s


def encode_e4m3(v):
    """uint8 bytes of e4m3 values (each must be representable; -0 encodes as 0x80)."""
    v = np.asarray(v, dtype=np.float64)
    if not np.all(round_e4m3(v) == v):
        raise ValueError("not an e4m3 value")
    a = np.abs(v)
    sign = (np.signbit(v).astype(np.int64)) << 7
    e = np.floor(np.log2(np.where(a > 0, a, 1.0))).astype(np.int64)
    normal = ((e + 7) << 3) | np.round((a / np.exp2(e) - 1.0) * 8).astype(np.int64)
    sub = np.round(a / 2.0 ** -9).astype(np.int64)          # a = m * 2^-9, m in 0..7
    return (np.where(a < 2.0 ** -6, sub, normal) | sign).astype(np.uint8)
