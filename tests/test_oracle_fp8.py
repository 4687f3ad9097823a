"""Pins for the e4m3 oracle: the format's own values and ties, and PyTorch's
float8_e4m3fn conversion as an independent library routine."""
import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import fp8 as OF8
from oracle import masks as OM


def test_format_has_the_expected_values():
    v = OF8.e4m3_values()
    assert len(v) == 253                      # 126 positive, 126 negative, one zero
    assert v.max() == 448.0 and v.min() == -448.0
    assert np.min(v[v > 0]) == 2.0 ** -9      # smallest subnormal
    assert np.all(OF8.round_e4m3(v) == v)     # every value is a fixed point


def test_ties_go_to_even_and_overflow_saturates():
    # 1.0625 lies halfway between 1 (mantissa 000) and 1.125 (001): to 1
    # 1.1875 between 1.125 (001) and 1.25 (010): to 1.25
    assert OF8.round_e4m3([1.0625, 1.1875, -1.0625]).tolist() == [1.0, 1.25, -1.0]
    assert OF8.round_e4m3([2.0 ** -10, 3 * 2.0 ** -10]).tolist() == [0.0, 2.0 ** -8]  # subnormal ties
    assert OF8.round_e4m3([447.0, 460.0, 1e6, -1e6]).tolist() == [448.0, 448.0, 448.0, -448.0]


def test_matches_torch_float8_in_range():
    # PyTorch's float8_e4m3fn conversion does not saturate (out-of-range
    # values become NaN), so the comparison stays inside +-440
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 100, 20000), rng.uniform(-440, 440, 20000),
                        rng.normal(0, 0.01, 20000)]).astype(np.float32)
    x = x[np.abs(x) <= 440.0]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(OF8.round_e4m3(x.astype(np.float64)), ref)


def test_block_quantisation_round_trip():
    rng = np.random.default_rng(1)
    x = rng.normal(0, 3, (200, 64))
    q, s = OF8.quantize(x, 64)
    assert len(s) == 4
    for b in range(4):  # each block's largest magnitude lands on 448 exactly
        blk = np.abs(q[b * 64:(b + 1) * 64])
        assert blk.max() == 448.0
    y = OF8.dequantize(q, s, 64)
    rel = np.abs(y - x) / np.maximum(np.abs(x), 2.0 ** -6 * np.repeat(s, 64)[:200, None])
    assert rel.max() <= 2.0 ** -4 + 1e-12    # half a step of a 3-bit mantissa
    assert np.all(OF8.block_scales(np.zeros((64, 8))) == 1.0)


def test_fp8_forward_is_the_plain_forward_on_representable_inputs():
    # inputs already on the e4m3 grid with block amax 448: quantisation is the identity
    rng = np.random.default_rng(2)
    v = OF8.e4m3_values()
    N, d = 128, 16
    q, k, vv = (rng.choice(v[np.abs(v) < 8], (N, d)) for _ in range(3))
    for t in (q, k, vv):
        t[0, 0] = 448.0
        t[64, 0] = 448.0
    deq = []
    for t in (q, k, vv):
        c, s = OF8.quantize(t, 64)
        assert np.all(s == 1.0) and np.array_equal(c, t)
        deq.append(OF8.dequantize(c, s, 64))
    fn = lambda r: OM.arrow_token_mask(N, 0, 64, 0, 0, r)
    a = OA.head_forward(*deq, 0, fn, d ** -0.5)
    b = OA.head_forward(q, k, vv, 0, fn, d ** -0.5)
    np.testing.assert_array_equal(a, b)


def test_encoding_matches_torch_float8_bytes():
    # every finite value, both zeros included, against PyTorch's float8_e4m3fn bit patterns
    v = np.concatenate([OF8.e4m3_values(), [-0.0]])
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(OF8.encode_e4m3(v), ref)
    assert OF8.encode_e4m3([448.0, 2.0 ** -9, 1.0]).tolist() == [0x7E, 0x01, 0x38]
    with pytest.raises(ValueError):
        OF8.encode_e4m3([1.03])


def test_fp32_decision_agrees_with_the_definition():
    rng = np.random.default_rng(4)
    x = (rng.normal(0, 1, (640, 128)) * rng.choice([1e-3, 1.0, 50.0], (640, 1))).astype(np.float32)
    c32, s32 = OF8.quantize_fp32(x)
    c64, s64 = OF8.quantize(x.astype(np.float64))
    np.testing.assert_allclose(s32, s64, rtol=2 ** -23)   # fl32(amax / 448) vs the exact ratio
    same = c32 == c64
    assert same.mean() > 0.9999
    # where they differ, they are neighbouring e4m3 values (a boundary straddled by fp32 rounding)
    vals = OF8.e4m3_values()
    idx = lambda a: np.searchsorted(vals, a)
    assert np.all(np.abs(idx(c32[~same]) - idx(c64[~same])) == 1)
    # every block's largest magnitude still lands on +-448, and zero blocks keep scale 1
    for b in range(10):
        assert np.abs(c32[b * 64:(b + 1) * 64]).max() == 448.0
    assert np.all(OF8.quantize_fp32(np.zeros((64, 8)))[1] == 1.0)
