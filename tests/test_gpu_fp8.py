"""GPU e4m3 path (bsa_quantize_fp8 + bsa_forward_fp8) against the fp64 oracle.

* The quantiser's codes decide an integer from floating point, so the oracle takes that decision
  in the kernel's precision (oracle.fp8.quantize_fp32): codes and scales must match bit for bit,
  bytes in the OCP e4m3 encoding, V transposed with zero padding.
* The forward is judged against fp64 attention on the dequantised operands (the oracle's codes,
  decided as above, times their scales, in fp64), within a bound per output element derived
  from the kernel's arithmetic. The kernel rounds each probability, held as P = p * sv / sigma
  (sigma the head's largest V scale, P <= 2^8 under the lazy max), to the nearest e4m3 value:
  the error is at most 2^-4 * P in e4m3's normal range and at most 2^-10 (half the subnormal
  step) below it. Summed through P V and the normalisation (the kernel's row sum, taken against
  a running max no larger than the true one, is at least the exact l = 1 / max_j p_ij):
    |O - O_ref| <= 2^-4 * sum_j p_ij |v_j| + 2^-10 * sigma * max_j p_ij * sum_j |code_j|
                   + 2^-8 |O_ref| (O rounded to bf16) + 1e-3 (fp32 accumulation),
  with the sums over the allowed keys j of row i, code_j the e4m3 value of v_j (v_j / sv_j).
  On Gaussian inputs the mean error must also stay within the bf16 bar of 5e-3; on strongly
  peaked rows the e4m3 floor on the many small probabilities lifts it above that (a numpy model
  of the kernel's arithmetic gives 7.7e-3 on the peaked case below), so there the per-element
  bound alone is the criterion.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from oracle import fp8 as OF8
from oracle import masks as OM
from oracle import permute as OP
from parity_util import bsa, f64

pytestmark = pytest.mark.gpu


def _dims(shp):
    return bsa().dims(shp.B, shp.H, shp.N, shp.d, shp.block_q, shp.block_k, shp.n_text)


def _quantize(dm, q, k, v):
    m = bsa()
    ops = m.Fp8Operands.empty(dm.B, dm.H, dm.N)
    ops.v8t.fill_(0xAB)  # the padding columns must come back zero
    m.quantize_fp8(dm, q.cuda(), k.cuda(), v.cuda(), ops)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    return ops


@pytest.mark.parametrize("B,H,N", [(1, 2, 300), (2, 1, 128), (1, 3, 64 * 7 + 5)])
def test_quantize_codes_scales_and_layout(B, H, N):
    q, k, v = W.qkv_normal(B, H, N, 128, N)
    v[:, :, :64] = 0  # an all-zero block: scale 1, codes 0
    dm = bsa().dims(B, H, N, 128, 128, 128, 0)
    ops = _quantize(dm, q, k, v)
    nt = (N + 15) // 16 * 16
    for b in range(B):
        for h in range(H):
            for x, codes, sc in ((q, ops.q8, ops.sq), (k, ops.k8, ops.sk)):
                c, s = OF8.quantize_fp32(x[b, h].float().numpy())
                np.testing.assert_array_equal(codes[b, h].cpu().numpy(), OF8.encode_e4m3(c))
                np.testing.assert_array_equal(sc[b, h].cpu().numpy(), s.astype(np.float32))
            c, s = OF8.quantize_fp32(v[b, h].float().numpy())
            vt = ops.v8t[b, h].cpu().numpy()
            np.testing.assert_array_equal(vt[:, :N], OF8.encode_e4m3(c).T)
            assert np.all(vt[:, N:nt] == 0)
            np.testing.assert_array_equal(ops.sv[b, h].cpu().numpy(), s.astype(np.float32))
            assert float(ops.sv[b, h, 0]) == 1.0


def test_quantize_bytes_equal_torch_float8_on_the_grid():
    """An independent encoder: a block already on the e4m3 grid with amax 448 has r = 1, so its
    codes are its own values, whose bytes PyTorch's float8_e4m3fn conversion gives."""
    q, k, v = W.qkv_normal(1, 1, 256, 128, 7)
    g = torch.from_numpy(np.random.default_rng(7).choice(OF8.e4m3_values(), (64, 128)).astype(np.float32))
    g[0, 0] = 448.0
    q[0, 0, 64:128] = g.to(torch.bfloat16)
    ops = _quantize(bsa().dims(1, 1, 256, 128, 128, 128, 0), q, k, v)
    assert float(ops.sq[0, 0, 1]) == 1.0
    ref = q[0, 0, 64:128].float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ops.q8[0, 0, 64:128].cpu().numpy(), ref)


def _operands(x):
    """The oracle's operand of one (b, h): codes decided in fp32 as the kernel does, their scales,
    and the dequantised values in fp64."""
    c, s = OF8.quantize_fp32(f64(x).astype(np.float32))
    return c, s, OF8.dequantize(c, s)


def _check_rows(got, q, k, v, mode, fn, rows, bias_fn=None, what="", mean_bar=5e-3):
    (_, _, qd), (_, _, kd), (cv, sv, vd) = (_operands(t) for t in (q, k, v))
    exp = OA.head_forward(qd, kd, vd, mode, fn, 128 ** -0.5, rows=rows, bias_fn=bias_fn)
    allowed = fn(rows)
    bias = None if bias_fn is None else bias_fn(rows)
    p = OA.attention_probs_rows(qd[rows], kd, allowed, 128 ** -0.5, bias)
    sigma = float(np.max(sv))
    floor = 2.0 ** -10 * sigma * p.max(axis=1, keepdims=True) * (allowed.astype(np.float64) @ np.abs(cv))
    bound = 2.0 ** -4 * (p @ np.abs(vd)) + floor + 2.0 ** -8 * np.abs(exp) + 1e-3
    err = np.abs(got - exp)
    ok = err <= bound
    worst = np.unravel_index(np.argmax(err / bound), err.shape)
    assert ok.all(), f"{what}: err {float(err[worst]):.3e} against bound {float(bound[worst]):.3e} at {worst}"
    if mean_bar is not None:
        assert err.mean() <= mean_bar, f"{what}: mean {float(err.mean()):.3e}"


def test_forward_fp8_schedule_after_other_kernels():
    """The forward's schedule is written lane by lane and read across lanes before the CTA's
    barrier (e4m3 tile reorder, geometry, tile counts). Without a warp sync between the two,
    the reorder could read what an earlier kernel left in shared memory. It then scrambled
    the schedule: a misaligned-tile error, and at times an out-of-range scale index. Ragged
    and even lengths in turn, each on fresh buffers after the other's kernels, many times;
    every forward must end with the error word clear."""
    m = bsa()
    cases = []
    for N in (128 * 6, 128 * 6 + 40):
        w = W.arrow_case(B=1, H=4, n_text=128, grid_hw=(1, N - 128), d=128, block=128, seed=N,
                         fracs=(0.25, 0.5, 0.25))
        cases.append(w)
    for rep in range(6):
        for w in cases:
            shp = w["shape"]
            dm = _dims(shp)
            ops = _quantize(dm, w["q"], w["k"], w["v"])
            modes = torch.from_numpy(w["head_mode"]).cuda()
            blocks = m.BlockList.empty(1, shp.H, shp.n_qb, shp.n_kb, bitmap=False)
            m.build_mask(dm, m.MASK_ARROW, blocks, head_mode=modes, window=torch.from_numpy(w["window"]).cuda())
            o = torch.empty(w["q"].shape, dtype=torch.bfloat16, device="cuda")
            m.forward_fp8(dm, ops, o, modes, blocks=blocks, cache_in=w["cache"].cuda())
            torch.cuda.synchronize()
            assert m.get_device_error() == 0, (rep, shp.N)
            del ops, blocks, o


@pytest.mark.parametrize("N", [128 * 6, 128 * 6 + 40])
def test_forward_fp8_arrow_full_skip(N):
    m = bsa()
    w = W.arrow_case(B=1, H=4, n_text=128, grid_hw=(1, N - 128), d=128, block=128, seed=N,
                     fracs=(0.25, 0.5, 0.25))
    shp = w["shape"]
    dm = _dims(shp)
    ops = _quantize(dm, w["q"], w["k"], w["v"])
    modes = torch.from_numpy(w["head_mode"]).cuda()
    blocks = m.BlockList.empty(1, shp.H, shp.n_qb, shp.n_kb, bitmap=False)
    m.build_mask(dm, m.MASK_ARROW, blocks, head_mode=modes, window=torch.from_numpy(w["window"]).cuda())
    o = torch.empty(w["q"].shape, dtype=torch.bfloat16, device="cuda")
    m.forward_fp8(dm, ops, o, modes, blocks=blocks, cache_in=w["cache"].cuda())
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    for h in range(shp.H):
        mode = int(w["head_mode"][h])
        if mode == W.HEAD_SKIP:  # the cache path is the bf16 one: exact
            exp = OA.bf16_round(w["cache"][0, h].numpy().astype(np.float32))
            np.testing.assert_array_equal(f64(o[0, h]), exp)
            continue
        fn = lambda r, h=h, mode=mode: OM.arrow_token_mask(N, shp.n_text, 128, mode, int(w["window"][h]), r)
        _check_rows(f64(o[0, h]), w["q"][0, h], w["k"][0, h], w["v"][0, h], mode, fn, np.arange(N), what=f"h{h}")


def test_forward_fp8_block_bias_and_peaked_rows():
    """A block bias and large logits (scaled Q) give peaked rows, where the lazy rescale and the
    P scaling into e4m3 range matter most."""
    m = bsa()
    B, H, N, bs = 1, 2, 128 * 5 + 30, 128
    q, k, v = W.qkv_normal(B, H, N, 128, 11)
    q = (q.float() * 3.0).to(torch.bfloat16)
    nb = -(-N // bs)
    bias, _ = W.dlm_bias(H, nb, nb - 1, seed=3, n_col_pre=2, n_col_gen=1, windows=(1,))
    dm = m.dims(B, H, N, 128, bs, bs, 0)
    ops = _quantize(dm, q, k, v)
    o = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    modes = torch.zeros(H, dtype=torch.int32, device="cuda")
    m.forward_fp8(dm, ops, o, modes, bias=bias.cuda())
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    for h in range(H):
        bfn = OA.block_bias_fn(bias[h].numpy(), bs, bs, N)
        _check_rows(f64(o[0, h]), q[0, h], k[0, h], v[0, h], OM.HEAD_FULL, lambda r: np.ones((len(r), N), bool),
                    np.arange(N), bias_fn=bfn, what=f"h{h}", mean_bar=None)


@pytest.mark.parametrize("stride", [(1, 1, 1), (2, 4, 4)])
def test_forward_fp8_gna_partial_tiles(stride):
    """GNA tiles of 2 x 8 x 8 = 128 tokens in tile order with partial tiles (the fine mask) and a
    padded grid."""
    m = bsa()
    n_text, grid, tile, window = 128, (4, 12, 20), (2, 8, 8), (3, 9, 11)
    wl = W.video_case(1, 2, n_text, grid, tile, window, stride, 128, 9)
    lay = OM.GnaLayout(n_text, grid, tile, window, stride)
    g = m.GnaGeom.make(grid, tile, window, stride)
    nt = m.gna_tiled_len(n_text, g)
    dm_r = m.dims(1, 2, wl["shape"].N, 128, lay.bs, lay.bs, n_text)
    dm = m.dims(1, 2, nt, 128, lay.bs, lay.bs, n_text)
    raster = [t.cuda() for t in (wl["q"], wl["k"], wl["v"])]
    tiled = [torch.empty((1, 2, nt, 128), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    m.permute_tiles(dm_r, g, raster, tiled)
    ops = _quantize(dm, *tiled)
    nb = nt // lay.bs
    blocks = m.BlockList.empty(1, 2, nb, nb, bitmap=False)
    modes = torch.ones(2, dtype=torch.int32, device="cuda")
    m.build_mask(dm, m.MASK_GNA, blocks, head_mode=modes, gna=g)
    o = torch.empty_like(tiled[0])
    m.forward_fp8(dm, ops, o, modes, blocks=blocks, gna=g)
    torch.cuda.synchronize()
    assert m.get_device_error() == 0
    rows = np.nonzero(lay.valid(np.arange(nt)))[0]
    for h in range(2):
        qt, kt, vt = (OP.permute_to_tiles(f64(t[0, h]), lay) for t in (wl["q"], wl["k"], wl["v"]))
        _check_rows(f64(o[0, h])[rows], torch.from_numpy(qt), torch.from_numpy(kt), torch.from_numpy(vt),
                    OM.HEAD_SPARSE, lambda r: OM.gna_token_mask(lay, r), rows, what=f"gna h{h}")


def test_fp8_rejects_what_it_does_not_cover():
    m = bsa()
    q = torch.zeros(1, 1, 256, 64, dtype=torch.bfloat16, device="cuda")
    ops = m.Fp8Operands.empty(1, 1, 256, 64)
    with pytest.raises(m.BsaError):  # d = 64
        m.quantize_fp8(m.dims(1, 1, 256, 64, 64, 64, 0), q, q, q, ops)
    ops = m.Fp8Operands.empty(1, 1, 256)
    o = torch.empty(1, 1, 256, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.BsaError):  # key blocks of 64
        m.forward_fp8(m.dims(1, 1, 256, 128, 64, 64, 0), ops, o, torch.zeros(1, dtype=torch.int32, device="cuda"))
