"""Device-side fault reporting: a corrupt block list or a wait that runs out is caught, recorded
and the GPU stays usable.

Faults are injected from the host (bad indices in a caller-owned list; a key tile the producer is
told never to load, with a short wait limit); nothing here traps, faults or hangs the GPU.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from oracle import masks as OM
from parity_util import assert_close_out, bsa, f64

pytestmark = pytest.mark.gpu


def test_bad_block_index_sets_device_error_and_gpu_stays_usable():
    m = bsa()
    B, H, N, d, bs = 1, 1, 512, 64, 64
    q, k, v = (t.cuda() for t in W.qkv_normal(B, H, N, d, 1))
    nb = N // bs
    blocks = m.BlockList.empty(B, H, nb, nb, bitmap=False)
    blocks.cnt.fill_(1)
    blocks.idx.fill_(-1)
    blocks.idx[..., 0] = 1000  # out of range
    blocks.flag.fill_(1)
    o = torch.empty_like(q)
    modes = torch.ones(H, dtype=torch.int32, device="cuda")
    assert m.get_device_error() == 0
    m.forward(m.dims(B, H, N, d, bs, bs, 0), q, k, v, o, modes, blocks=blocks)
    assert m.get_device_error() == m.DEVERR_BAD_INDEX
    assert m.get_device_error() == 0  # read clears it
    # the context is still healthy: a normal call works
    blocks.idx[..., 0] = 0
    m.forward(m.dims(B, H, N, d, bs, bs, 0), q, k, v, o, modes, blocks=blocks)
    assert m.get_device_error() == 0
    assert torch.isfinite(o.float()).all()


def test_count_above_capacity_is_reported():
    m = bsa()
    B, H, N, d, bs = 1, 1, 256, 64, 64
    q, k, v = (t.cuda() for t in W.qkv_normal(B, H, N, d, 2))
    nb = N // bs
    blocks = m.BlockList.empty(B, H, nb, nb, bitmap=False)
    blocks.cnt.fill_(99)
    blocks.idx.copy_(torch.arange(nb, dtype=torch.int32).expand_as(blocks.idx))
    blocks.flag.fill_(1)
    o = torch.empty_like(q)
    m.forward(m.dims(B, H, N, d, bs, bs, 0), q, k, v, o, torch.ones(H, dtype=torch.int32, device="cuda"),
              blocks=blocks)
    assert m.get_device_error() == m.DEVERR_BAD_INDEX


@pytest.mark.parametrize("d", [64, 128])
def test_a_wait_that_runs_out_is_reported_and_the_context_survives(d):
    """The producer withholds key tile 2 (its K is never loaded, so nothing completes the waits on
    it) and every pipeline wait is bounded by 2 ms: the forward must end with BSA_DEVERR_TIMEOUT,
    its CTAs having drained the copies and MMAs in flight before freeing tensor memory. The next
    normal call on the same context is then exact against the oracle with error word 0.
    d = 64 runs the polling MMA issuer, d = 128 the fixed-order one."""
    m = bsa()
    B, H, N, bs = 1, 2, 1024, 64
    q, k, v = (t.cuda() for t in W.qkv_normal(B, H, N, d, 5))
    dm = m.dims(B, H, N, d, bs, bs, 0)
    modes = torch.zeros(H, dtype=torch.int32, device="cuda")  # full heads: 8 key tiles per CTA
    o = torch.empty_like(q)
    assert m.get_device_error() == 0
    m.set_wait_limit_ns(2_000_000)
    m.set_withheld_tile(2)
    try:
        m.forward(dm, q, k, v, o, modes)
        assert m.get_device_error() == m.DEVERR_TIMEOUT
    finally:
        m.set_withheld_tile(-1)
        m.set_wait_limit_ns(0)
    assert m.get_device_error() == 0
    m.forward(dm, q, k, v, o, modes)
    assert m.get_device_error() == 0
    qc, kc, vc = (f64(t.cpu()) for t in (q, k, v))
    rows = np.array([0, 1, 300, 777, N - 1])
    for h in range(H):
        exp = OA.head_forward(qc[0, h], kc[0, h], vc[0, h], OM.HEAD_FULL, lambda r: np.ones((len(r), N), bool),
                              d ** -0.5, rows=rows)
        assert_close_out(f64(o[0, h].cpu())[rows], exp, f"h{h}")


