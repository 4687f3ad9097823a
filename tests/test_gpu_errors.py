"""Device-side fault reporting: a corrupt block list is caught, recorded and the GPU stays usable.

Faults are injected from the host (bad indices in a caller-owned list); nothing
here traps, faults or hangs the GPU.
"""
import numpy as np
import pytest
import torch

import workloads as W
from parity_util import bsa

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
