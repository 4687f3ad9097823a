"""Seeded synthetic inputs shaped like the workloads on the pages.

This module only draws numbers: Q/K/V tensors, per-head mode tables, arrow
windows, cached outputs and the block-bias tables used by the DLM workload.
It holds none of the attention method's arithmetic (no masks, no pooling, no
selection, no softmax), so both the fp64 oracle and the CUDA path can take
their inputs from here without sharing any of the computation.

Every tensor is drawn from a seeded ``torch.Generator`` on the CPU in fp32
and rounded to bf16 with round-to-nearest-even (``Tensor.to(torch.bfloat16)``).
Discrete draws (mode tables, windows, bias patterns) use
``numpy.random.default_rng(seed)``.

Workload shapes (the pages' models stand in as shapes only; their prompts,
datasets and weights are not used):

* ``c1``  tiny arrow case, 64 text + 16x28 image tokens, block 64.
* ``c2``  SD3-1024-like MMDiT joint attention (256 text + 64x64 image tokens,
  d=64, block 64) with a drawn per-head mode table (full / arrow / skip),
  DiTFastAttnV2 "Head-wise Arrow Attention" and "Head-wise Caching".
* ``c3``  FLUX-2048-like content-driven selection (512 text + 128x128 image
  tokens, d=128, block 128); Q and K share a smooth 2-D field so that pooled
  block scores carry spatial structure (lmnt.cn BSA post, section 2.2).
* ``c4``  SparseD-like DLM attention (30720 prefill + 2048 generation tokens,
  d=128, block 128) with a per-head block bias that gives "column" or
  "slide-window" heads (SparseD, "Core contradiction" observation (1)).
* ``c5``  GNA-like 3-D video neighborhood attention (256 text + 16x48x80
  video tokens, tile 4x8x8, window 8x16x24).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

# Encodings of the per-head mode table that the library consumes.
HEAD_FULL = 0
HEAD_SPARSE = 1
HEAD_SKIP = 2


def normal_f32(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    """fp32 N(0, std^2) samples from a CPU generator seeded with ``seed``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x


def to_bf16(x: torch.Tensor) -> torch.Tensor:
    """Round an fp32 tensor to bf16 (round to nearest, ties to even)."""
    return x.to(torch.bfloat16)


def qkv_normal(B, H, N, d, seed):
    """Q, K, V ~ N(0,1) in bf16, shape [B,H,N,d], three consecutive seeds."""
    return tuple(to_bf16(normal_f32((B, H, N, d), seed * 3 + i)) for i in range(3))


@dataclass
class Shape:
    B: int
    H: int
    N: int
    d: int
    block_q: int
    block_k: int
    n_text: int

    @property
    def n_qb(self):
        return -(-self.N // self.block_q)

    @property
    def n_kb(self):
        return -(-self.N // self.block_k)


# ----------------------------------------------------------------------------
# mode tables


def largest_remainder(fracs, total):
    """Integer counts proportional to ``fracs`` summing to ``total``.

    Floors first, then the leftover units go to the largest fractional parts,
    ties to the earlier entry.
    """
    raw = [f * total for f in fracs]
    counts = [int(math.floor(r)) for r in raw]
    rest = total - sum(counts)
    order = sorted(range(len(fracs)), key=lambda i: (-(raw[i] - counts[i]), i))
    for i in order[:rest]:
        counts[i] += 1
    return counts


def draw_mode_table(H, seed, fracs=(0.40, 0.45, 0.15), windows=(1, 2, 4)):
    """Per-head (mode, arrow window) drawn from ``seed``.

    Counts of FULL / SPARSE(arrow) / SKIP heads follow ``fracs`` by largest
    remainder; their order is a seeded permutation; each arrow head's window
    (in blocks) is a seeded choice from ``windows``.
    """
    rng = np.random.default_rng(seed)
    counts = largest_remainder(fracs, H)
    modes = np.array([HEAD_FULL] * counts[0] + [HEAD_SPARSE] * counts[1] + [HEAD_SKIP] * counts[2],
                     dtype=np.int32)
    modes = modes[rng.permutation(H)]
    win = np.zeros(H, dtype=np.int32)
    for h in range(H):
        if modes[h] == HEAD_SPARSE:
            win[h] = int(rng.choice(np.array(windows)))
    return modes, win


# ----------------------------------------------------------------------------
# C1 / C2: arrow attention with a per-head mode table


def c1(seed: int = 0):
    shp = Shape(B=1, H=2, N=512, d=64, block_q=64, block_k=64, n_text=64)
    q, k, v = qkv_normal(shp.B, shp.H, shp.N, shp.d, seed)
    modes = np.array([HEAD_FULL, HEAD_SPARSE], dtype=np.int32)
    win = np.array([0, 1], dtype=np.int32)
    return dict(shape=shp, q=q, k=k, v=v, head_mode=modes, window=win, grid=(16, 28))


def arrow_case(B, H, n_text, grid_hw, d, block, seed, fracs=(0.40, 0.45, 0.15), windows=(1, 2, 4),
               with_cache=True):
    """Joint text+image attention inputs with a drawn mode table."""
    N = n_text + grid_hw[0] * grid_hw[1]
    shp = Shape(B=B, H=H, N=N, d=d, block_q=block, block_k=block, n_text=n_text)
    q, k, v = qkv_normal(B, H, N, d, seed)
    modes, win = draw_mode_table(H, seed, fracs, windows)
    cache = normal_f32((B, H, N, d), seed * 3 + 7) if with_cache else None
    return dict(shape=shp, q=q, k=k, v=v, head_mode=modes, window=win, cache=cache, grid=grid_hw)


def c2(seed: int = 1):
    return arrow_case(B=2, H=24, n_text=256, grid_hw=(64, 64), d=64, block=64, seed=seed)


# ----------------------------------------------------------------------------
# C3: content-driven selection on a smooth 2-D field


def smooth_field(H, gh, gw, d, sigma, seed):
    """Per-head d-channel Gaussian-blurred noise on a periodic gh x gw grid.

    The blur is applied in the Fourier domain (transfer function
    exp(-2 pi^2 sigma^2 |f|^2)); each channel is then renormalised to zero
    mean and unit standard deviation. Returns fp32 [H, gh*gw, d].
    """
    noise = normal_f32((H, d, gh, gw), seed)
    fy = torch.fft.fftfreq(gh, dtype=torch.float64)
    fx = torch.fft.fftfreq(gw, dtype=torch.float64)
    tf = torch.exp(-2.0 * math.pi ** 2 * sigma ** 2 * (fy[:, None] ** 2 + fx[None, :] ** 2))
    f = torch.fft.ifft2(torch.fft.fft2(noise.double()) * tf).real
    f = f - f.mean(dim=(-2, -1), keepdim=True)
    f = f / f.std(dim=(-2, -1), keepdim=True)
    return f.permute(0, 2, 3, 1).reshape(H, gh * gw, d).float()


def content_case(B, H, n_text, grid_hw, d, block, seed, sigma=8.0, noise_var=0.5):
    """Q = F + eps_q, K = F + eps_k with a shared smooth field F per head."""
    gh, gw = grid_hw
    N = n_text + gh * gw
    shp = Shape(B=B, H=H, N=N, d=d, block_q=block, block_k=block, n_text=n_text)
    std = math.sqrt(noise_var)
    qs, ks = [], []
    for b in range(B):
        fld = smooth_field(H, gh, gw, d, sigma, seed * 101 + b)
        for which, out in ((0, qs), (1, ks)):
            img = fld + normal_f32((H, gh * gw, d), seed * 101 + 10 + 2 * b + which, std)
            txt = normal_f32((H, n_text, d), seed * 101 + 50 + 2 * b + which)
            out.append(torch.cat([txt, img], dim=1))
    q = to_bf16(torch.stack(qs))
    k = to_bf16(torch.stack(ks))
    v = to_bf16(normal_f32((B, H, N, d), seed * 101 + 99))
    return dict(shape=shp, q=q, k=k, v=v, grid=grid_hw)


def c3(seed: int = 2):
    """FLUX-2048-like: keep the top 30% of image KV blocks, text always kept."""
    w = content_case(B=1, H=24, n_text=512, grid_hw=(128, 128), d=128, block=128, seed=seed)
    shp = w["shape"]
    ntb = -(-shp.n_text // shp.block_k)
    n_img = shp.n_kb - ntb
    w["groups"] = [(ntb, shp.n_kb, (30 * n_img + 99) // 100)]
    w["keep_text"] = True
    return w


# ----------------------------------------------------------------------------
# C4: DLM bidirectional attention with isolated prefill / generation selection


def dlm_bias(H, n_blocks, n_prefill_blocks, seed, beta=2.0, n_col_pre=24, n_col_gen=2,
             windows=(2, 4, 8)):
    """Block-constant logit bias per head, fp32 [H, n_blocks, n_blocks].

    Each head is drawn (p = 0.5) as a 'column' head (beta on a seeded set of
    prefill and generation key blocks, the same for every query block) or a
    'slide-window' head (beta where |I - J| <= w_h, w_h drawn from windows).
    Values are in natural-log units and are added to the scaled logits.
    """
    rng = np.random.default_rng(seed)
    bias = np.zeros((H, n_blocks, n_blocks), dtype=np.float32)
    kinds = []
    n_gen = n_blocks - n_prefill_blocks
    for h in range(H):
        if rng.random() < 0.5:
            cols = np.concatenate([
                rng.choice(n_prefill_blocks, size=min(n_col_pre, n_prefill_blocks), replace=False),
                n_prefill_blocks + rng.choice(n_gen, size=min(n_col_gen, n_gen), replace=False)])
            bias[h][:, cols] = beta
            kinds.append(("column", sorted(int(c) for c in cols)))
        else:
            w = int(rng.choice(np.array(windows)))
            ii = np.arange(n_blocks)
            bias[h][np.abs(ii[:, None] - ii[None, :]) <= w] = beta
            kinds.append(("slide-window", w))
    return torch.from_numpy(bias), kinds


def dlm_case(B, H, n_prefill, n_gen, d, block, seed, rho_pct=30):
    N = n_prefill + n_gen
    shp = Shape(B=B, H=H, N=N, d=d, block_q=block, block_k=block, n_text=0)
    npb = -(-n_prefill // block)
    nb = shp.n_kb
    bias, kinds = dlm_bias(H, nb, npb, seed)
    groups = [(0, npb, (rho_pct * npb + 99) // 100),
              (npb, nb, (rho_pct * (nb - npb) + 99) // 100)]
    return dict(shape=shp, bias=bias, bias_kinds=kinds, groups=groups, keep_text=False,
                n_prefill=n_prefill)


def dlm_step_qkv(shape: Shape, seed: int, step: int):
    """Fresh Q, K, V for denoising step ``step`` (step 0 is the selection step)."""
    return qkv_normal(shape.B, shape.H, shape.N, shape.d, 1000 * seed + 100 + step)


def c4(seed: int = 3):
    return dlm_case(B=1, H=32, n_prefill=30720, n_gen=2048, d=128, block=128, seed=seed)


# ----------------------------------------------------------------------------
# C5: GNA-like 3-D neighborhood attention over a video token grid


@dataclass
class GnaGeom:
    grid: tuple
    tile: tuple
    window: tuple
    stride: tuple

    @property
    def ndim(self):
        return len(self.grid)


def video_case(B, H, n_text, grid, tile, window, stride, d, seed):
    """Q/K/V in raster order: text first, then the video grid in (t, y, x) order."""
    n_vid = int(np.prod(grid))
    N = n_text + n_vid
    vol = int(np.prod(tile))
    shp = Shape(B=B, H=H, N=N, d=d, block_q=vol, block_k=vol, n_text=n_text)
    q, k, v = qkv_normal(B, H, N, d, seed)
    return dict(shape=shp, q=q, k=k, v=v,
                geom=GnaGeom(tuple(grid), tuple(tile), tuple(window), tuple(stride)))


def c5(stride=(4, 8, 8), seed: int = 4):
    return video_case(B=1, H=24, n_text=256, grid=(16, 48, 80), tile=(4, 8, 8),
                      window=(8, 16, 24), stride=stride, d=128, seed=seed)
