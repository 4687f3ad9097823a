"""Head sharding of one attention problem across the ranks of a process group.

Every (b, h) unit of the hot path is independent: the block mask, the block
selection and the forward are all computed per head. One problem therefore
splits by heads with nothing to exchange before the forward. Rank r of W
owns the contiguous head range [r * H / W, (r + 1) * H / W) and runs the
whole path (bsa_build_mask or bsa_select_topk, then bsa_forward) on those
heads alone. A caller that already holds its heads sharded (sequence
parallelism that redistributes by heads) needs nothing more. A caller that
wants every head's output on every rank gathers O with one NCCL all-gather
per batch item (gather_heads): the ranks' head ranges are contiguous and in
rank order, so the gathered buffer is O in its own [B, H, N, d] layout and
needs no reordering.

This module only slices and gathers; the compute stays in the library's
kernels and the transfer in the process group's collective.
"""
from __future__ import annotations

import torch


def head_range(H: int, rank: int, world: int) -> tuple[int, int]:
    """The heads [h0, h1) that `rank` of `world` owns. H must be a multiple of world."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if H % world:
        raise ValueError(f"{H} heads do not split evenly over {world} ranks")
    hl = H // world
    return rank * hl, (rank + 1) * hl


def local_heads(x: torch.Tensor, rank: int, world: int, head_dim: int = 1) -> torch.Tensor:
    """The rank's heads of a per-head tensor ([B, H, ...] with head_dim 1, or [H, ...] with
    head_dim 0), as a contiguous tensor."""
    h0, h1 = head_range(x.shape[head_dim], rank, world)
    return x.narrow(head_dim, h0, h1 - h0).contiguous()


def gather_heads(o_local: torch.Tensor, world: int, group=None, out: torch.Tensor | None = None) -> torch.Tensor:
    """[B, H / world, N, d] on every rank -> [B, H, N, d] on every rank.

    One all-gather per batch item: out[b] ([H, N, d], contiguous) is the rank-ordered
    concatenation of every rank's o_local[b], which is exactly the head order."""
    import torch.distributed as dist
    if not o_local.is_contiguous():
        raise ValueError("o_local must be contiguous")
    B, hl = o_local.shape[0], o_local.shape[1]
    shape = (B, hl * world) + tuple(o_local.shape[2:])
    if out is None:
        out = torch.empty(shape, dtype=o_local.dtype, device=o_local.device)
    elif tuple(out.shape) != shape or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {shape} tensor")
    for b in range(B):
        dist.all_gather_into_tensor(out[b], o_local[b], group=group)
    return out
