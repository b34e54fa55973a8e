"""Head sharding of one SLA / SLA2 forward across ranks.

Every (batch, head) problem of the forward is independent: mask prediction,
the linear statistics, the marginal aggregation and the fused kernel read only
their own head's Q, K, V ("SLA: Beyond Sparsity in Diffusion Transformers via
Fine-Tunable Sparse-Linear Attention", §2 Q2: every step is per head).  One
problem therefore splits across GPUs by heads with no exchange at all; the
output stays head-sharded, or one all-gather assembles it when the caller wants
it whole.  A rank passes its slice to the C ABI as a strided view (the ABI takes
element strides for B, H, N), so nothing is copied.

This module holds the host logic only: which heads a rank owns, the strided
views, and the gather.  The collective runs on whatever process group the
caller set up (NCCL between GPUs, gloo on CPU).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def head_range(H: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous heads [h0, h1) of `rank`: H split into `world` parts whose sizes
    differ by at most one (the first H % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def head_slice(x: torch.Tensor, H: int, rank: int, world: int) -> torch.Tensor:
    """The rank's heads of a [B, H, N, d] tensor (or of a per-head [B, H]
    parameter) as a view."""
    h0, h1 = head_range(H, rank, world)
    return x[:, h0:h1]


def gather_heads(o_local: torch.Tensor, H: int, group=None) -> torch.Tensor:
    """All ranks' head slices of O, assembled into [B, H, N, d] on every rank with
    one all_gather (slices are padded to the largest share, then trimmed)."""
    world = dist.get_world_size(group)
    sizes = [head_range(H, r, world) for r in range(world)]
    most = max(h1 - h0 for h0, h1 in sizes)
    B, h, N, d = o_local.shape
    pad = o_local.new_zeros((B, most, N, d))
    pad[:, :h] = o_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([p[:, :h1 - h0] for p, (h0, h1) in zip(parts, sizes)], dim=1)
