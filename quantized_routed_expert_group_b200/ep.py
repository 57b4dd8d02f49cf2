"""Expert parallelism: the layer's routed experts spread over the ranks of a
process group (wpnews.pro "Colibri — รัน GLM-5.2 ...", "Multi-GPU expert
tier": experts spread over several GPUs).

Every rank holds the router and routes every token itself (the routing is
cheap next to the experts and the same on every rank), computes the share of
the layer output of the routed experts it owns (rank 0 also adds the shared
expert) with moe_layer_forward_partial, and the shares are summed with one
all-reduce.  The exchange is that one collective on T x hidden fp32 values.

Ranges are contiguous and balanced: rank r owns experts
[r * E // world, (r + 1) * E // world).
"""
from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist


def expert_range(rank: int, world: int, n_experts: int) -> tuple[int, int]:
    """The routed experts [lo, hi) that `rank` of `world` owns."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    return rank * n_experts // world, (rank + 1) * n_experts // world


def owns_shared(rank: int) -> bool:
    """Exactly one rank adds the shared expert: rank 0."""
    return rank == 0


def ep_forward(partial: Callable[[torch.Tensor, int, int, bool], torch.Tensor], x: torch.Tensor, n_experts: int,
               group=None) -> torch.Tensor:
    """The layer output on this rank: its share from `partial(x, lo, hi,
    with_shared)`, summed over the group's ranks (every rank gets the sum)."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    lo, hi = expert_range(rank, world, n_experts)
    out = partial(x, lo, hi, owns_shared(rank))
    if world > 1:
        dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


class ExpertParallelLayer:
    """A MoeLayer used as one rank of an expert-parallel group: forward()
    returns the full layer output, computed from this rank's experts and one
    all-reduce."""

    def __init__(self, layer, group=None):
        self.layer = layer
        self.group = group

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        return ep_forward(lambda xx, lo, hi, sh: self.layer.forward_partial(xx, lo, hi, sh), x,
                          self.layer.shape.n_experts, self.group)
