"""Host-side logic for running the sampler on several GPUs (one process per GPU).

Every block's distribution is independent of every other block's (MaskLLM summary, s.3.4
"Block-wise independent distributions"), so ranks share no data on the hot path. Two ways
to split the work:
  * weak scaling (the benchmark): every rank owns a full copy of the workload's shapes with
    disjoint global block ids, as if the model were world times larger;
  * strong scaling: the layers of one model are dealt round-robin to the ranks, each layer
    keeping its global block ids, so the noise a block sees does not depend on the split.
The only exchange is the regulariser (a scalar term of the loss): a sum over ranks.
"""
from __future__ import annotations

from typing import List

from .configs import Workload, layer_block_offsets


def weak_block_offsets(w: Workload, rank: int) -> List[List[int]]:
    """Global block id of block 0 of every matrix of rank `rank`'s copy of the workload."""
    base = rank * w.total_blocks()
    return [[base + o for o in row] for row in layer_block_offsets(w)]


def strong_layers(w: Workload, rank: int, world: int) -> List[int]:
    """Layers owned by `rank` when one model's layers are split over `world` ranks."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return [l for l in range(w.layers) if l % world == rank]


def all_reduce_sum(t, group=None):
    """Sum a tensor (e.g. the per-layer regulariser sums) over all ranks, in place."""
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The largest of every rank's value (used for device-timed durations)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
