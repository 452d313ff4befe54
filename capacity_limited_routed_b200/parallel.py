"""Data-parallel replicas of the MoE block: the one exchange the block needs.

Each GPU is one source with its own T tokens (its own slots, caps and drops).  The bias
step, though, must see the load of the whole step so that every replica keeps the same
bias: the per-expert selection histograms are summed over ranks (int32, exact) and the
step uses the total token count.  Nothing else crosses ranks on the block's data path.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def global_histogram(hist: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the int32 [E] selection histogram over the ranks of ``group`` (in place)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(hist, op=dist.ReduceOp.SUM, group=group)
    return hist


def global_tokens(T_local: int, group=None) -> int:
    """Tokens of the whole step (every replica holds the same T)."""
    if dist.is_available() and dist.is_initialized():
        return T_local * dist.get_world_size(group)
    return T_local
