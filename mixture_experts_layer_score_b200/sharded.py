"""Token-sharded data parallelism for the layer forward, one process per GPU.

Tokens are independent through the whole layer, so each rank runs the forward on
its own contiguous shard of the batch with a full copy of the weights and no
data-path exchange. The one step that spans ranks is the expert-level balance
statistics f_i and P_i (DeepSeekMoE summary, "Expert-level balance loss"),
which are defined over every token of the batch: each rank's token counts and
score sums are summed across ranks (one all-reduce of 2 N' words) and the
library turns the sums into f and P (dsmoe_balance_stats).
"""
from __future__ import annotations

from typing import Tuple

import torch
import torch.distributed as dist


def shard_rows(T_total: int, rank: int, world: int) -> Tuple[int, int]:
    """[start, stop) of rank's contiguous token shard; shard sizes differ by at most one."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    base, extra = divmod(T_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def reduce_balance_sums(counts: torch.Tensor, P_sum: torch.Tensor, group=None) -> None:
    """Sum every rank's per-expert token counts (int32) and score sums (fp32) in place."""
    dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(P_sum, op=dist.ReduceOp.SUM, group=group)


def global_balance_stats(handle, T_total: int, counts: torch.Tensor, P_sum: torch.Tensor, f: torch.Tensor,
                         P: torch.Tensor, group=None, stream=None) -> None:
    """All-reduce the shard sums, then f_i and P_i over all T_total tokens (device kernel)."""
    from .binding import dsmoe_balance_stats
    reduce_balance_sums(counts, P_sum, group)
    dsmoe_balance_stats(handle, T_total, counts, P_sum, f, P, stream)
