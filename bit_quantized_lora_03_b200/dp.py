"""Data-parallel plumbing for the QLoRA linear: one process per GPU, torch.distributed.

Every rank holds a full packed NF4 replica of the frozen W (the weights never change, so they
are never communicated) and its own slice of the tokens. The only exchange of a training step
is the sum of the adapter gradients dL1, dL2 over ranks: they are sums over tokens, so the sum
of the per-rank gradients equals the gradient of the whole batch.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def token_shard(t_total: int, rank: int, world: int) -> slice:
    """Contiguous, nearly equal slice of t_total tokens for `rank` of `world`."""
    base, extra = divmod(t_total, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


def allreduce_adapter_grads(grads: list[torch.Tensor], group=None) -> None:
    """Sum the fp32 adapter gradients over all ranks, in place, with one collective."""
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return
    flat = torch.cat([g.reshape(-1) for g in grads])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    off = 0
    for g in grads:
        n = g.numel()
        g.copy_(flat[off:off + n].view_as(g))
        off += n


def max_over_ranks(value: float, device=None) -> float:
    """The largest of `value` over all ranks (timing: the slowest rank sets the pace)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
