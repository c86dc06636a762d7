"""Data parallelism over tokens: host-side plumbing only.

Each rank holds the whole frozen low-bit base and the adapter, and runs the
layer on its own tokens. The forward pass and the activation gradient need no
exchange between ranks. The adapter is shared, so a training step sums its
gradient over the ranks: the one collective of the path (an NCCL all-reduce
over NVLink on GPUs; gloo in the CPU tests).

The adapter gradient is a sum over rows of x^T dx' (per expert, per 32 x 32
block), and every row belongs to exactly one rank, so the sum over ranks of
the per-rank gradients is the gradient of the whole batch.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def token_shard(T: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous, balanced token range [start, stop) of `rank` out of `world`."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    base, extra = divmod(T, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_adapter_grad(d_adapter: torch.Tensor, group=None) -> torch.Tensor:
    """Sums the FP32 adapter gradient over the ranks of `group`, in place."""
    if d_adapter.dtype != torch.float32:
        raise TypeError("the adapter gradient is float32")
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(d_adapter, op=dist.ReduceOp.SUM, group=group)
    return d_adapter
