"""Data parallelism for the QLoRA layer: every rank runs the layer on its own tokens with a replica of the
frozen NF4 weight and of the adapters; the only exchange is the sum of the adapter gradients dA, dB.

The forward and dX are row-independent, so they need no communication.  dA and dB are sums over tokens,
so the data-parallel gradient is the all-reduce (sum) of the per-rank gradients -- r (K + N) fp32 values
per layer, sent over NCCL on NVLink.  The weight is frozen (no dW), which is why this exchange is tiny.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def token_shard(M_total: int, world: int, rank: int) -> tuple[int, int]:
    """[begin, end) of the tokens rank `rank` owns when M_total tokens are split as evenly as possible."""
    base, extra = divmod(M_total, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def allreduce_adapter_grads(grads, group=None) -> None:
    """Sum the adapter gradients (tensors, in place) over the ranks of `group`."""
    for g in grads:
        if g is not None:
            dist.all_reduce(g, op=dist.ReduceOp.SUM, group=group)
