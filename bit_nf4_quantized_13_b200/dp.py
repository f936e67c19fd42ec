"""Data-parallel plumbing for the QLoRA linear.

Under data parallelism every rank holds the same frozen NF4 weight and the
same adapters (A, B), and processes its own slice of the tokens.  The only
exchange per step is the sum of the adapter gradients dA (r x K) and dB
(N x r) across ranks; there is no gradient for the frozen weight, so the
exchange is r (N + K) values per linear.  torch.distributed carries it
(NCCL over NVLink on GPUs, gloo on CPU).
"""
from __future__ import annotations


def shard_rows(M: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous token range [start, stop) of `rank` when M tokens are split
    as evenly as possible over `world` ranks (the first M % world ranks take
    one extra token)."""
    if world < 1 or not 0 <= rank < world or M < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_adapter_grads(dA, dB, group=None, average: bool = False):
    """Sum (or average) dA and dB over the ranks of `group`, in place.

    Both tensors go through one flat buffer so the exchange is a single
    collective; every rank must call this in the same order."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized():
        return dA, dB
    world = dist.get_world_size(group)
    if world == 1:
        return dA, dB
    flat = torch.cat([dA.reshape(-1).float(), dB.reshape(-1).float()])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    if average:
        flat /= world
    na = dA.numel()
    dA.copy_(flat[:na].view_as(dA))
    dB.copy_(flat[na:].view_as(dB))
    return dA, dB
