"""Multi-GPU plumbing for decoding: one process per GPU, no data-path collective.

Coded tensors are independent (every chunk decodes on its own), so a model's weights shard across
ranks by whole tensors and each rank decodes only its share; nothing is exchanged on the decode
path.  The one collective is the timing reduction (the slowest rank sets the step time).
torch.distributed is the plumbing: NCCL between GPUs, gloo on CPU (tests).
"""
from __future__ import annotations

import datetime
import os


def env_rank() -> tuple[int, int, int]:
    """(world size, rank, local rank) from the launcher's environment (1, 0, 0 when absent)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 120.0, device=None) -> tuple[int, int, int]:
    """Join the process group when launched with WORLD_SIZE > 1; returns (world, rank, local)."""
    import torch.distributed as dist
    world, rank, local = env_rank()
    if world > 1 and not dist.is_initialized():
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if device is not None:
            kw["device_id"] = device
        dist.init_process_group(backend, **kw)
    return world, rank, local


def barrier() -> None:
    import torch.distributed as dist
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(value: float, device="cpu") -> float:
    """The largest value any rank holds (the step time of the slowest rank)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device="cpu") -> float:
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shard_tensors(sizes: list[int], world: int, rank: int) -> list[int]:
    """Indices of the tensors rank `rank` decodes: greedy largest-first onto the least-loaded rank
    (ties to the lower rank), so every tensor is decoded by exactly one rank and the weights per
    rank differ by at most one tensor's size."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank")
    load = [0] * world
    owner = [0] * len(sizes)
    for i in sorted(range(len(sizes)), key=lambda i: (-sizes[i], i)):
        r = min(range(world), key=lambda r: (load[r], r))
        owner[i] = r
        load[r] += sizes[i]
    return [i for i in range(len(sizes)) if owner[i] == rank]


def shutdown() -> None:
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
