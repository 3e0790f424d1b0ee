"""Process-per-GPU plumbing for the batch-sharded path.

Every (batch, head) pair is independent in all three forms of the method (the
state of one head never reads another head's tokens), so several GPUs split
the batch: rank r owns sequences [start, stop) of the global batch and never
exchanges data with the other ranks.  The only collectives are for timing:
a barrier around the timed region and the maximum of the per-rank times.
Ranks are launched one per GPU (torchrun); NCCL is used on GPUs and gloo on
CPU (tests).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def shard(total: int, world: int, rank: int) -> tuple[int, int]:
    """Balanced contiguous range [start, stop) of `total` items for `rank`."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def env_world() -> tuple[int, int, int]:
    """(world_size, rank, local_rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0, device=None) -> None:
    """Join the process group named by the environment (no-op for one rank)."""
    world, rank, _ = env_world()
    if world > 1 and not dist.is_initialized():
        kw = {"device_id": device} if device is not None else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def barrier() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device="cpu") -> float:
    """Largest value of `x` over all ranks (x itself for one rank)."""
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def finalize() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
