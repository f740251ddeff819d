"""Process-group plumbing for running the path on N GPUs of one node.

The path shards over independent (batch, kv-head) problems with no exchange,
so N ranks each run their own shard (weak scaling) and only the timing is
reduced: the job time is the maximum over ranks.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def world() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> bool:
    """Initialises the default process group when WORLD_SIZE > 1."""
    rank, local, ws = world()
    if ws <= 1 or dist.is_initialized():
        return dist.is_initialized()
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    kw = {}
    if backend == "nccl":
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return True


def barrier() -> None:
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device="cpu") -> float:
    """The maximum of a per-rank scalar (e.g. a device-timed duration)."""
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(seed: int, rank: int) -> int:
    """Seed of this rank's shard: rank 0 keeps the workload's own seed."""
    return seed + 7919 * rank


def finalize() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
