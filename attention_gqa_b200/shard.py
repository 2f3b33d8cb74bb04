"""Host-side helpers for running the attention path with one process per GPU.

The path has no exchange step: every sequence of a batch is independent (and
so is every key/value-head group with its 8 query heads and sinks), so several
GPUs either run independent replicas or split the batch, with no collective on
the data path. The only cross-process operations are set-up and the reduction
of timings (the slowest rank sets the time of a step).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def batch_range(batch: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous, balanced slice [lo, hi) of `batch` sequences owned by `rank`."""
    if world < 1 or not 0 <= rank < world or batch < 0:
        raise ValueError("bad shard request: batch=%d rank=%d world=%d" % (batch, rank, world))
    base, rem = divmod(batch, world)
    lo = rank * base + min(rank, rem)
    return lo, lo + base + (1 if rank < rem else 0)


def init_from_env(backend: str, device: torch.device | None = None,
                  timeout_s: float = 120.0) -> tuple[int, int]:
    """Joins the process group described by RANK / WORLD_SIZE / MASTER_* (as set
    by torch.distributed.run). A short timeout makes ranks that wait on a dead
    peer fail instead of hanging. Returns (rank, world)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1 and not dist.is_initialized():
        kwargs = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if device is not None and backend == "nccl":
            kwargs["device_id"] = device
        dist.init_process_group(backend, **kwargs)
    return rank, world


def max_over_ranks(values, device: torch.device | str = "cpu") -> list[float]:
    """Element-wise maximum of `values` over all ranks (identity with one rank).
    `device` must suit the backend: a CUDA device for NCCL, the CPU for gloo."""
    vals = [float(v) for v in values]
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu().tolist()]
