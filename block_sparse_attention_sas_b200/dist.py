"""Process-group plumbing for running independent SAS problems on several GPUs.

Every (batch, KV head) unit of gated sparse attention is independent: the
gate softmax, the selection, the forward, the backward (dK/dV only sum within
a unit) and the decode never read another unit's data. So several GPUs run
disjoint units with no collective on the data path; the only collectives are
the timing barrier and the max over ranks of the measured time.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_rank() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment (0, 0, 1 without it)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str, timeout_s: float = 120.0) -> bool:
    """Initialise the default process group when WORLD_SIZE > 1. Returns True if it did."""
    _, _, world = env_rank()
    if world <= 1 or dist.is_initialized():
        return dist.is_initialized()
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return True


def shard_range(n_units: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous [lo, hi) share of n_units for `rank`; shares differ by at most one."""
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's own synthetic batch (rank 0 keeps the workload's seed)."""
    return base_seed + 1000003 * rank


def barrier(device: torch.device | None = None) -> None:
    if dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value: float, device: torch.device | None = None) -> float:
    """Max of a per-rank scalar (used for timings: the slowest rank sets the step time)."""
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device: torch.device | None = None) -> float:
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shutdown() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
