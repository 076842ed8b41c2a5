"""Data-parallel plumbing: one process per GPU, each rank owning an independent batch of sequences.

KV-cache quantisation and decode attention work on (sequence, kv head) units that never read one another, so
the path shards across ranks with no exchange step on the data path.  Ranks meet only on the host side of a
measurement: a barrier on both sides of the timed region and one max-reduction of the elapsed time, so that
the job's time is that of its slowest rank.
"""
from __future__ import annotations

import datetime
import os

import torch


def world_from_env() -> tuple[int, int, int]:
    """(world size, rank, local rank) as a torch.distributed launcher exports them; (1, 0, 0) otherwise."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(world: int, backend: str = "nccl", device: torch.device | None = None, timeout_s: float = 120.0) -> None:
    """Join the process group when world > 1.  The short timeout makes a rank that never arrives an error."""
    if world <= 1:
        return
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if backend == "nccl" and device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def finish(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: torch.device | str = "cpu") -> float:
    """Largest x over all ranks (every rank gets it)."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_floats(x: float, world: int, device: torch.device | str = "cpu") -> list[float]:
    """x of every rank, in rank order (every rank gets the list)."""
    if world <= 1:
        return [float(x)]
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    out = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(out, t)
    return [float(o.item()) for o in out]


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's synthetic batch: every rank draws a batch of its own."""
    return int(base) + 1000 * int(rank)


def aggregate_rate(units_per_rank: float, slowest_seconds: float, world: int) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / slowest_seconds
