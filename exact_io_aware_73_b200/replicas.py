"""Multi-GPU scaffolding: independent replicas, one process per GPU.

Every (batch, head, query-tile) unit of attention is independent, so
running on N GPUs needs no data exchange.  By default each rank computes a
whole problem of its own (its own seeded inputs) and the job's throughput is
the sum of the ranks' work over the slowest rank's time.  Alternatively the
B*H heads of one problem are split into contiguous ranges (head_shard), each
rank computing its range with K and V of its heads only.  ``torch.distributed``
is used only for a barrier and for the max-over-ranks of the device timings.
Nothing here touches tensors of the attention itself.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist

# Per-rank seed stride: ranks draw disjoint, reproducible input streams.
SEED_STRIDE = 7919


def env_ranks():
    """(world, rank, local_rank) from the launcher's environment."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return world, rank, local


def init(backend: str, world: int, device=None, timeout_s: int = 120):
    """Join the process group (only when world > 1)."""
    if world > 1 and not dist.is_initialized():
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if device is not None and backend == "nccl":
            kw["device_id"] = device
        dist.init_process_group(backend, **kw)


def rank_seed(seed: int, rank: int) -> int:
    return int(seed) + SEED_STRIDE * int(rank)


def barrier(world: int):
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device="cpu") -> float:
    """The maximum of a per-rank scalar (e.g. elapsed device time)."""
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def head_shard(bh: int, world: int, rank: int):
    """The contiguous range of the B*H heads of one problem that a rank
    computes when one problem is split over ranks: (first head, count).
    Heads are independent (no key or value crosses heads), so the ranks'
    outputs tile the single-GPU output exactly; the first bh % world ranks
    take one head more."""
    bh, world, rank = int(bh), int(world), int(rank)
    base, extra = divmod(bh, world)
    first = rank * base + min(rank, extra)
    return first, base + (1 if rank < extra else 0)


def job_throughput(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job rate: every rank's units over the slowest rank's time."""
    return world * float(units_per_rank) / float(max_seconds)


def finish(world: int):
    if world > 1 and dist.is_initialized():
        dist.destroy_process_group()
