"""Process-level plumbing for running the step on one or more GPUs of a node.

One process per GPU.  The step has no exchange between sequences, so ranks
run independent batches (weak scaling: every rank owns its own sequences and
KV cache) and the only collectives are the host-side barrier and the
max-over-ranks reduction of the measured time.
"""
from __future__ import annotations

import datetime
import os
from typing import Optional

import torch
import torch.distributed as dist


def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: Optional[str] = None, timeout_s: int = 120):
    """Initialises the process group when WORLD_SIZE > 1; returns
    (rank, world, local_rank, device)."""
    rank, world, local = env_rank()
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        device = torch.device("cuda", local)
    else:
        device = torch.device("cpu")
    if world > 1 and not dist.is_initialized():
        backend = backend or ("nccl" if device.type == "cuda" else "gloo")
        kw = {}
        if backend == "nccl":
            kw["device_id"] = device
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return rank, world, local, device


def barrier(device=None):
    if dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(x: float, device) -> float:
    """Max of a host scalar over all ranks (identity on one process)."""
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device) -> float:
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shard(n_items: int, rank: int, world: int):
    """Contiguous share [lo, hi) of n_items for this rank (sizes differ by at
    most one)."""
    base, extra = divmod(n_items, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def weak_throughput(units_per_rank, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time."""
    total = float(sum(units_per_rank))
    return total / max_seconds if max_seconds > 0 else 0.0


def finalize():
    if dist.is_initialized():
        dist.destroy_process_group()
