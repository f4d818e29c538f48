"""Host-side logic of running the round on several GPUs.

Requests are independent through drafting and verification, and by default
the prefix cut is per engine (every GPU schedules its own batch against its
own cost table), so N GPUs run N independent batches with no collective on the
data path (weak scaling); the only collectives are then the timing
bookkeeping: a barrier around the timed region and MAX / SUM reductions of
per-rank numbers. Optionally one schedule spans every GPU's requests
(spec_round.GlobalSchedule): its single data-path collective is the
all-gather of the confidence logits, all_gather_rows below.
"""
from __future__ import annotations

import os
from datetime import timedelta
from typing import Tuple

import torch
import torch.distributed as dist

from . import workloads as wl


def env_ranks() -> Tuple[int, int, int]:
    """(world size, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0) -> Tuple[int, int, int]:
    """Joins the process group when WORLD_SIZE > 1 (NCCL on GPUs, gloo on CPU)."""
    world, rank, local = env_ranks()
    if world > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)
    elif backend == "nccl":
        torch.cuda.set_device(local)
    return world, rank, local


def rank_workload(w: wl.Workload, rank: int) -> wl.Workload:
    """Rank r's own batch: the same recipe with a rank-dependent seed."""
    return w if rank == 0 else wl.scaled(w, seed=w.seed + 1000003 * rank)


def _reduce(v: float, op, device) -> float:
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(v)
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(v: float, device="cpu") -> float:
    return _reduce(v, dist.ReduceOp.MAX, device)


def sum_over_ranks(v: float, device="cpu") -> float:
    return _reduce(v, dist.ReduceOp.SUM, device)


def all_gather_rows(t: torch.Tensor) -> torch.Tensor:
    """Every rank's t (same shape on every rank) stacked along dim 0 in rank
    order; t itself when there is one rank. Runs on the current stream."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return t
    parts = [torch.empty_like(t) for _ in range(dist.get_world_size())]
    dist.all_gather(parts, t.contiguous())
    return torch.cat(parts, 0)


def barrier() -> None:
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def finish() -> None:
    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
