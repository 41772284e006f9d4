"""Multi-GPU bookkeeping for decode replicas.

Every (batch row, kv head) item of a decode step is independent, so N GPUs
run N independent replicas of the step (one process per GPU) and exchange
nothing in the data path. The only collectives are the timing ones: the
slowest rank's time bounds the whole job, and the whole-job throughput is the
units all ranks processed divided by that time.
"""
from __future__ import annotations

import torch


def _dist():
    import torch.distributed as dist
    return dist if dist.is_available() and dist.is_initialized() else None


def world_size() -> int:
    d = _dist()
    return d.get_world_size() if d else 1


def max_over_ranks(x: float) -> float:
    """Maximum of x over all ranks (x itself without a process group)."""
    d = _dist()
    if d is None or d.get_world_size() == 1:
        return float(x)
    dev = (torch.device("cuda", torch.cuda.current_device()) if d.get_backend() == "nccl"
           else torch.device("cpu"))
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    d.all_reduce(t, op=d.ReduceOp.MAX)
    return float(t.item())


def barrier() -> None:
    d = _dist()
    if d is not None and d.get_world_size() > 1:
        d.barrier()


def whole_job_rate(units_per_rank: float, seconds_max: float, world: int | None = None) -> float:
    """Units per second of the whole job: every rank processed units_per_rank
    in at most seconds_max."""
    world = world_size() if world is None else world
    return world * units_per_rank / seconds_max
