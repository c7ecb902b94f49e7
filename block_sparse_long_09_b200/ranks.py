"""Host-side plumbing for one process per GPU.

The QSA layer partitions by independent sequences: every rank runs the whole
path on its own seeded inputs and nothing crosses ranks on the data path.  Only
the timing is combined: the job's time is the slowest rank's device time, and
the job's throughput counts the units of every rank.  The process group carries
the barriers around the timed region and that max-reduction (NCCL on GPUs, gloo
in the CPU tests).
"""
from __future__ import annotations

import datetime
import os
from typing import Dict, Iterable, List, Optional

import torch


def env_ranks() -> Dict[str, int]:
    """rank, world size and local rank from the torchrun environment (1 process when unset)."""
    return {
        "rank": int(os.environ.get("RANK", "0")),
        "world": int(os.environ.get("WORLD_SIZE", "1")),
        "local": int(os.environ.get("LOCAL_RANK", "0")),
    }


def rank_seeds(rank: int) -> Dict[str, int]:
    """Seeds of a rank's own prefill and decode inputs: distinct problems per rank."""
    return {"prefill": rank, "decode": 100 + rank}


def init(backend: str, world: int, device: Optional[torch.device] = None, timeout_s: float = 120.0) -> bool:
    """Join the process group (from the env:// rendezvous) when world > 1; a short timeout
    makes ranks that wait on a missing peer fail instead of hanging."""
    if world <= 1:
        return False
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    torch.distributed.init_process_group(backend, **kw)
    return True


def barrier(world: int) -> None:
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(values: Iterable[float], world: int, device: Optional[torch.device] = None) -> List[float]:
    """Element-wise max over ranks of a few host floats (every rank gets the result)."""
    vals = [float(v) for v in values]
    if world <= 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device if device is not None else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.cpu().tolist()]


def job_throughput(world: int, units_per_rank: float, max_ms: float) -> float:
    """Units per second of the whole job: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / (max_ms / 1e3)


def finish(world: int) -> None:
    if world > 1 and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()
