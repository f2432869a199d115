"""Host-side helpers for running the operator on several GPUs of one node.

The operator has no exchange step: every (batch entry, head) map is an
independent problem.  N GPUs therefore take disjoint, contiguous slices of
the batch with no collective on the data path; the process group is used
only to line the ranks up before and after a timed region and to take the
maximum of their times.
"""
from __future__ import annotations

import os

import torch
import torch.distributed as dist


def shard_range(units: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous slice [begin, end) of `units` owned by `rank` (sizes differ by at most 1)."""
    if world < 1 or not 0 <= rank < world or units < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(units, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def env_rank() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the launcher's environment (1 process: 0, 0, 1)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def max_over_ranks(value: float, device: torch.device | None = None) -> float:
    """Maximum of a per-rank float over the process group (identity without one)."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device: torch.device | None = None):
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()
