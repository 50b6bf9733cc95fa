"""Multi-process timing for the benchmark: every rank times its own replica
of the workload on its own GPU (no data-path collective); the job time is
the maximum over ranks and the throughput counts the work of all ranks."""
from __future__ import annotations

import torch
import torch.distributed as dist


def max_over_ranks(ms: float, device: torch.device | str = "cpu") -> float:
    """Largest elapsed time (ms) over all ranks of the default process group."""
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Units per second of the whole job: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / (ms_max / 1e3)
