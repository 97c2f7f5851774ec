"""Host-side aggregation of independent replicas (one process per GPU).

The decode-step hot path has no cross-sequence exchange, so N GPUs run N
independent replicas of the workload; the job's time is the slowest rank's and
its throughput is the sum of what every rank processed in that time.
"""
from __future__ import annotations

from typing import List, Sequence

import torch
import torch.distributed as dist


def max_over_ranks(values: Sequence[float], device=None) -> List[float]:
    """Element-wise maximum of `values` over all ranks (identity without a group)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def replica_throughput(units_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Units per second of the whole job: every rank did `steps` steps."""
    return world * units_per_step * steps / (max_ms / 1e3)
