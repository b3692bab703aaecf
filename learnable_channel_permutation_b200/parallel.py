"""Multi-GPU host logic: one process per GPU, layers sharded across ranks.

The layers of a calibration step are independent problems (each has its own
W, L, P, dL and loss), so N GPUs run N independent layer-steps with no
collective on the data path; the only communication is the timing reduction
(the job time is the maximum over ranks).  Used by bench.py under torchrun and
tested with the gloo backend on CPU.
"""
from __future__ import annotations

import copy
from typing import List, Sequence

import torch
import torch.distributed as dist

from . import synth


def rank_workload(wl: synth.Workload, rank: int) -> synth.Workload:
    """The workload rank `rank` runs: same shapes, its own seed (an independent layer)."""
    out = copy.deepcopy(wl)
    out.seed = wl.seed + rank
    return out


def shard(items: Sequence, rank: int, world: int) -> List:
    """Round-robin share of `items` (e.g. the layers of a model) for `rank`."""
    return [x for i, x in enumerate(items) if i % world == rank]


def max_over_ranks(values: Sequence[float], device=None) -> List[float]:
    """Element-wise maximum of per-rank values (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(units_per_rank: int, world: int, max_ms: float) -> float:
    """Units per second of the whole job: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)
