"""Multi-GPU host logic: one process per GPU.

Two ways to split a calibration step across ranks:

* by layer: the layers of a step are independent problems (each has its own
  W, L, P, dL and loss), so N GPUs run N independent layer-steps with no
  collective on the data path; the only communication is the timing reduction
  (the job time is the maximum over ranks).  bench.py runs this under torchrun.
* by token: the loss is a mean over the calibration tokens, so one layer's
  batch of T tokens splits into contiguous shards (PermLLM summary,
  "Implementation details": 7B trained on 4 GPUs, 13B on 8).  Each rank runs
  lcp_step_shard on its tokens, with the mean over the global T, which stops
  before the Sinkhorn reverse pass; one all-reduce sums every layer's dP and
  loss; every rank then runs the Sinkhorn reverse pass on the sums and holds the
  whole batch's dL.  dP is C_in * B floats a layer (1 MB for a 4096-channel
  layer at B = 64), so the exchange is one small NCCL all-reduce.

Tested with the gloo backend on CPU (world size 2), with the oracle standing in
for the GPU step.
"""
from __future__ import annotations

import copy
from typing import Callable, List, Optional, Sequence

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


def token_shard(tokens: int, rank: int, world: int) -> slice:
    """Contiguous share of `tokens` calibration tokens for `rank`; shard sizes
    differ by at most one and cover every token once, in rank order."""
    base, extra = divmod(tokens, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


def allreduce_sum_(tensors: Sequence[torch.Tensor], group=None) -> Sequence[torch.Tensor]:
    """Replace every tensor by its sum over the ranks, with one all-reduce of
    their concatenation (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return tensors
    flat = torch.cat([t.reshape(-1) for t in tensors])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    off = 0
    for t in tensors:
        n = t.numel()
        t.copy_(flat[off:off + n].view_as(t))
        off += n
    return tensors


def token_parallel_step(run_shard: Callable[[], None], finish: Callable[[], None], dP: Sequence[torch.Tensor],
                        losses: Sequence[torch.Tensor], group=None) -> None:
    """One token-parallel step: `run_shard()` fills this rank's dP (one tensor
    a layer) and losses (one-element tensors) for its shard, normalised by the
    global token count; both are summed over the ranks in place; `finish()`
    then runs the Sinkhorn reverse pass on the sums.  Every rank takes the same
    collective steps in the same order."""
    run_shard()
    allreduce_sum_(list(dP) + list(losses), group)
    finish()


class TokenParallelStep:
    """The GPU form of token_parallel_step for a set of layers: ``layers`` are
    this rank's tensors (as binding.alloc_outputs makes them) whose X hold its
    token shard; ``total_tokens`` is the whole batch.  ``run()`` leaves in every
    layer the whole batch's loss and dL."""

    def __init__(self, layers, block: int, n: int, m: int, iters: int, tau: float, total_tokens: int,
                 flags: int = 0, group=None):
        from . import binding
        self.b = binding
        self.step = binding.Step(layers, block, n, m, iters, tau, flags=flags)
        self.layers, self.tau, self.iters, self.total, self.group = list(layers), tau, iters, total_tokens, group
        self.dP = [torch.empty_like(d["L"]) for d in layers]
        self.ckpt = [torch.empty(d["L"].shape[0], iters, 2, block, dtype=torch.float32, device=d["L"].device)
                     for d in layers]

    def run(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        b = self.b

        def shard():
            b.step_shard(self.step, self.total, self.dP, self.ckpt, stream)

        def finish():
            for d, dP, ck in zip(self.layers, self.dP, self.ckpt):
                b.sinkhorn_bwd(d["L"], ck, dP, d["dL"], self.tau, self.iters)

        token_parallel_step(shard, finish, self.dP, [d["loss"][:1] for d in self.layers], self.group)
