"""Replica (data-parallel) bookkeeping for the decode benchmark.

The batch-1 decode step does not shard: every GPU decodes its own independent
sequence (one process per GPU), so there is no collective on the data path.  The
only cross-rank steps are around the timed region: a barrier before and after it,
and the maximum of the ranks' device times, from which rank 0 reports the
whole-job throughput (tokens of all ranks / slowest rank's time).
"""
from __future__ import annotations

import torch


def barrier(world: int) -> None:
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(values, world: int, device=None) -> list[float]:
    """Elementwise maximum of `values` over all ranks (a no-op for one rank)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_tokens_per_s(steps: int, batch: int, world: int, max_ms: float) -> float:
    """Whole-job decode throughput: every rank decodes steps * batch tokens; the job
    takes as long as its slowest rank."""
    if max_ms <= 0:
        raise ValueError("timed region must be positive")
    return steps * batch * world / (max_ms / 1e3)
