"""Rank plumbing of a multi-GPU run: which units a rank processes, how its
timings combine into whole-job numbers.

The method's units, the (b, h) heads of independent clouds, need no data
exchange ("FLARE++: Low-rank attention with dynamic attention routing",
"Méthodologie : FLARE++": every head's encode-decode reads only that head's
tokens), so a job over N ranks gives each rank its own batch element
b = rank and runs no collective on the data path.  The only collectives are
host-side: a barrier around the timed region and a max over the ranks' device
times, so that the slowest rank sets the job's time.

Backend-agnostic: the same functions run over NCCL on GPUs and over gloo on
CPU (how the tests exercise them).
"""
from __future__ import annotations

import os
from dataclasses import dataclass


@dataclass(frozen=True)
class RankEnv:
    rank: int
    world: int
    local: int

    @staticmethod
    def from_environ() -> "RankEnv":
        """RANK / WORLD_SIZE / LOCAL_RANK as torchrun sets them (a lone process is rank 0 of 1)."""
        return RankEnv(int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
                       int(os.environ.get("LOCAL_RANK", 0)))


def rank_workload(base, world: int, heads: int | None = None):
    """The job's workload seen from one rank: the batch grows to `world`
    (one cloud per rank), the per-rank shape is the base workload's."""
    from . import inputs

    H = heads or base.H
    return inputs.Workload(base.name, world, H, base.N, base.M, base.D, base.dtype, base.kind, base.index)


def rank_batch_element(env: RankEnv) -> int:
    """Batch element this rank processes (weak scaling: one cloud per rank)."""
    return env.rank


def max_over_ranks(x: float, env: RankEnv, device=None) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if env.world == 1:
        return float(x)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, env: RankEnv, ms_per_step_max: float) -> float:
    """Whole-job throughput: the tokens all ranks processed in one step over
    the slowest rank's step time."""
    return tokens_per_rank * env.world / (ms_per_step_max * 1e-3)


def reports(env: RankEnv) -> bool:
    """Only rank 0 prints the job's line."""
    return env.rank == 0
