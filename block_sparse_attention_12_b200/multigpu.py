"""Host-side plumbing of the multi-GPU benchmark (one process per GPU).

Every (b, h, q-block) row of AB-Attention is independent and the plan's
uniforms are counter-based on (b, h, q-block, KV block), so the work shards
across GPUs with no data-path collective: each rank runs whole layers (or
any subset of heads) on its own GPU and the plan it builds equals the
corresponding rows of a single-GPU plan.  The only collectives are a
barrier around the timed region and a max-reduce of the per-rank time.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def max_over_ranks(ms: float, device=None) -> float:
    """The slowest rank's time (the job's time); identity without a process group."""
    if not (dist.is_available() and dist.is_initialized()):
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (units per second)."""
    return units_per_rank * world / (ms_max / 1e3)


def head_shard(H: int, rank: int, world: int) -> range:
    """Contiguous heads [lo, hi) owned by `rank` when H heads are split over
    `world` ranks (the first H % world ranks take one extra head)."""
    base, extra = divmod(H, world)
    lo = rank * base + min(rank, extra)
    return range(lo, lo + base + (1 if rank < extra else 0))
