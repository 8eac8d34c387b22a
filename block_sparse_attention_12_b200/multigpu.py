"""Host-side plumbing of the multi-GPU paths (one process per GPU).

Every (b, h, q-block) row of AB-Attention is independent and the plan's
uniforms are counter-based on (b, h, q-block, KV block), so the work shards
across GPUs with no exchange inside the op:
  * weak scaling: each rank runs whole layers on its own GPU; the only
    collectives are a barrier around the timed region and a max-reduce of
    the per-rank time;
  * head sharding (strong scaling of one layer): each rank holds a
    contiguous slice of the layer's heads, plans it with the slice's first
    global head as `head_offset` (so its plan equals those rows of the
    single-GPU plan) and runs the forward; one all-gather then assembles O
    on every rank.
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


def gather_heads(O_local: torch.Tensor, H: int, world: int, group=None) -> torch.Tensor:
    """All-gather of per-rank head slices [B, h_r, N, d] (the slices of
    head_shard) into the whole layer's [B, H, N, d] on every rank.  The
    slices are padded to the largest shard, as an all-gather needs equal
    sizes."""
    if world == 1:
        return O_local
    B, _, N, d = O_local.shape
    hmax = -(-H // world)
    pad = O_local.new_zeros(B, hmax, N, d)
    pad[:, :O_local.shape[1]] = O_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    out = O_local.new_empty(B, H, N, d)
    for r in range(world):
        hs = head_shard(H, r, world)
        out[:, hs.start:hs.stop] = parts[r][:, :len(hs)]
    return out
