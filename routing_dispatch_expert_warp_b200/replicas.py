"""Data-parallel replicas: the job's load record.

Each GPU holds every expert and runs the whole layer on its own tokens; at EP = 1 the layer
has no exchange step.  The only collective is for the job's record of the layer ("MoE expert
parallelism needs measurements before launch", "Mean expert load proves almost nothing": one
record per layer for the job).  Each replica adds its routed and kept counts to everyone's
(an all-reduce SUM of 2E int32) and shares its own record (an all-gather).  Then one kernel
(moe_load_stats_merge) computes the record of the union of the replicas' picks.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import moe_load_stats_merge, stats_buffer


def gather_counts(routed_counts: torch.Tensor, kept_counts: torch.Tensor,
                  record: torch.Tensor, group=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Collective plumbing, called by every rank of `group` in the same order: returns
    (routed summed over the ranks [E], kept summed [E], every rank's record stacked
    [world, record bytes]).  The rank's own buffers are not modified."""
    import torch.distributed as dist
    E = routed_counts.numel()
    counts = torch.cat([routed_counts.reshape(-1), kept_counts.reshape(-1)])
    dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    world = dist.get_world_size(group)
    flat = torch.empty(world * record.numel(), dtype=record.dtype, device=record.device)
    dist.all_gather_into_tensor(flat, record.reshape(-1).contiguous(), group=group)
    return counts[:E], counts[E:], flat.view(world, record.numel())


def job_load_stats(cfg, bufs, group=None, host: bool = True,
                   out: Optional[torch.Tensor] = None) -> Optional[dict]:
    """The job's record of one layer over every replica of `group` (each rank calls it after
    its own layer forward wrote bufs.routed_counts, bufs.kept_counts and bufs.stats).  Returns
    the record as a dict on every rank when host=True; the device record is in `out`."""
    routed, kept, recs = gather_counts(bufs.routed_counts, bufs.kept_counts, bufs.stats, group)
    if out is None:
        out = stats_buffer(bufs.stats.device)
    return moe_load_stats_merge(cfg, routed, kept, recs, out, host)
