"""Multi-process plumbing for the RPTQ path (torch.distributed; NCCL on GPUs, gloo on CPU).

The path shards by tokens: every rank calibrates, quantizes and dequantizes its own tokens.
The one exchange is calibration: the global per-channel max / min over all ranks' calibration
tokens is the elementwise MAX / MIN of the per-rank statistics (RPTQ article, text after
Fig. 2: statistics over the whole calibration set).  KMeans then runs on every rank on identical
statistics and, being deterministic, yields identical clusters everywhere.
"""
from __future__ import annotations

import os

import torch
import torch.distributed as dist


def world() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the launcher's environment (1 process if unset)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def allreduce_minmax(ch_max: torch.Tensor, ch_min: torch.Tensor, group=None) -> None:
    """In place: ch_max <- max over ranks, ch_min <- min over ranks (no-op on one process)."""
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return
    dist.all_reduce(ch_max, op=dist.ReduceOp.MAX, group=group)
    dist.all_reduce(ch_min, op=dist.ReduceOp.MIN, group=group)


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The largest `value` of all ranks (timings are reported as the slowest rank)."""
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def sum_over_ranks(value: float, device=None, group=None) -> float:
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return float(t.item())
