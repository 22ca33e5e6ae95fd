"""Data-parallel plumbing of the layer's training step: one process per GPU.

Graphs are independent, so ranks split the batch and run the layer on their
own graphs with no exchange on the data path (weak scaling: every rank keeps
the per-GPU batch).  The one collective is the sum of the weight gradients
over ranks after each backward, as in any data-parallel training step; on
GPUs it runs on NCCL over NVLink / NVSwitch, on CPU (tests) on gloo.  Step
times are reported as the maximum over ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of the synthetic batch of `rank`: distinct graphs on every rank."""
    return base_seed + 100 * rank


def allreduce_weight_grads(flat: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the flat fp32 weight-gradient buffer over all ranks, in place."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    return flat


def max_over_ranks(value: float, device: torch.device | str = "cpu", group=None) -> float:
    """The largest `value` over all ranks (every rank gets the same number)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
