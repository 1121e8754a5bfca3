"""Multi-GPU plumbing for the tied NVFP4 tensor scale.

The hot path shards without communication: tensors, rows and MoE experts are
independent, so replicas (one process per GPU) need no collective.  The one
exchange the method has appears when a tie group's weights are themselves
sharded across GPUs (tensor or fully-sharded data parallelism): the group's
amax -- and so its FP32 tensor scale, shared by the projections an engine fuses
(QATFactory project page, Method, "Numerics") -- is the max over every shard.
That is one all-reduce(MAX) of one FP32 per group between qf_amax_tied and
qf_fakequant, over NCCL (NVLink / NVSwitch) on GPUs or gloo on CPU.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch
import torch.distributed as dist


def reduce_group_amax(group_amax: torch.Tensor, group=None) -> torch.Tensor:
    """In place: group_amax <- max over all ranks of group_amax (FP32, exact)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(group_amax, op=dist.ReduceOp.MAX, group=group)
    return group_amax


def fold_tracked(group_amax: torch.Tensor, tracked: Optional[torch.Tensor]) -> torch.Tensor:
    """In place: tracked <- max(tracked, group_amax), then group_amax <- tracked, the
    value the step quantizes with (the tracked amax is a running max kept across
    steps).  With tracked None, group_amax is left as it is."""
    if tracked is not None:
        torch.maximum(tracked, group_amax, out=tracked)
        group_amax.copy_(tracked)
    return group_amax


def amax_tied_sharded(xs: Sequence[torch.Tensor], groups: Sequence[int],
                      group_amax: torch.Tensor, tracked: Optional[torch.Tensor] = None,
                      group=None, stream=None) -> torch.Tensor:
    """Tied amax of tie groups whose tensors are sharded across the ranks of `group`:
    the local qf_amax_tied, then the all-reduce(MAX); `tracked` is updated with the
    global value, so every rank quantizes with the same tensor scale."""
    from .binding import qf_amax_tied
    qf_amax_tied(xs, groups, group_amax, None, stream)
    reduce_group_amax(group_amax, group)
    return fold_tracked(group_amax, tracked)
