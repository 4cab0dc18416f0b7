"""Data-parallel exchange of the POET layer (one process per GPU).

The layer is token-parallel: every rank runs its own tokens through replicated
W0 and skew parameters, so the only exchange is the sum of the packed-skew
gradients over ranks (W0 is fixed and has no gradient; merge and resample are
replicated deterministically from (seed, layer, side, epoch)).  The loss of a
step is the sum over all ranks' tokens, whose gradient is the sum of the
per-rank gradients.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def allreduce_gradients_(flat: torch.Tensor, group=None) -> torch.Tensor:
    """Sum a flat gradient buffer over the ranks of `group`, in place."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    return flat


def max_over_ranks(values, device=None, group=None) -> list[float]:
    """Element-wise maximum of a list of floats over the ranks (timings)."""
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1):
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return [float(x) for x in t.cpu()]
