"""Host-side logic of the branch-parallel multi-GPU path.

Branches are independent (SpecOPD review (jaehun.me) §3.1: the joint sample
factorises over branches), so a batch shards by whole branches with no data
exchange; the only exchange the method defines is the distributed
normalisation of review §3.2 ("numerical consistency"): numerators and
counts are gathered separately over the ranks and the loss is normalised
once, so loss weights do not depend on how many positions each rank scored.

With torch.distributed (NCCL on GPUs, gloo on CPU):
  * global_count(): all-reduce of the per-rank position counts, done once
    per step before the E2E-TV call; the result is the norm_count of every
    rank's call, so every rank's gradient already carries the global 1/N.
  * global_numer(): all-reduce of the per-rank prefix-product sums (the
    `numer` output of specopd_e2e_tv) after the call;
  * global_loss(): that sum, then the library's specopd_e2e_tv_finalize,
    which writes loss = 1 - sum / N on the device.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def shard_branches(nbranch: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous branch range (start, count) of `rank`; counts differ by at
    most one, and every branch is owned by exactly one rank."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("bad rank/world")
    base, extra = divmod(nbranch, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def global_count(local_positions: int, group=None, device="cpu") -> int:
    """Sum of the per-rank supervised-position counts (the loss divisor)."""
    t = torch.tensor([int(local_positions)], dtype=torch.int64, device=device)
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, group=group)
    return int(t.item())


def global_numer(numer: torch.Tensor, group=None) -> torch.Tensor:
    """Sum over ranks of the prefix-product sums, in place.  `numer` is this
    rank's fp64 numerator (1 element, the `numer` output of specopd_e2e_tv)."""
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(numer, group=group)
    return numer


def global_loss(numer: torch.Tensor, count: int, loss: torch.Tensor = None, group=None,
                stream=None) -> torch.Tensor:
    """loss = 1 - (sum over ranks of the prefix-product sums) / count, on the
    device: the all-reduce of `numer` (in place, a CUDA tensor), then the
    library's specopd_e2e_tv_finalize.  Returns the fp32 loss (1 element)."""
    from . import api
    global_numer(numer, group)
    return api.specopd_e2e_tv_finalize(numer, count, loss=loss, stream=stream)
