"""Multi-GPU helpers: token-sharded static calibration.

The forward shards by tokens (rows of X) with no collective: every rank holds
the quantized weights and writes its own rows of Y.  Calibration over data that
is sharded the same way needs one exchange so that all ranks quantize with the
same static scales (SegQuant: scales are fixed offline, Spanish technical
summary 1 "compiler gap" and section 3 item 4).

Rounding to fp32 is monotone, so the maximum over ranks of the local scales
fl(P_r / 127) equals fl(max_r P_r / 127): an all-reduce(MAX) of the 2*J local
scales gives exactly the scales of the unsharded calibration rows.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def allreduce_scales_(s_pos: torch.Tensor, s_neg: torch.Tensor, group=None) -> None:
    """In place: s_pos, s_neg <- element-wise max over the ranks of `group`."""
    both = torch.cat([s_pos.reshape(-1), s_neg.reshape(-1)])
    dist.all_reduce(both, op=dist.ReduceOp.MAX, group=group)
    J = s_pos.numel()
    s_pos.copy_(both[:J].view_as(s_pos))
    s_neg.copy_(both[J:].view_as(s_neg))


def calibrate_sharded(x_local: torch.Tensor, kseg: Sequence[int], group=None,
                      stream=None, s_pos: Optional[torch.Tensor] = None,
                      s_neg: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Static DualScale scales of the union of every rank's calibration rows.

    Each rank calibrates its own rows on its GPU, then the 2*J scales are
    all-reduced with MAX (NCCL over NVLink for CUDA tensors).  ``s_pos`` /
    ``s_neg`` (fp32 [J]) receive the scales when given."""
    from . import calibrate
    s_pos, s_neg = calibrate(x_local, kseg, s_pos, s_neg, stream=stream)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        allreduce_scales_(s_pos, s_neg, group)
    return s_pos, s_neg


def calibrate_hadamard_sharded(x_local: torch.Tensor, kseg: Sequence[int], group=None,
                               stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The same for the block-Hadamard variant: the transform acts within each
    row (blocks of 16 along K), so each rank's scales of its own rows of XH
    all-reduce with MAX to the scales of all rows of XH."""
    from . import calibrate_hadamard
    s_pos, s_neg = calibrate_hadamard(x_local, kseg, stream=stream)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        allreduce_scales_(s_pos, s_neg, group)
    return s_pos, s_neg


def shard_rows(M: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous row range [r0, r1) of X owned by `rank` (balanced to one row)."""
    base, extra = divmod(M, world)
    r0 = rank * base + min(rank, extra)
    return r0, r0 + base + (1 if rank < extra else 0)
