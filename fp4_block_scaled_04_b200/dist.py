"""Host-side plumbing for running the quantizers on several GPUs.

Every block of every recipe is independent (Qiita NVFP4 note, "Blockwise";
Ultralytics glossary "FP4の仕組み"), so the path shards without exchanging
data.  What several ranks do share is:

* the per-tensor amax when ONE tensor is split across ranks: the second-level
  FP32 scale is computed from the amax of the whole tensor (Qiita note,
  "scaleの導出"), so each rank reduces its shard's amax and the ranks agree on
  the maximum with a 4-byte all-reduce before they quantize;
* the timing of a step, which is the slowest rank's.

Shards are contiguous row ranges whose boundaries fall on multiples of
``align`` rows: 16 keeps the column-wise 16-row blocks and the 16x16 tiles
whole, 128 also keeps the 128x4 swizzled scale tiles whole.  With such
boundaries the shards' outputs are slices of the whole tensor's outputs
(row-wise codes and scales by rows, column-wise codes by their byte columns).

Nothing here computes a step of the method: the ranks call the C ABI for that.
This module works with any ``torch.distributed`` backend (``nccl`` on GPUs,
``gloo`` for the host-side tests).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def world():
    """(world_size, rank) of the default process group, (1, 0) without one."""
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(), dist.get_rank()
    return 1, 0


def shard_rows(rows: int, world_size: int, rank: int, align: int = 16):
    """[start, stop) of ``rank``'s contiguous row shard.

    ``rows`` must be a multiple of ``align``; the ``rows // align`` aligned
    groups are dealt out as evenly as possible, the first ranks taking one
    more group when they do not divide evenly.  A rank may get an empty shard
    (``start == stop``) when there are fewer groups than ranks.
    """
    if align <= 0 or rows < 0 or rows % align:
        raise ValueError(f"rows={rows} is not a multiple of align={align}")
    if world_size <= 0 or not 0 <= rank < world_size:
        raise ValueError(f"rank {rank} outside world of {world_size}")
    groups = rows // align
    base, extra = divmod(groups, world_size)
    start = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    return start * align, (start + count) * align


def global_amax(local_amax: torch.Tensor, group=None) -> torch.Tensor:
    """All-reduce MAX of a 1-element FP32 amax tensor, in place; returns it.

    ``local_amax`` lives where the backend wants it (a CUDA tensor for
    ``nccl``, a CPU tensor for ``gloo``).  Without a process group this is
    the identity.
    """
    if local_amax.numel() != 1 or local_amax.dtype != torch.float32:
        raise ValueError("global_amax expects a 1-element float32 tensor")
    ws, _ = world()
    if ws > 1:
        dist.all_reduce(local_amax, op=dist.ReduceOp.MAX, group=group)
    return local_amax


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The largest ``value`` over all ranks (for step times)."""
    ws, _ = world()
    if ws == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def aggregate_gbs(bytes_per_rank_step: int, world_size: int, steps: int, max_ms: float) -> float:
    """Whole-job GB/s: the bytes all ranks moved over the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("time must be positive")
    return world_size * bytes_per_rank_step * steps / (max_ms * 1e-3) / 1e9
