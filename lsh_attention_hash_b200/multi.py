"""Host-side pieces of the one-process-per-GPU run (no data-path collective).

Every (b, h) slice goes through hash, sort, chunk attention and round merge on
its own, so N GPUs either run N independent replicas (weak scaling: each rank
its own batch) or split the B*H slices of one batch (strong scaling).  The only
cross-rank traffic is timing: the step time of a run is the maximum over the
ranks of their device-timed spans.
"""

from __future__ import annotations

from typing import List, Sequence, Tuple


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's synthetic inputs (weak scaling: each rank its own batch)."""
    return int(base_seed) * 1_000_003 + int(rank)


def slice_shard(B: int, H: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous range [lo, hi) of the B*H flattened (b, h) slices owned by `rank`
    when one batch is split over `world` ranks (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    n = B * H
    lo = rank * n // world
    hi = (rank + 1) * n // world
    return lo, hi


def shard_slices(B: int, H: int, rank: int, world: int) -> List[Tuple[int, int]]:
    """The (b, h) pairs of `slice_shard`."""
    lo, hi = slice_shard(B, H, rank, world)
    return [divmod(i, H) for i in range(lo, hi)]


def max_over_ranks(values: Sequence[float], device=None) -> List[float]:
    """Element-wise maximum over all ranks of the default process group (identity
    when torch.distributed is not initialised).  Every rank must call it."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()
