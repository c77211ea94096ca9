"""Host-side plumbing for running the loss data-parallel, one process per GPU.

Every token's target and KL row depend only on that token's own inputs (its
Q rows, the window keys before it, its idx row) and on its sequence's pool,
so ranks split the batch by whole sequences and run the three calls on their
share with nothing exchanged on the data path. What remains for the host:

* which sequences (or, for synthetic runs, which seed) a rank owns;
* the max over ranks of a device-timed duration (the slowest rank decides);
* turning per-rank losses, each a mean over that rank's valid rows, into the
  mean over the whole batch, and the factor that rescales a rank's dscores to
  match (both are linear in 1/N).

The collectives here act on a handful of host scalars after the path has run;
they work with any torch.distributed backend (nccl on GPUs, gloo on CPU).
"""
from __future__ import annotations

from typing import Tuple

__all__ = ["rank_seed", "split_sequences", "max_over_ranks", "global_mean_loss"]


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's synthetic batch: distinct per rank, fixed per run."""
    if rank < 0:
        raise ValueError(f"rank must be >= 0, got {rank}")
    return int(base_seed) + int(rank)


def split_sequences(B: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [start, stop) range of the B sequences that `rank` owns.

    The first B % world ranks take one extra sequence; a rank can own none
    when B < world (its range is then empty and it has no work)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world of size {world}")
    if B < 0:
        raise ValueError(f"B must be >= 0, got {B}")
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def _dist():
    import torch.distributed as dist
    return dist if dist.is_available() and dist.is_initialized() else None


def max_over_ranks(value: float, device=None) -> float:
    """Largest `value` over all ranks (the value itself without a process group)."""
    dist = _dist()
    if dist is None or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def global_mean_loss(local_loss: float, local_rows: int, device=None) -> Tuple[float, float]:
    """Batch-wide loss from per-rank ones, and this rank's dscores factor.

    Each rank's loss is coeff * sum(KL over its rows) / max(N_r, 1), with N_r
    its number of rows that have a valid slot. The batch-wide loss is
    coeff * sum_r sum(KL_r) / max(N, 1) with N = sum_r N_r, i.e.
    sum_r loss_r * max(N_r, 1) / max(N, 1). A rank's dscores carry the same
    1/max(N_r, 1), so multiplying them by max(N_r, 1) / max(N, 1) gives the
    batch-wide gradient. Returns (global_loss, dscores_factor)."""
    if local_rows < 0:
        raise ValueError(f"local_rows must be >= 0, got {local_rows}")
    n_r = max(int(local_rows), 1)
    kl_sum = float(local_loss) * n_r          # coeff * sum of this rank's KL rows
    rows = int(local_rows)
    dist = _dist()
    if dist is not None and dist.get_world_size() > 1:
        import torch
        t = torch.tensor([kl_sum, float(rows)], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        kl_sum, rows = float(t[0].item()), int(round(float(t[1].item())))
    n = max(rows, 1)
    return kl_sum / n, n_r / n
