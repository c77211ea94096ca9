"""Host-side plumbing for running the loss data-parallel, one process per GPU.

Every token's target and KL row depend only on that token's own inputs (its
Q rows, the W-1 window keys before it, its idx row) and on its sequence's
pool. So ranks can split a batch two ways:

* by whole sequences (``split_sequences``): each rank runs the three calls on
  its share, nothing is exchanged on the data path, and per-rank losses are
  combined afterwards (``global_mean_loss``);
* by token range within every sequence (``token_ranges``), for batches with
  fewer sequences than ranks (one long sequence): a rank holds its positions'
  Q, idx, scores, valid and doc_start rows, the W-1 window keys before its
  first position (the halo) and the whole pool, and runs the range calls.
  The one exchange step is N, the batch's count of rows with a valid slot,
  which every rank's dscores are normalised by: each rank counts its rows on
  the device, one all-reduce of that integer gives N, and the KL call reads it
  from device memory (``sharded_distill_loss``).

Also here: per-rank seeds for synthetic runs and the max over ranks of a
device-timed duration. The collectives work with any torch.distributed
backend (nccl on GPUs, gloo on CPU).
"""
from __future__ import annotations

from typing import Sequence, Tuple

__all__ = ["rank_seed", "split_sequences", "max_over_ranks", "global_mean_loss", "token_cost",
           "token_ranges", "halo_rows", "range_views", "sharded_distill_loss"]


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


def token_cost(S: int, cr: int, K: int, W: int):
    """Relative work of each position t of a sequence: its window keys plus
    the compressed blocks it can select, min(W, t+1) + min(K, (t+1)//cr)
    (each costs 2*H*D flops; a sparse selection can leave fewer, never more)."""
    import numpy as np
    t = np.arange(S, dtype=np.int64)
    return np.minimum(W, t + 1) + np.minimum(K, (t + 1) // cr)


def token_ranges(S: int, world: int, cost=None) -> Sequence[Tuple[int, int]]:
    """[t_begin, t_end) for every rank: contiguous, covering 0..S-1, each
    non-empty when S >= world. With ``cost`` (per position, e.g. token_cost)
    the cut points split the cumulative cost evenly, so the later positions,
    which select more blocks, are spread over more ranks; else equal
    lengths."""
    if world < 1 or S < 1:
        raise ValueError(f"need world >= 1 and S >= 1, got world={world} S={S}")
    import numpy as np
    if cost is None:
        cuts = [(S * r) // world for r in range(world + 1)]
    else:
        c = np.cumsum(np.asarray(cost, dtype=np.float64))
        if c.shape != (S,):
            raise ValueError("cost must hold one value per position")
        cuts = [0]
        for r in range(1, world):
            t = int(np.searchsorted(c, c[-1] * r / world, side="left")) + 1
            # keep every range non-empty
            t = max(t, cuts[-1] + 1)
            t = min(t, S - (world - r))
            cuts.append(t)
        cuts.append(S)
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def halo_rows(t_begin: int, W: int) -> int:
    """Window keys a range starting at t_begin needs before it."""
    return min(max(W - 1, 0), t_begin)


def range_views(t_begin: int, t_end: int, W: int, Q, Kw, idx, scores, valid, doc_start=None):
    """The slices of whole-sequence [B,S,...] arrays (numpy or torch) that a
    rank owning positions [t_begin, t_end) holds: its own rows of Q, idx,
    scores, valid and doc_start, and Kw from t_begin - halo on. The pool is
    not sliced: every rank holds the whole pool. Returns a dict with kw_lead."""
    h = halo_rows(t_begin, W)
    return {
        "Q": Q[:, t_begin:t_end],
        "Kw": Kw[:, t_begin - h:t_end],
        "idx": None if idx is None else idx[:, t_begin:t_end],
        "scores": scores[:, t_begin:t_end],
        "valid": valid[:, t_begin:t_end],
        "doc_start": None if doc_start is None else doc_start[:, t_begin:t_end],
        "kw_lead": h,
        "t_begin": t_begin,
    }


def sharded_distill_loss(calls, view, pool, *, S_seq: int, W: int, cr: int, scale: float, coeff: float,
                         sink=None, err=None, fused_window: bool = False):
    """One rank's share of the loss over a batch split by token range.

    ``calls`` provides window_lse_range, distill_target_range,
    count_valid_rows and distill_kl (the package itself on GPUs). ``view`` is
    this rank's range_views() dict with contiguous tensors. The sequence:

      window_lse_range -> distill_target_range   (this rank's positions)
      count_valid_rows -> all-reduce(sum)        (N over the whole batch)
      distill_kl(n_rows=N)                       (dscores with the batch-wide 1/N)
      all-reduce(sum) of the loss shares         (the batch loss on every rank)

    With fused_window=True the first two calls are one,
    distill_target_window_range (the window band inside the target kernel,
    Q read once), which also returns the window log-mass.

    Returns (loss [1], dscores, p, window_lse) with dscores, p and window_lse
    for this rank's positions. Every rank must call it (two collectives)."""
    t_begin = view["t_begin"]
    if fused_window:
        p, wl = calls.distill_target_window_range(view["Q"], view["Kw"], pool, view["idx"], W, cr, scale, S_seq,
                                                  t_begin, view["kw_lead"], sink=sink, doc_start=view["doc_start"],
                                                  err=err)
    else:
        wl = calls.window_lse_range(view["Q"], view["Kw"], W, scale, t_begin, view["kw_lead"],
                                    doc_start=view["doc_start"])
        p = calls.distill_target_range(view["Q"], pool, view["idx"], wl, cr, scale, S_seq, t_begin, sink=sink,
                                       doc_start=view["doc_start"], err=err)
    n = calls.count_valid_rows(view["valid"])
    dist = _dist()
    if dist is not None and dist.get_world_size() > 1:
        dist.all_reduce(n, op=dist.ReduceOp.SUM)
    loss, ds = calls.distill_kl(p, view["scores"], view["valid"], coeff, n_rows=n)
    if dist is not None and dist.get_world_size() > 1:
        dist.all_reduce(loss, op=dist.ReduceOp.SUM)
    return loss, ds, p, wl
