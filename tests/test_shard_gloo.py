"""The data-parallel host plumbing on two CPU ranks (gloo).

Two ranks each own one sequence of the two-sequence small workload, run the
oracle on their share (the path itself needs a GPU; what is under test here is
the host logic around it), and combine: the batch-wide loss from per-rank
losses must equal the loss of the whole batch, each rank's rescaled dscores
must equal the whole batch's rows, and the max-over-ranks timing must pick the
slowest rank.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

from sparse_attention_indexer_window_b200 import shard  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import oracle
        import synth
        w = synth.make("small")
        K = w.K
        b0, b1 = shard.split_sequences(w.B, rank, world)
        tokens = np.arange(b0 * w.S, b1 * w.S, dtype=np.int64)
        wl = oracle.window_lse(w.Q, w.Kw, w.doc_start, w.W, w.scale, tokens)
        p, bad = oracle.distill_target(w.Q, w.pool, w.idx, wl, w.sink, w.doc_start, w.cr, w.scale, tokens)
        assert bad == 0
        sc = w.scores.reshape(-1, K)[tokens]
        va = w.valid.reshape(-1, K)[tokens]
        loss_r, ds_r, _ = oracle.distill_kl(p, sc, va, w.coeff)
        n_r = oracle.count_valid_rows(va)
        g_loss, factor = shard.global_mean_loss(loss_r, n_r)
        slowest = shard.max_over_ranks(10.0 + rank)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), g_loss=g_loss, factor=factor,
                 ds=ds_r * factor, tokens=tokens, slowest=slowest, loss_r=loss_r, n_r=n_r)
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_combine(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    import oracle
    import synth
    w = synth.make("small")
    _, _, loss_all, ds_all, bad = oracle.run_all(w)
    assert bad == 0
    ds_all = ds_all.reshape(-1, w.K)
    rs = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    for r in rs:
        # every rank holds the same batch-wide loss, equal to the whole batch's
        assert float(r["g_loss"]) == pytest.approx(loss_all, rel=1e-12, abs=1e-300)
        np.testing.assert_allclose(r["ds"], ds_all[r["tokens"]], rtol=1e-12, atol=1e-300)
        assert float(r["slowest"]) == 10.0 + world - 1
    # the shares cover the batch exactly once
    toks = np.concatenate([r["tokens"] for r in rs])
    assert np.array_equal(np.sort(toks), np.arange(w.B * w.S))
    # per-rank losses differ (distinct sequences), so the combine is not trivial
    assert float(rs[0]["loss_r"]) != float(rs[1]["loss_r"])


def test_split_sequences_covers_every_row_once():
    for B in range(0, 9):
        for world in range(1, 6):
            got = []
            for r in range(world):
                s, e = shard.split_sequences(B, r, world)
                assert 0 <= s <= e <= B
                got.extend(range(s, e))
            assert got == list(range(B))
    with pytest.raises(ValueError):
        shard.split_sequences(4, 2, 2)


def test_single_process_defaults():
    # without a process group the helpers reduce over one rank
    assert shard.max_over_ranks(3.5) == 3.5
    loss, factor = shard.global_mean_loss(0.25, 7)
    assert loss == pytest.approx(0.25) and factor == 1.0
    # a rank with no valid rows contributes nothing and keeps its gradient at zero scale
    loss0, f0 = shard.global_mean_loss(0.0, 0)
    assert loss0 == 0.0 and f0 == 1.0
    assert shard.rank_seed(1003, 0) == 1003 and shard.rank_seed(1003, 3) == 1006
