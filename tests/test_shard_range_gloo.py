"""Splitting sequences across ranks by token range, on two CPU ranks (gloo).

Each rank holds only its positions' rows, the W-1 window keys before its first
position and the whole pool (shard.range_views), and runs the call sequence of
shard.sharded_distill_loss: the range calls on its positions, a device count
of its valid rows, one all-reduce of that count (the batch-wide N), the KL
with that N, and an all-reduce of the loss shares. The range calls need a GPU,
so here they are answered by the fp64 oracle, which only ever sees what the
rank was handed: the rank's rows are placed at their positions in otherwise
empty whole-sequence arrays. A halo that is too short, a position offset that
is wrong, or an N that is not the batch's then shows up as a mismatch against
the oracle run on the whole batch.
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


class OracleRangeCalls:
    """The four range calls of shard.sharded_distill_loss, answered by the
    oracle from the rank's own arrays only."""

    def __init__(self, S_seq):
        self.S_seq = S_seq

    def _tokens(self, B, t_begin, S):
        return np.concatenate([b * self.S_seq + np.arange(t_begin, t_begin + S) for b in range(B)]).astype(np.int64)

    def window_lse_range(self, Q, Kw, W, scale, t_begin, kw_lead, doc_start=None):
        import oracle
        B, S, H, D = Q.shape
        Qf = np.zeros((B, self.S_seq, H, D), np.uint16)
        Qf[:, t_begin:t_begin + S] = Q
        Kf = np.zeros((B, self.S_seq, D), np.uint16)
        Kf[:, t_begin - kw_lead:t_begin + S] = Kw
        dsf = None
        if doc_start is not None:
            dsf = np.zeros((B, self.S_seq), np.int32)
            dsf[:, t_begin:t_begin + S] = doc_start
        wl = oracle.window_lse(Qf, Kf, dsf, W, scale, self._tokens(B, t_begin, S))
        return wl.reshape(B, S, H)

    def distill_target_range(self, Q, pool, idx, wl, cr, scale, S_seq, t_begin, sink=None, doc_start=None,
                             err=None):
        import oracle
        assert S_seq == self.S_seq
        B, S, H, D = Q.shape
        K = idx.shape[-1]
        Qf = np.zeros((B, S_seq, H, D), np.uint16)
        Qf[:, t_begin:t_begin + S] = Q
        idf = np.full((B, S_seq, K), -1, np.int32)
        idf[:, t_begin:t_begin + S] = idx
        dsf = None
        if doc_start is not None:
            dsf = np.zeros((B, S_seq), np.int32)
            dsf[:, t_begin:t_begin + S] = doc_start
        p, bad = oracle.distill_target(Qf, pool, idf, wl.reshape(-1, H), sink, dsf, cr, scale,
                                       self._tokens(B, t_begin, S))
        assert bad == 0
        return p.reshape(B, S, K)

    def distill_target_window_range(self, Q, Kw, pool, idx, W, cr, scale, S_seq, t_begin, kw_lead, sink=None,
                                    doc_start=None, err=None):
        # the fused call's contract: (p, window log-mass) from the same inputs
        wl = self.window_lse_range(Q, Kw, W, scale, t_begin, kw_lead, doc_start=doc_start)
        p = self.distill_target_range(Q, pool, idx, wl, cr, scale, S_seq, t_begin, sink=sink, doc_start=doc_start,
                                      err=err)
        return p, wl

    def count_valid_rows(self, valid):
        import oracle
        return torch.tensor([oracle.count_valid_rows(valid)], dtype=torch.int64)

    def distill_kl(self, p, scores, valid, coeff, n_rows=None):
        import oracle
        K = scores.shape[-1]
        loss, ds, _ = oracle.distill_kl(p.reshape(-1, K), scores.reshape(-1, K), valid.reshape(-1, K), coeff,
                                        n_norm=int(n_rows.item()))
        return torch.tensor([loss], dtype=torch.float64), ds.reshape(p.shape)


def _workload(name):
    import synth
    if name == "flash":
        return synth.make("flash", S=512, K=64, H=16, D=64, seed=31)
    return synth.make("packed", B=2, S=512, K=64, H=16, D=64, seed=32)


def _rank_main(rank, world, port, out_dir, name, balanced, fused=False):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w = _workload(name)
        cost = shard.token_cost(w.S, w.cr, w.K, w.W) if balanced else None
        t0, t1 = shard.token_ranges(w.S, world, cost)[rank]
        v = shard.range_views(t0, t1, w.W, w.Q, w.Kw, w.idx, w.scores, w.valid, w.doc_start)
        loss, ds, p, wl = shard.sharded_distill_loss(OracleRangeCalls(w.S), v, w.pool, S_seq=w.S, W=w.W, cr=w.cr,
                                                     scale=w.scale, coeff=w.coeff, sink=w.sink,
                                                     fused_window=fused)
        np.savez(os.path.join(out_dir, f"{name}_rank{rank}.npz"), loss=float(loss.item()), ds=ds, p=p, wl=wl,
                 t0=t0, t1=t1, kw_lead=v["kw_lead"], kw_rows=v["Kw"].shape[1])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,balanced,fused", [("flash", True, False), ("packed", False, False),
                                                ("packed", True, True)])
def test_two_rank_token_range_split(tmp_path, name, balanced, fused):
    """fused: the rank's window and target come from the one window-fused
    range call (shard.sharded_distill_loss(fused_window=True))."""
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), name, balanced, fused), nprocs=world,
                       join=True, start_method="spawn")
    import oracle
    w = _workload(name)
    owl, op, oloss, ods, bad = oracle.run_all(w)
    assert bad == 0
    owl = owl.reshape(w.B, w.S, w.H)
    op = op.reshape(w.B, w.S, w.K)
    ods = ods.reshape(w.B, w.S, w.K)
    rs = [np.load(tmp_path / f"{name}_rank{r}.npz") for r in range(world)]
    assert int(rs[0]["t0"]) == 0 and int(rs[-1]["t1"]) == w.S
    for r in rs:
        t0, t1 = int(r["t0"]), int(r["t1"])
        # the rank was handed its rows plus exactly the halo it needs
        assert int(r["kw_lead"]) == min(w.W - 1, t0)
        assert int(r["kw_rows"]) == t1 - t0 + int(r["kw_lead"])
        # every rank ends with the whole batch's loss
        assert float(r["loss"]) == pytest.approx(oloss, rel=1e-12)
        np.testing.assert_allclose(r["wl"], owl[:, t0:t1], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(r["p"], op[:, t0:t1], rtol=1e-12, atol=1e-300)
        # dscores carry the batch-wide 1/N
        np.testing.assert_allclose(r["ds"], ods[:, t0:t1], rtol=1e-12, atol=1e-300)
    assert int(rs[0]["t1"]) == int(rs[1]["t0"])


def test_token_ranges_cover_and_balance():
    for S in (1, 2, 7, 512, 4096):
        for world in range(1, 5):
            if world > S:
                continue
            for cost in (None, shard.token_cost(S, 4, min(512, max(1, S // 4)), 128)):
                rg = shard.token_ranges(S, world, cost)
                assert rg[0][0] == 0 and rg[-1][1] == S
                for (a, b), (c, d) in zip(rg, rg[1:]):
                    assert b == c
                assert all(b > a for a, b in rg)
    # the flash shape: later positions select more blocks, so the balanced
    # cut lies past the middle and splits the work within 1 %
    S, cr, K, W = 4096, 4, 512, 128
    c = shard.token_cost(S, cr, K, W)
    (a0, a1), (b0, b1) = shard.token_ranges(S, 2, c)
    assert a1 > S // 2
    assert abs(c[a0:a1].sum() - c[b0:b1].sum()) <= 0.01 * c.sum()
    assert shard.halo_rows(0, 128) == 0 and shard.halo_rows(5, 128) == 5 and shard.halo_rows(3000, 128) == 127
    with pytest.raises(ValueError):
        shard.token_ranges(0, 2)
