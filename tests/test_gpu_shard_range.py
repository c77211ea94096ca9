"""GPU: the token-range calls against the fp64 oracle on the whole batch.

One GPU plays the ranks of a split by token range one after another: each
range gets only its own rows, its W-1 halo keys and the whole pool
(shard.range_views), and runs sai_window_lse_range, sai_distill_target_range
and sai_count_valid_rows; the ranges' counts are added on the device (the sum
an all-reduce forms across GPUs) and every range's sai_distill_kl_ex reads it.
The ranges' p, window_lse and dscores must equal the whole batch's rows and
their loss shares must add up to its loss, within the usual tolerances.
"""
import numpy as np
import pytest

import oracle
import synth
from sparse_attention_indexer_window_b200 import shard
from tests.gpu_util import TOL_DS, TOL_LOSS_REL, TOL_P, assert_close, tol_wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sai():
    import sparse_attention_indexer_window_b200 as m
    return m


def _dev(a, bf16=False):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if bf16:
        t = t.view(torch.int16)
    return t.cuda().contiguous()


def _run_ranges(sai, w, ranges, fused=False):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pool = _dev(w.pool, True)
    sink = None if w.sink is None else _dev(w.sink)
    parts, counts = [], []
    for t0, t1 in ranges:
        v = shard.range_views(t0, t1, w.W, w.Q, w.Kw, w.idx, w.scores, w.valid, w.doc_start)
        Q, Kw = _dev(v["Q"], True), _dev(v["Kw"], True)
        idx, sc, va = _dev(v["idx"]), _dev(v["scores"]), _dev(v["valid"])
        ds0 = None if v["doc_start"] is None else _dev(v["doc_start"])
        if fused:
            # the window band inside the target kernel: one call per range
            wl = torch.full((w.B, t1 - t0, w.H), float("nan"), device="cuda")
            p = sai.distill_target_window_range(Q, Kw, pool, idx, w.W, w.cr, w.scale, w.S, t0, v["kw_lead"],
                                                sink=sink, doc_start=ds0, err=err, wl_out=wl)
        else:
            wl = sai.window_lse_range(Q, Kw, w.W, w.scale, t0, v["kw_lead"], doc_start=ds0)
            p = sai.distill_target_range(Q, pool, idx, wl, w.cr, w.scale, w.S, t0, sink=sink, doc_start=ds0,
                                         err=err)
        counts.append(sai.count_valid_rows(va))
        parts.append((t0, t1, wl, p, sc, va))
    n_all = torch.stack(counts).sum(0).to(torch.int32)   # what the all-reduce gives every rank
    out = []
    for t0, t1, wl, p, sc, va in parts:
        loss, ds = sai.distill_kl(p, sc, va, w.coeff, n_rows=n_all)
        out.append((t0, t1, wl, p, loss, ds))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert int(n_all.item()) == oracle.count_valid_rows(w.valid)
    return out


def _check(sai, w, ranges, fused=False):
    owl, op, oloss, ods, bad = oracle.run_all(w)
    assert bad == 0
    owl = owl.reshape(w.B, w.S, w.H)
    op = op.reshape(w.B, w.S, w.K)
    ods = ods.reshape(w.B, w.S, w.K)
    loss = 0.0
    for t0, t1, wl, p, l, ds in _run_ranges(sai, w, ranges, fused):
        ref = owl[:, t0:t1]
        assert_close("window_lse", wl.cpu().numpy() - ref, 0 * ref, tol_wl(ref))
        pg = p.cpu().numpy()
        assert_close("p", pg, op[:, t0:t1], TOL_P)
        assert np.all(pg[op[:, t0:t1] == 0] == 0)
        dg = ds.cpu().numpy()
        assert_close("dscores", dg, ods[:, t0:t1], TOL_DS)
        assert np.all(dg[w.valid[:, t0:t1] == 0] == 0)
        loss += float(l.item())
    assert abs(loss - oloss) <= TOL_LOSS_REL * abs(oloss)


@pytest.mark.parametrize("fused", [False, True])
def test_flash_recipe_two_ranges_balanced(sai, fused):
    """H=64, D=512 tensor-core kernels; the cut balances the work. fused: the
    window-fused range call."""
    w = synth.make("flash", S=1024, K=200, seed=41)
    rg = shard.token_ranges(w.S, 2, shard.token_cost(w.S, w.cr, w.K, w.W))
    rg = [(a, b) for a, b in rg]
    # an even cut keeps both ranges on the tensor-core window tiles (2 tokens)
    if rg[0][1] % 2:
        rg = [(0, rg[0][1] + 1), (rg[0][1] + 1, w.S)]
    _check(sai, w, rg, fused)


@pytest.mark.parametrize("fused", [False, True])
def test_flash_recipe_four_ranges_odd_cuts(sai, fused):
    """Cuts at odd positions and inside a window; an odd-length range runs the
    CUDA-core window kernel (fused: the window tile of each range's first
    tokens reaches into its halo)."""
    w = synth.make("flash", S=768, K=128, seed=42)
    _check(sai, w, [(0, 100), (100, 301), (301, 556), (556, 768)], fused)


@pytest.mark.parametrize("fused", [False, True])
def test_packed_two_documents_ranges(sai, fused):
    """Two sequences with a document split each: positions, not row numbers,
    decide the causal and document rules."""
    w = synth.make("packed", B=2, S=512, K=96, seed=43)
    _check(sai, w, [(0, 200), (200, 512)], fused)


def test_tiny_generic_ranges(sai):
    w = synth.make("tiny")
    _check(sai, w, [(0, 17), (17, 40), (40, 64)])


def test_short_halo_is_rejected(sai):
    w = synth.make("tiny")
    Q = _dev(w.Q[:, 20:40], True)
    Kw = _dev(w.Kw[:, 10:40], True)           # 10 keys before position 20, W - 1 = 15 needed
    with pytest.raises(sai.SaiError):
        sai.window_lse_range(Q, Kw, w.W, w.scale, 20, 10)
