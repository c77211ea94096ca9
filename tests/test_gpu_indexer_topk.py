"""GPU parity of sai_indexer_topk (top-K block selection from indexer scores)
against the oracle: indices, selected scores and valid flags must be equal
bit for bit.

The selection rule follows the MaxText page "Add Indexer Loss [Deepseek v4]"
(top-k block indices, -1 where the choice is invalid, the scores returned
with them; causal block and packing masks). Covered: tie-heavy rows with
NaN, +-inf and -0 entries, documents, K = 1 and K = P, cr = 1, the flash
and long shapes at full size, and the selection feeding the loss calls.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import TOL_DS, TOL_LOSS_REL, TOL_P, assert_close, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sai():
    import sparse_attention_indexer_window_b200 as m
    return m


def doc_starts(rng, B, S):
    ds = np.zeros((B, S), dtype=np.int32)
    for b in range(B):
        s0 = int(rng.integers(1, S))
        ds[b, s0:] = s0
    return ds


def tricky_scores(rng, B, S, P, step):
    sc = rng.standard_normal((B, S, P)).astype(np.float32)
    if step:
        sc = (np.round(sc / step) * step).astype(np.float32)
    sc[rng.random(sc.shape) < 0.03] = -np.inf
    sc[rng.random(sc.shape) < 0.01] = np.nan
    sc[rng.random(sc.shape) < 0.01] = -0.0
    sc[rng.random(sc.shape) < 0.005] = np.inf
    return sc


def check_topk(sai, sc, ds, cr, K):
    B, S, P = sc.shape
    dsd = None if ds is None else torch.from_numpy(ds).cuda()
    idx = torch.full((B, S, K), -7, dtype=torch.int32, device="cuda")
    sel = torch.full((B, S, K), float("nan"), device="cuda")
    val = torch.full((B, S, K), 7, dtype=torch.uint8, device="cuda")
    sai.indexer_topk(torch.from_numpy(sc).cuda(), cr, K, doc_start=dsd, idx=idx, sel_scores=sel, valid=val)
    torch.cuda.synchronize()
    oi, osel, ov = oracle.indexer_topk(sc, ds, cr, K)
    gi = idx.cpu().numpy().reshape(-1, K)
    assert np.array_equal(gi, oi), f"{int((gi != oi).any(axis=1).sum())} rows differ"
    assert np.array_equal(val.cpu().numpy().reshape(-1, K), ov)
    assert np.array_equal(sel.cpu().numpy().reshape(-1, K).view(np.uint32), osel.view(np.uint32))
    return idx, sel, val


@pytest.mark.parametrize("seed,B,S,cr,K,step,docs", [
    (70, 2, 64, 4, 5, 0.5, True),
    (71, 1, 256, 4, 40, 0.0, False),
    (72, 2, 512, 4, 100, 0.125, True),
    (73, 2, 128, 2, 30, 1.0, True),
    (74, 1, 64, 1, 64, 0.25, False),      # K = P: every candidate
    (75, 1, 128, 4, 1, 0.5, True),        # K = 1
])
def test_topk_tricky_rows(sai, seed, B, S, cr, K, step, docs):
    rng = np.random.default_rng(seed)
    P = S // cr
    sc = tricky_scores(rng, B, S, P, step)
    check_topk(sai, sc, doc_starts(rng, B, S) if docs else None, cr, K)


def test_topk_flash_full_size(sai):
    # the flash shape: S = 4096, cr = 4 (P = 1024 blocks), K = 512
    sc = synth.index_scores(1, 4096, 4, seed=1003)
    check_topk(sai, sc, None, 4, 512)


def test_topk_packed_flash(sai):
    rng = np.random.default_rng(76)
    sc = synth.index_scores(2, 4096, 4, seed=1004)
    check_topk(sai, sc, doc_starts(rng, 2, 4096), 4, 512)


def test_topk_long_full_size(sai):
    # the long shape: S = 16384 (P = 4096 blocks), K = 2048
    sc = synth.index_scores(1, 16384, 4, seed=1005)
    check_topk(sai, sc, None, 4, 2048)


def test_topk_feeds_the_loss(sai):
    """The selection's outputs are the loss calls' inputs: idx for the
    target, the selected scores and valid flags for the KL. The chain on the
    device matches the oracle chain on the same inputs."""
    w = synth.make("flash", S=1024, K=200)
    sc = synth.index_scores(w.B, w.S, w.cr, seed=77)
    t = to_dev(w)
    idx, sel, val = sai.indexer_topk(torch.from_numpy(sc).cuda(), w.cr, w.K)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    wl = sai.window_lse(t["Q"], t["Kw"], w.W, w.scale)
    p = sai.distill_target(t["Q"], t["pool"], idx, wl, w.cr, w.scale, sink=t["sink"], err=err)
    loss, ds = sai.distill_kl(p, sel, val, w.coeff)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    oi, osel, ov = oracle.indexer_topk(sc, None, w.cr, w.K)
    owl = oracle.window_lse(w.Q, w.Kw, None, w.W, w.scale)
    op, bad = oracle.distill_target(w.Q, w.pool, oi.reshape(w.B, w.S, w.K), owl, w.sink, None, w.cr, w.scale)
    assert bad == 0
    oloss, ods, _ = oracle.distill_kl(op, osel, ov, w.coeff)
    assert_close("p (selected by the kernel)", p.cpu().numpy().reshape(-1, w.K), op, TOL_P)
    assert abs(float(loss.item()) - oloss) <= TOL_LOSS_REL * abs(oloss)
    assert_close("dscores (selected by the kernel)", ds.cpu().numpy().reshape(-1, w.K), ods, TOL_DS)
