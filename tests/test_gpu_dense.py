"""GPU parity of the dense warm-up stage (sai_distill_target with idx NULL)
against the fp64 oracle in the same mode.

In the dense stage (MaxText page "Add Indexer Loss [Deepseek v4]": dense
warm-up before sparse training) every compressed block is a slot: slot k is
block k, and the causal and document rules mask the blocks a token cannot see.
Covered: the CUDA-core kernel (tiny), few heads (small), V4-Flash widths with
several TMEM groups per late token, document packing, the per-branch target in
dense mode, and the KL stage on the dense target.
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


def dense_valid(w):
    """The dense stage's valid mask: block k visible to token t."""
    P = w.S // w.cr
    t = np.arange(w.S)[:, None]
    k = np.arange(P)[None, :]
    v = np.broadcast_to(((k + 1) * w.cr - 1 <= t), (w.B, w.S, P)).copy()
    if w.doc_start is not None:
        d0 = np.clip(w.doc_start, 0, np.arange(w.S)[None, :])
        v &= (k[None] * w.cr >= d0[:, :, None])
    return v.astype(np.uint8)


def check_dense(sai, w, per_branch=False, kl=False):
    t = to_dev(w)
    B, S, H, P = w.B, w.S, w.H, w.S // w.cr
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    wl = torch.empty((B, S, H), device="cuda")
    sai.window_lse(t["Q"], t["Kw"], w.W, w.scale, t["doc_start"], out=wl)
    p = torch.full((B, S, P), float("nan"), device="cuda")
    sai.distill_target(t["Q"], t["pool"], None, wl, w.cr, w.scale, sink=t["sink"], doc_start=t["doc_start"],
                       err=err, out=p, per_branch=per_branch)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    owl = oracle.window_lse(w.Q, w.Kw, w.doc_start, w.W, w.scale)
    op, bad = oracle.distill_target(w.Q, w.pool, None, owl, w.sink, w.doc_start, w.cr, w.scale,
                                    per_branch=per_branch)
    assert bad == 0
    pg = p.cpu().numpy().reshape(-1, P)
    assert_close("p (dense)", pg, op, TOL_P)
    assert np.all(pg[op == 0] == 0)
    valid = dense_valid(w)
    assert np.all(pg[valid.reshape(-1, P) == 0] == 0)
    if kl:
        rng = np.random.default_rng(5)
        scores = (rng.standard_normal((B, S, P)) * np.sqrt(2.0)).astype(np.float32)
        loss, ds = sai.distill_kl(p, torch.from_numpy(scores).cuda(), torch.from_numpy(valid).cuda(), w.coeff)
        torch.cuda.synchronize()
        oloss, ods, _ = oracle.distill_kl(op, scores, valid, w.coeff)
        assert abs(float(loss.item()) - oloss) <= TOL_LOSS_REL * abs(oloss) + 2.0 ** -149
        assert_close("dscores (dense)", ds.cpu().numpy().reshape(-1, P), ods, TOL_DS)


def test_dense_tiny(sai):
    check_dense(sai, synth.make("tiny"))


def test_dense_small(sai):
    check_dense(sai, synth.make("small"), kl=True)


def test_dense_flash_widths(sai):
    # P = 256 slots per token at H=64: ragged tiles, contiguous-row tiles
    check_dense(sai, synth.make("flash", S=1024, K=200), kl=True)


def test_dense_multi_group(sai):
    # P = 576: tokens past t = 2047 have more than 512 visible blocks, i.e.
    # more scores than one TMEM group holds at H=64
    check_dense(sai, synth.make("flash", S=2304, K=200))


def test_dense_packed_documents(sai):
    check_dense(sai, synth.make("packed", B=2, S=512, K=96))


def test_dense_per_branch(sai):
    check_dense(sai, synth.make("flash", S=512, K=64), per_branch=True)
