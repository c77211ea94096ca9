"""GPU parity of sai_distill_target_kl (the target and the KL stage in one
call, the KL computed in the target kernel's epilogue where K <= 512) against
the fp64 oracle, and against the three-call path on the same inputs.

Covered: the fused route without p (the target never written), the fused route
with p, the per-branch target, document packing, several TMEM groups (K > 512:
the unfused route inside the same call), and the CUDA-core route (tiny).
"""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import TOL_DS, TOL_DS_REL_MAX, TOL_LOSS_REL, TOL_P, assert_close, run_chain, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sai():
    import sparse_attention_indexer_window_b200 as m
    return m


def run_fused(sai, w, with_p, per_branch=False):
    t = to_dev(w)
    B, S, H, K = w.B, w.S, w.H, w.K
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    wl = torch.empty((B, S, H), device="cuda")
    sai.window_lse(t["Q"], t["Kw"], w.W, w.scale, t["doc_start"], out=wl)
    p = torch.full((B, S, K), float("nan"), device="cuda") if with_p else None
    ds = torch.full((B, S, K), float("nan"), device="cuda")
    loss, ds = sai.distill_target_kl(t["Q"], t["pool"], t["idx"], wl, w.cr, w.scale, t["scores"], t["valid"],
                                     w.coeff, sink=t["sink"], doc_start=t["doc_start"], err=err, p=p,
                                     per_branch=per_branch, dscores=ds)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return loss, ds, p


def check_fused(sai, w, with_p=False, per_branch=False):
    loss, ds, p = run_fused(sai, w, with_p, per_branch)
    owl = oracle.window_lse(w.Q, w.Kw, w.doc_start, w.W, w.scale)
    op, bad = oracle.distill_target(w.Q, w.pool, w.idx, owl, w.sink, w.doc_start, w.cr, w.scale,
                                    per_branch=per_branch)
    assert bad == 0
    oloss, ods, _ = oracle.distill_kl(op, w.scores, w.valid, w.coeff)
    lg = float(loss.item())
    assert abs(lg - oloss) <= TOL_LOSS_REL * abs(oloss) + 2.0 ** -149, (lg, oloss)
    dg = ds.cpu().numpy().reshape(-1, w.K)
    assert_close("dscores (fused)", dg, ods, TOL_DS)
    assert np.abs(dg - ods).max() <= TOL_DS_REL_MAX * max(np.abs(ods).max(), 1e-30)
    assert np.all(dg[w.valid.reshape(-1, w.K) == 0] == 0)
    if with_p:
        pg = p.cpu().numpy().reshape(-1, w.K)
        assert_close("p (fused)", pg, op, TOL_P)
        assert np.all(pg[op == 0] == 0)
    return loss, ds


def test_fused_small_without_p(sai):
    check_fused(sai, synth.make("small"))


def test_fused_flash_ragged_with_p(sai):
    check_fused(sai, synth.make("flash", S=1024, K=200), with_p=True)


def test_fused_packed_documents(sai):
    check_fused(sai, synth.make("packed", B=2, S=512, K=96))


def test_fused_per_branch(sai):
    check_fused(sai, synth.make("flash", S=512, K=64), per_branch=True)


def test_fused_pro_heads_two_groups(sai):
    check_fused(sai, synth.make("flash", S=1280, K=300, H=128))


def test_fused_multi_group_falls_back_inside_the_call(sai):
    # K = 576 > 512: the call runs the target kernel and the KL pass separately
    check_fused(sai, synth.make("long", S=2304, K=576), with_p=True)


def test_fused_tiny_cuda_core_route(sai):
    check_fused(sai, synth.make("tiny"), with_p=True)


def test_fused_matches_three_calls_and_is_deterministic(sai):
    w = synth.make("flash", S=1024, K=200, seed=77)
    t = to_dev(w)
    _, _, loss3, ds3 = run_chain(sai, w, t)
    l1, d1, _ = run_fused(sai, w, with_p=False)
    l2, d2, _ = run_fused(sai, w, with_p=False)
    assert float(l1.item()) == float(l2.item())
    assert torch.equal(d1, d2)
    assert abs(float(l1.item()) - float(loss3.item())) <= 1e-5 * abs(float(loss3.item()))
    assert float((d1 - ds3).abs().max()) <= 1e-7
