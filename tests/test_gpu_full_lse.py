"""GPU parity of the given-LSE target (sai_distill_target_ex with
SAI_TARGET_FULL_LSE) against the fp64 oracle in the same mode.

When the CSA attention forward has returned its per-head LSE (Primus page
"Docker Build for DeepSeek-v4", gluon_v3 "Optimization Notes"), that LSE is
already lse_full: the normaliser over the window keys, the selected compressed
entries and the sink (Primus page "perf(deepseek-v4): fuse and enable the
indexer distillation loss", first commit message). The target then needs no
window pass. The LSE handed in here is the joint one computed term by term
in numpy (fp64, rounded to fp32 for both sides), optionally offset per head so
that the call sees inputs no window pass would produce.

Covered: the CUDA-core kernel (tiny), few heads (small), V4-Flash widths with
ragged tiles, document packing, tokens with more selected slots than one TMEM
group holds, the FLT_MIN floor, agreement with the joint three-call chain, and
the fused target + KL call in this mode.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import TOL_DS, TOL_LOSS_REL, TOL_P, assert_close, run_chain, to_dev
from tests.longway import joint_lse_long_way

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sai():
    import sparse_attention_indexer_window_b200 as m
    return m


def full_lse_input(w, offset_seed=None, shift=0.0):
    """[B,S,H] fp32: the joint LSE of every (token, head), plus a seeded
    per-(token, head) offset when offset_seed is set, plus `shift`."""
    lf = joint_lse_long_way(w.Q, w.Kw, w.pool, w.idx, w.sink, w.doc_start, w.W, w.cr, w.scale)
    if offset_seed is not None:
        lf = lf + np.random.default_rng(offset_seed).standard_normal(lf.shape)
    return (lf + shift).astype(np.float32).reshape(w.B, w.S, w.H)


def check_full_lse(sai, w, lf):
    t = to_dev(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = torch.full((w.B, w.S, w.K), float("nan"), device="cuda")
    # a sink passed alongside is not read in this mode
    sai.distill_target(t["Q"], t["pool"], t["idx"], torch.from_numpy(lf).cuda(), w.cr, w.scale, sink=t["sink"],
                       doc_start=t["doc_start"], err=err, out=p, full_lse=True)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    op, bad = oracle.distill_target(w.Q, w.pool, w.idx, lf.reshape(-1, w.H).astype(np.float64), None,
                                    w.doc_start, w.cr, w.scale, full_lse=True)
    assert bad == 0
    pg = p.cpu().numpy().reshape(-1, w.K)
    assert_close("p (given LSE)", pg, op, TOL_P)
    assert np.all(pg[op == 0] == 0)
    return p, op


def test_full_lse_tiny(sai):
    w = synth.make("tiny")
    check_full_lse(sai, w, full_lse_input(w, offset_seed=1))


def test_full_lse_small(sai):
    w = synth.make("small")
    check_full_lse(sai, w, full_lse_input(w, offset_seed=2))


def test_full_lse_flash_ragged_matches_joint_chain(sai):
    """With the exact joint LSE the given-LSE target is the joint target: it
    agrees with the window_lse -> distill_target chain on the same inputs."""
    w = synth.make("flash", S=1024, K=200)
    p, _ = check_full_lse(sai, w, full_lse_input(w))
    _, pj, _, _ = run_chain(sai, w, to_dev(w))
    assert_close("p (given LSE vs joint chain)", p.cpu().numpy(), pj.cpu().numpy(), 2 * TOL_P)


def test_full_lse_packed_documents(sai):
    w = synth.make("packed", B=2, S=512, K=96)
    check_full_lse(sai, w, full_lse_input(w, offset_seed=4))


def test_full_lse_multi_group(sai):
    w = synth.make("long", S=2304, K=576)
    check_full_lse(sai, w, full_lse_input(w, offset_seed=5))


def test_full_lse_floor(sai):
    """A normaliser far above every logit leaves the row mass below FLT_MIN:
    both sides divide by the floor, so p no longer sums to 1."""
    w = synth.make("small")
    _, op = check_full_lse(sai, w, full_lse_input(w, shift=95.0))
    sums = op.sum(axis=1)
    assert np.all(sums[sums > 0] < 0.5)


def test_full_lse_fused_kl(sai):
    w = synth.make("flash", S=1024, K=200)
    lf = full_lse_input(w, offset_seed=7)
    t = to_dev(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    loss, ds = sai.distill_target_kl(t["Q"], t["pool"], t["idx"], torch.from_numpy(lf).cuda(), w.cr, w.scale,
                                     t["scores"], t["valid"], w.coeff, doc_start=t["doc_start"], err=err,
                                     full_lse=True)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    op, _ = oracle.distill_target(w.Q, w.pool, w.idx, lf.reshape(-1, w.H).astype(np.float64), None,
                                  w.doc_start, w.cr, w.scale, full_lse=True)
    oloss, ods, _ = oracle.distill_kl(op, w.scores, w.valid, w.coeff)
    assert abs(float(loss.item()) - oloss) <= TOL_LOSS_REL * abs(oloss) + 2.0 ** -149
    assert_close("dscores (given LSE, fused)", ds.cpu().numpy().reshape(-1, w.K), ods, TOL_DS)
