"""GPU parity of the per-branch target mode (sai_distill_target_ex with
SAI_TARGET_PER_BRANCH) against the fp64 oracle's per-branch mode.

The per-branch target is the earlier form that the Primus page keeps as an A/B
switch and the MaxText page prints: each head is normalised over the selected
compressed entries alone, the floor is 1e-10, and the window log-mass and the
sink play no part (the call is made without them). Covered: the CUDA-core
kernel (tiny), the tensor-core kernel with few heads (small), V4-Flash widths
with ragged tiles and contiguous-row tiles, document packing, and tokens with
more selected slots than one TMEM group holds.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import TOL_P, assert_close, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sai():
    import sparse_attention_indexer_window_b200 as m
    return m


def check_per_branch(sai, w):
    t = to_dev(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = torch.full((w.B, w.S, w.K), float("nan"), device="cuda")
    sai.distill_target(t["Q"], t["pool"], t["idx"], None, w.cr, w.scale, doc_start=t["doc_start"], err=err,
                       out=p, per_branch=True)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    op, bad = oracle.distill_target(w.Q, w.pool, w.idx, None, None, w.doc_start, w.cr, w.scale, per_branch=True)
    assert bad == 0
    pg = p.cpu().numpy().reshape(-1, w.K)
    assert_close("p (per-branch)", pg, op, TOL_P)
    assert np.all(pg[op == 0] == 0)
    # every row with a selected slot sums to 1 (H full distributions, averaged)
    rows = pg.sum(axis=1)
    nonempty = op.sum(axis=1) > 0
    np.testing.assert_allclose(rows[nonempty], 1.0, atol=1e-5)
    return p


def test_per_branch_tiny(sai):
    check_per_branch(sai, synth.make("tiny"))


def test_per_branch_small(sai):
    check_per_branch(sai, synth.make("small"))


def test_per_branch_flash_ragged(sai):
    check_per_branch(sai, synth.make("flash", S=1024, K=200))


def test_per_branch_packed_documents(sai):
    check_per_branch(sai, synth.make("packed", B=2, S=512, K=96))


def test_per_branch_multi_group(sai):
    check_per_branch(sai, synth.make("long", S=2304, K=576))


def test_per_branch_differs_from_joint(sai):
    """Same inputs, the two modes give different targets (the flag is live)."""
    from tests.gpu_util import run_chain
    w = synth.make("small")
    t = to_dev(w)
    _, pj, _, _ = run_chain(sai, w, t)
    pb = check_per_branch(sai, w)
    assert float((pj - pb).abs().max()) > 1e-3
