"""GPU parity of sai_distill_target_window (the window band and the target in
one kernel, Q read once) against the fp64 oracle.

The fused kernel forms each head's window log-mass from Kw itself; the test
reads it back (window_lse out) and checks it against the oracle's window_lse,
and checks p against the oracle's target, element by element, on the same
shapes and edge cases as the three-call path: ragged tiles, several TMEM
groups (with and without the raw-score spill), H in {16, 32, 64, 128},
document packing, no sink, the extreme-sink floor, scattered and bad
indices, and the cases this kernel adds: tokens whose 128-row window box
starts before row 0 (read as zeros), boxes shorter than 128 rows (fewer Kw
rows than that), rows of the previous sequence in a packed batch (masked)
and groups of one pipeline stage (the TMEM tile ring turning over fastest).
Tolerances as for the three-call path (tests/gpu_util.py).
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import (TOL_DS, TOL_LOSS_REL, TOL_P, assert_close, to_dev, tol_wl)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sai():
    import sparse_attention_indexer_window_b200 as m
    return m


def run_fused(sai, w, t, err=None, workspace=None, dense=False):
    """p and the window log-mass from the fused call; outputs pre-filled with
    NaN so a slot or head the kernel forgets to write shows up."""
    B, S, H = w.B, w.S, w.H
    K = S // w.cr if dense else w.K
    wl = torch.full((B, S, H), float("nan"), device="cuda")
    p = torch.full((B, S, K), float("nan"), device="cuda")
    sai.distill_target_window(t["Q"], t["Kw"], t["pool"], None if dense else t["idx"], w.W, w.cr, w.scale,
                              sink=t["sink"], doc_start=t["doc_start"], err=err, out=p, wl_out=wl,
                              workspace=workspace)
    torch.cuda.synchronize()
    return wl, p


def check_fused(sai, w, *, tokens=None, err_expect=0, with_loss=True):
    t = to_dev(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    wl, p = run_fused(sai, w, t, err)
    owl, op, oloss, ods, bad = oracle.run_all(w, tokens)
    assert (bad > 0) == (err_expect != 0)
    assert int(err.item()) == err_expect
    wg = wl.cpu().numpy().reshape(-1, w.H)
    pg = p.cpu().numpy().reshape(-1, w.K)
    if tokens is not None:
        wg, pg = wg[tokens], pg[tokens]
    assert_close("window_lse", wg - owl, 0 * owl, tol_wl(owl))
    assert_close("p", pg, op, TOL_P)
    assert np.all(pg[op == 0] == 0)
    if tokens is None and with_loss:
        # the KL stage on the fused target: the whole chain in two calls
        loss, ds = sai.distill_kl(p, t["scores"], t["valid"], w.coeff)
        lg = float(loss.item())
        assert abs(lg - oloss) <= TOL_LOSS_REL * abs(oloss) + 2.0 ** -149, (lg, oloss)
        assert_close("dscores", ds.cpu().numpy().reshape(-1, w.K), ods, TOL_DS)
    return wl, p


def test_small_h16(sai):
    """H=16, D=128, W=64: eight score tiles per TMEM group, 32 tile slots."""
    check_fused(sai, synth.make("small"))


def test_flash_recipe_ragged_tiles(sai):
    """H=64, D=512, K=200 (a ragged last tile); the first 127 tokens' window
    boxes start before row 0."""
    check_fused(sai, synth.make("flash", S=1024, K=200))


def test_pro_heads_h128_two_groups(sai):
    """H=128: two score tiles per group and four tile slots; 300 selected
    slots take two groups (spill workspace allocated by the binding)."""
    check_fused(sai, synth.make("flash", S=1280, K=300, H=128))


def test_h32_d256(sai):
    check_fused(sai, synth.make("flash", S=512, K=96, H=32, D=256))


def test_h64_d128_one_stage_groups(sai):
    """D=128: one pipeline stage per tile, so the window group and every
    short token's score group are single stages and the tile ring and its
    commit barriers turn over as fast as they can."""
    check_fused(sai, synth.make("flash", S=512, K=100, D=128))


def test_h64_d64_one_chunk_stages(sai):
    """D=64: stages of one 64-column chunk (the other shared-memory layout)."""
    check_fused(sai, synth.make("flash", S=512, K=100, D=64))


def test_short_sequence_box_under_128_rows(sai):
    """B*S = 64 < 128 Kw rows: the window box has 64 rows and the token's own
    key sits in its last row."""
    check_fused(sai, synth.make("small", B=1, S=64, K=12))


@pytest.mark.parametrize("W", [1, 37, 128])
def test_window_lengths(sai, W):
    """W = 1 (the token's own key alone), an odd length and the full tile."""
    check_fused(sai, synth.make("flash", S=512, K=64, W=W, seed=300 + W))


def test_packed_documents(sai):
    """Two sequences, two documents each: the window clipped at the document
    start; a box reaching into the previous sequence's rows is masked."""
    check_fused(sai, synth.make("packed", B=2, S=512, K=96))


def test_no_sink(sai):
    check_fused(sai, synth.make("flash", S=512, K=100, with_sink=False, seed=77))


@pytest.mark.parametrize("sink_val", [40.0, 200.0])
def test_extreme_sink_floor(sai, sink_val):
    w = synth.make("flash", S=512, K=96, seed=88)
    kf = synth.bf16_to_f32(w.Kw)
    rng = np.random.default_rng(89)
    w.Q[:] = synth.bf16_bits(kf[:, :, None, :] + np.float32(0.1) * rng.standard_normal(w.Q.shape, dtype=np.float32))
    w.sink[:] = sink_val
    check_fused(sai, w)


def test_scattered_and_bad_indices(sai):
    w = synth.make("flash", S=512, K=64, seed=99)
    rng = np.random.default_rng(100)
    idx = w.idx.copy()
    idx[rng.random(idx.shape) < 0.2] = -1
    idx[0, 10, 3] = 100
    idx[0, 200, 7] = w.P
    idx[0, 201, 0] = -5
    w.idx = idx
    t = np.arange(w.S)[None, :, None]
    w.valid = ((idx >= 0) & (idx < w.P) & ((idx + 1) * w.cr - 1 <= t)).astype(np.uint8)
    check_fused(sai, w, err_expect=5)


def test_dense_warm_up(sai):
    """idx = NULL: every causal block is a slot (K = S/cr)."""
    w = synth.make("small", S=512, K=128, seed=31)
    t = to_dev(w)
    wl, p = run_fused(sai, w, t, dense=True)
    dense_idx = np.broadcast_to(np.arange(w.P, dtype=np.int32), (w.B, w.S, w.P))
    owl = oracle.window_lse(w.Q, w.Kw, w.doc_start, w.W, w.scale)
    op, _ = oracle.distill_target(w.Q, w.pool, dense_idx, owl, w.sink, w.doc_start, w.cr, w.scale)
    assert_close("window_lse", wl.cpu().numpy().reshape(-1, w.H) - owl, 0 * owl, tol_wl(owl))
    assert_close("p", p.cpu().numpy().reshape(-1, w.P), op, TOL_P)


@pytest.mark.parametrize("K,S", [(576, 2304), (2048, 8192)])
def test_multi_group_spill_matches_second_sweep(sai, K, S):
    """Two and four TMEM groups per late token (K > 512 at H=64): with the
    spill workspace and without it (second sweep) the fused kernel's window
    log-mass is bit-identical and its p agrees within the target's
    tolerance; both match the oracle on late tokens and a sample of the
    rest."""
    w = synth.make("long", S=S, K=K)
    t = to_dev(w)
    ws_bytes = sai.target_workspace_bytes(w.B, S, w.H, w.D, K)
    assert ws_bytes > 0
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    wl1, p1 = run_fused(sai, w, t, workspace=ws)
    wl2 = torch.full_like(wl1, float("nan"))
    p2 = torch.full_like(p1, float("nan"))
    st = sai.lib().sai_distill_target_window(
        ctypes.c_void_p(t["Q"].data_ptr()), ctypes.c_void_p(t["Kw"].data_ptr()),
        ctypes.c_void_p(t["pool"].data_ptr()), ctypes.c_void_p(t["idx"].data_ptr()),
        ctypes.c_void_p(t["sink"].data_ptr()), None, w.B, S, w.H, w.D, K, w.cr, w.W, ctypes.c_float(w.scale),
        ctypes.c_void_p(p2.data_ptr()), ctypes.c_void_p(wl2.data_ptr()), None, None, 0,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(wl1, wl2)
    assert_close("p spill vs second sweep", p1.cpu().numpy(), p2.cpu().numpy(), TOL_P)
    tok = np.unique(np.concatenate([np.arange(S - 24, S), synth.sample_tokens(w.B, S, 24)]))
    owl, op, _, _, _ = oracle.run_all(w, tok)
    assert_close("window_lse", wl1.cpu().numpy().reshape(-1, w.H)[tok] - owl, 0 * owl, tol_wl(owl))
    assert_close("p", p1.cpu().numpy().reshape(-1, K)[tok], op, TOL_P)
    assert_close("p (second sweep)", p2.cpu().numpy().reshape(-1, K)[tok], op, TOL_P)


@pytest.mark.parametrize("fused", [False, True])
def test_pro_shape_sampled(sai, fused):
    """The V4-Pro head count with its 1024 pool entries (H=128, K=1024,
    S=4096): two score tiles per TMEM group, so late tokens take four groups
    through the raw-score spill. Both routes, against the oracle on the last
    tokens and a sample of the rest."""
    w = synth.make("flash", S=4096, K=1024, H=128, seed=2024)
    t = to_dev(w)
    if fused:
        wl, p = run_fused(sai, w, t)
    else:
        wl = sai.window_lse(t["Q"], t["Kw"], w.W, w.scale)
        p = sai.distill_target(t["Q"], t["pool"], t["idx"], wl, w.cr, w.scale, sink=t["sink"])
        torch.cuda.synchronize()
    tok = np.unique(np.concatenate([np.arange(w.S - 16, w.S), synth.sample_tokens(w.B, w.S, 32)]))
    owl, op, _, _, _ = oracle.run_all(w, tok)
    assert_close("window_lse", wl.cpu().numpy().reshape(-1, w.H)[tok] - owl, 0 * owl, tol_wl(owl))
    assert_close("p", p.cpu().numpy().reshape(-1, w.K)[tok], op, TOL_P)


def test_matches_three_call_route(sai):
    """The fused call and window_lse -> distill_target agree to within both
    routes' tolerance of the oracle, and the fused call is deterministic."""
    w = synth.make("flash", S=1024, K=200, seed=11)
    t = to_dev(w)
    wl_a, p_a = run_fused(sai, w, t)
    wl_b, p_b = run_fused(sai, w, t)
    assert torch.equal(p_a, p_b) and torch.equal(wl_a, wl_b)
    wl3 = sai.window_lse(t["Q"], t["Kw"], w.W, w.scale, t["doc_start"])
    p3 = sai.distill_target(t["Q"], t["pool"], t["idx"], wl3, w.cr, w.scale, sink=t["sink"],
                            doc_start=t["doc_start"])
    torch.cuda.synchronize()
    ref = wl3.cpu().numpy()
    assert_close("window_lse", wl_a.cpu().numpy() - ref, 0 * ref, 2 * tol_wl(ref))
    assert_close("p", p_a.cpu().numpy(), p3.cpu().numpy(), 2 * TOL_P)


def test_without_window_out(sai):
    """window_lse out = NULL: p is unchanged."""
    w = synth.make("flash", S=512, K=96, seed=12)
    t = to_dev(w)
    _, p_a = run_fused(sai, w, t)
    p_b = sai.distill_target_window(t["Q"], t["Kw"], t["pool"], t["idx"], w.W, w.cr, w.scale,
                                    sink=t["sink"], doc_start=t["doc_start"])
    torch.cuda.synchronize()
    assert torch.equal(p_a, p_b)


def test_unsupported_shapes_refused(sai):
    """W > 128, or a shape only the CUDA-core kernels take (H = 4): refused
    with SAI_ERR_UNSUPPORTED before anything runs; no fallback."""
    w = synth.make("flash", S=512, K=64, seed=13)
    t = to_dev(w)
    with pytest.raises(sai.SaiError) as e:
        sai.distill_target_window(t["Q"], t["Kw"], t["pool"], t["idx"], 129, w.cr, w.scale, sink=t["sink"])
    assert e.value.status == 3
    wt = synth.make("tiny")
    tt = to_dev(wt)
    with pytest.raises(sai.SaiError) as e:
        sai.distill_target_window(tt["Q"], tt["Kw"], tt["pool"], tt["idx"], wt.W, wt.cr, wt.scale)
    assert e.value.status == 3


def test_flash_full_size(sai):
    """The V4-Flash workload, every token: window log-mass, p, and the loss
    and dscores of the KL stage on the fused target."""
    check_fused(sai, synth.make("flash"))


def test_packed_full_size_sampled(sai):
    w = synth.make("packed")
    tok = synth.sample_tokens(w.B, w.S, 256)
    check_fused(sai, w, tokens=tok)


def test_long_full_size_sampled(sai):
    w = synth.make("long")
    tok = np.unique(np.concatenate([np.arange(w.S - 32, w.S), synth.sample_tokens(w.B, w.S, 96)]))
    check_fused(sai, w, tokens=tok)
