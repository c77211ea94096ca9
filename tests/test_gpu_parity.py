"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Element-by-element on seeded inputs: the whole batch where the oracle
finishes in seconds (the tiny and small workloads and mid-size cuts of the
V4-Flash recipe that span several tiles with a ragged tail, several TMEM
groups, document packing and the extreme-sink floor) and the full V4-Flash,
packed and long-context workloads, every token, in the launch configuration the
benchmark times. Tolerances (tests/gpu_util.py): p 1e-5, loss 1e-4 relative,
dscores 1e-6 (and 1e-3 of max|dscores|), window_lse 1e-5 relative to max(1,|x|).
Index and mask work must be exact: p and dscores are exactly 0 on masked slots.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import (TOL_DS, TOL_DS_REL_MAX, TOL_LOSS_REL, TOL_P, assert_close, run_chain, to_dev,
                            tol_wl)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sai():
    import sparse_attention_indexer_window_b200 as m
    return m


_CACHE = {}


def workload(key, **kw):
    if key not in _CACHE:
        _CACHE[key] = synth.make(**kw)
    return _CACHE[key]


def check_full(sai, w, *, err_expect=0):
    t = to_dev(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    wl, p, loss, ds = run_chain(sai, w, t, err)
    owl, op, oloss, ods, bad = oracle.run_all(w)
    assert (bad > 0) == (err_expect != 0)
    assert int(err.item()) == err_expect
    assert_close("window_lse", wl.cpu().numpy().reshape(-1, w.H) - owl, 0 * owl, tol_wl(owl))
    pg = p.cpu().numpy().reshape(-1, w.K)
    assert_close("p", pg, op, TOL_P)
    # bit-exact masks: p is exactly 0 wherever the oracle's is
    assert np.all(pg[op == 0] == 0)
    lg = float(loss.item())
    # a float32 result cannot resolve below its spacing at zero (2^-149)
    assert abs(lg - oloss) <= TOL_LOSS_REL * abs(oloss) + 2.0 ** -149, (lg, oloss)
    dg = ds.cpu().numpy().reshape(-1, w.K)
    assert_close("dscores", dg, ods, TOL_DS)
    assert np.abs(dg - ods).max() <= TOL_DS_REL_MAX * max(np.abs(ods).max(), 1e-30)
    assert np.all(dg[w.valid.reshape(-1, w.K) == 0] == 0)
    return wl, p, loss, ds


# ------------------------------------------------------------------ full oracle

def test_tiny_full(sai):
    check_full(sai, workload("tiny", name="tiny"))


def test_small_full(sai):
    check_full(sai, workload("small", name="small"))


def test_flash_recipe_ragged_tiles(sai):
    """H=64, D=512 tensor-core path; K=200 leaves a ragged last tile."""
    check_full(sai, workload("flash_s1024_k200", name="flash", S=1024, K=200))


def test_pro_heads_h128(sai):
    # V4-Pro head count: a window tile is one token, two score tiles per TMEM
    # group, so 300 selected slots take two groups
    check_full(sai, workload("pro_s1280_k300", name="flash", S=1280, K=300, H=128))


def test_h32_d256(sai):
    # four tokens per window tile, eight score tiles per TMEM group, D/64 = 4
    check_full(sai, workload("h32_d256", name="flash", S=512, K=96, H=32, D=256))


def test_h64_d128(sai):
    # two 64-column chunks of D: one two-chunk window stage per tile
    check_full(sai, workload("h64_d128", name="flash", S=512, K=100, D=128))


def test_h64_d64(sai):
    # D = 64: stages of one 64-column chunk (the one-chunk shared-memory layout)
    check_full(sai, workload("h64_d64", name="flash", S=512, K=100, D=64))


def test_flash_recipe_odd_k(sai):
    """K not a multiple of 4: idx rows are read directly, not staged."""
    check_full(sai, synth.make("flash", S=512, K=101, seed=4242))


def test_packed_recipe_documents(sai):
    """Two documents per row: window clipped at the document start, blocks
    across the boundary masked, document-2 tokens without a block empty."""
    check_full(sai, workload("packed_b2_s512", name="packed", B=2, S=512, K=96))


def test_no_sink_tensor_core_path(sai):
    w = synth.make("flash", S=512, K=100, with_sink=False, seed=77)
    check_full(sai, w)


@pytest.mark.parametrize("sink_val", [40.0, 200.0])
def test_extreme_sink_floor_tensor_core_path(sai, sink_val):
    """Every head local (q = k_t + noise) with a large sink: the compressed
    mass is about e^-40 (between float32 tiny and 1e-10) or below float32
    tiny (the floor branch). No NaN, and p still matches the oracle."""
    w = synth.make("flash", S=512, K=96, seed=88)
    kf = synth.bf16_to_f32(w.Kw)
    rng = np.random.default_rng(89)
    w.Q[:] = synth.bf16_bits(kf[:, :, None, :] + np.float32(0.1) * rng.standard_normal(w.Q.shape, dtype=np.float32))
    w.sink[:] = sink_val
    check_full(sai, w)


def test_scattered_and_bad_indices(sai):
    """-1 scattered inside rows, non-causal blocks (masked, no error), and two
    out-of-range entries (masked, error word = SAI_ERR_INDEX)."""
    w = synth.make("flash", S=512, K=64, seed=99)
    rng = np.random.default_rng(100)
    idx = w.idx.copy()
    idx[rng.random(idx.shape) < 0.2] = -1
    # non-causal: a future block
    idx[0, 10, 3] = 100
    idx[0, 300, 5] = w.P - 1
    idx[0, 200, 7] = w.P          # out of range
    idx[0, 201, 0] = -5           # out of range
    w.idx = idx
    w.valid = (idx >= 0).astype(np.uint8)
    # valid must follow the selection rule: clear the masked ones
    t = np.arange(w.S)[None, :, None]
    ok = (idx >= 0) & (idx < w.P) & ((idx + 1) * w.cr - 1 <= t)
    w.valid = ok.astype(np.uint8)
    check_full(sai, w, err_expect=5)


def test_random_slot_order_permutes_outputs(sai):
    w = synth.make("flash", S=512, K=80, seed=123)
    t = to_dev(w)
    _, p1, l1, d1 = run_chain(sai, w, t)
    perm = np.random.default_rng(5).permutation(w.K)
    w2 = synth.make("flash", S=512, K=80, seed=123)
    w2.idx = np.ascontiguousarray(w.idx[..., perm])
    w2.valid = np.ascontiguousarray(w.valid[..., perm])
    w2.scores = np.ascontiguousarray(w.scores[..., perm])
    _, p2, l2, d2 = run_chain(sai, w2, to_dev(w2))
    np.testing.assert_allclose(p2.cpu().numpy(), p1.cpu().numpy()[..., perm], rtol=0, atol=2e-7)
    np.testing.assert_allclose(d2.cpu().numpy(), d1.cpu().numpy()[..., perm], rtol=0, atol=1e-9)


def test_many_tiles_few_heads(sai):
    """H=16 with up to 700 selected slots per token: six 128-slot tiles in one
    TMEM group (row offsets read from shared memory). Sampled tokens."""
    w = workload("small_s4096_k700", name="small", S=4096, K=700, B=1)
    t = to_dev(w)
    wl, p, loss, ds = run_chain(sai, w, t)
    tok = np.unique(np.concatenate([np.arange(w.S - 24, w.S), synth.sample_tokens(w.B, w.S, 40)]))
    owl, op, _, ods, bad = oracle.run_all(w, tok)
    assert_close("window_lse", wl.cpu().numpy().reshape(-1, w.H)[tok] - owl, 0 * owl, tol_wl(owl))
    assert_close("p", p.cpu().numpy().reshape(-1, w.K)[tok], op, TOL_P)
    assert_close("dscores", ds.cpu().numpy().reshape(-1, w.K)[tok], ods, TOL_DS)


def test_multi_group_tokens(sai):
    """More than 512 selected slots per token at H=64 (two TMEM groups, the
    two-pass statistics path). Sampled late tokens against the oracle."""
    w = workload("long_s2304", name="long", S=2304, K=576)
    t = to_dev(w)
    wl, p, loss, ds = run_chain(sai, w, t)
    tok = np.unique(np.concatenate([np.arange(w.S - 40, w.S), synth.sample_tokens(w.B, w.S, 40)]))
    owl, op, _, ods, bad = oracle.run_all(w, tok)
    assert_close("window_lse", wl.cpu().numpy().reshape(-1, w.H)[tok] - owl, 0 * owl, tol_wl(owl))
    assert_close("p", p.cpu().numpy().reshape(-1, w.K)[tok], op, TOL_P)
    assert_close("dscores", ds.cpu().numpy().reshape(-1, w.K)[tok], ods, TOL_DS)


@pytest.mark.parametrize("K,S", [(576, 2304), (1000, 4096), (2048, 8192)])
def test_spill_matches_second_sweep(sai, K, S):
    """Tokens of two to four TMEM groups (K > 512 at H=64): the target with its
    raw-score spill (one sweep of gathers and MMAs, the last group kept in
    TMEM) and the two-sweep target without a workspace agree within the
    target's tolerance, and both match the oracle on late tokens (the most
    groups) and a sample of the rest. K=1000 leaves a ragged last group."""
    w = workload(f"long_s{S}_k{K}", name="long", S=S, K=K)
    t = to_dev(w)
    B, H, D = w.B, w.H, w.D
    assert sai.target_workspace_bytes(B, S, H, D, K) > 0
    wl = sai.window_lse(t["Q"], t["Kw"], w.W, w.scale, t["doc_start"])
    p_ws = sai.distill_target(t["Q"], t["pool"], t["idx"], wl, w.cr, w.scale, sink=t["sink"],
                              doc_start=t["doc_start"])
    p_two = torch.full((B, S, K), float("nan"), device="cuda")
    lib = sai.lib()
    st = lib.sai_distill_target_ws(
        ctypes.c_void_p(t["Q"].data_ptr()), ctypes.c_void_p(t["pool"].data_ptr()),
        ctypes.c_void_p(t["idx"].data_ptr()), ctypes.c_void_p(wl.data_ptr()),
        ctypes.c_void_p(t["sink"].data_ptr()), None, B, S, S, 0, H, D, K, w.cr, ctypes.c_float(w.scale), 0,
        ctypes.c_void_p(p_two.data_ptr()), None, None, 0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    pw, pt = p_ws.cpu().numpy(), p_two.cpu().numpy()
    assert_close("p spill vs second sweep", pw, pt, TOL_P)
    assert np.array_equal(pw == 0, pt == 0)   # the same masked slots
    tok = np.unique(np.concatenate([np.arange(w.S - 24, w.S), synth.sample_tokens(w.B, w.S, 24)]))
    _, op, _, _, _ = oracle.run_all(w, tok)
    assert_close("p", pw.reshape(-1, w.K)[tok], op, TOL_P)
    assert_close("p (second sweep)", pt.reshape(-1, w.K)[tok], op, TOL_P)


def test_deterministic(sai):
    w = workload("flash_s1024_k200", name="flash", S=1024, K=200)
    t = to_dev(w)
    a = run_chain(sai, w, t)
    b = run_chain(sai, w, t)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


# ------------------------------------------------------- distill_kl edge cases

@pytest.mark.parametrize("K", [1, 7, 64, 130, 512, 2048])
def test_kl_shapes(sai, K):
    rng = np.random.default_rng(K)
    B, S = 2, 96
    p = rng.random((B, S, K)).astype(np.float64)
    p[rng.random(p.shape) < 0.2] = 0
    valid = (rng.random((B, S, K)) < 0.8).astype(np.uint8)
    valid[0, :5] = 0                       # rows without a valid slot
    p = p * valid
    s = p.sum(-1, keepdims=True)
    p = np.where(s > 0, p / np.where(s > 0, s, 1), 0).astype(np.float32)
    scores = (rng.standard_normal((B, S, K)) * np.sqrt(2)).astype(np.float32)
    loss, ds = sai.distill_kl(torch.from_numpy(p).cuda(), torch.from_numpy(scores).cuda(),
                              torch.from_numpy(valid).cuda(), 0.01)
    ol, ods, _ = oracle.distill_kl(p.astype(np.float64), scores, valid, 0.01)
    assert abs(float(loss.item()) - ol) <= TOL_LOSS_REL * abs(ol)
    assert_close("dscores", ds.cpu().numpy().reshape(-1, K), ods, TOL_DS)
    assert np.all(ds.cpu().numpy()[valid == 0] == 0)


def test_kl_forward_only(sai):
    w = workload("small", name="small")
    t = to_dev(w)
    p = torch.rand((w.B, w.S, w.K), device="cuda")
    l1, d1 = sai.distill_kl(p, t["scores"], t["valid"], w.coeff)
    l2, d2 = sai.distill_kl(p, t["scores"], t["valid"], w.coeff, want_grad=False)
    assert d2 is None and torch.equal(l1, l2)


# ------------------------------------------------------------- full-size runs
# The three full-size workloads against the fp64 oracle over every token: the
# loss within 1e-4 relative, p and dscores element by element, exact zeros on
# masked slots. Each runs the launch configuration the benchmark times.

def test_flash_full_size(sai):
    check_full(sai, workload("flash", name="flash"))


def test_packed_full_size(sai):
    """B=4, two documents per row (the packed-batch recipe), every token."""
    check_full(sai, synth.make("packed"))


def test_long_full_size(sai):
    """S=16384, K=2048: up to 1536 selected slots per token, every token."""
    check_full(sai, synth.make("long"))
