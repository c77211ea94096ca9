"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each test ties one part of the oracle to something fixed independently: a
value a source page prints (fixtures under tests/golden/), a closed form, a
special case that reduces to a library routine, the joint softmax computed
term by term, or an invariant. They are chosen so that a plausible slip in the
oracle (an off-by-one window bound, a dropped sink or window term, a wrong
causal rule, a transposed operand, a sign error in the gradient) fails one.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.special import logsumexp

import oracle
import synth
from tests.longway import FLT_MIN, compressed_lse_long_way, joint_lse_long_way, target_long_way

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _f64(bits):
    return synth.bf16_to_f32(bits).astype(np.float64)


def _rand_problem(seed, B=1, S=32, H=3, D=16, K=6, cr=4, W=5, docs=False, sink=True, scatter=True):
    rng = np.random.default_rng(seed)
    Q = synth.bf16_bits(rng.standard_normal((B, S, H, D), dtype=np.float32))
    Kw = synth.bf16_bits(rng.standard_normal((B, S, D), dtype=np.float32))
    P = S // cr
    pool = synth.bf16_bits(rng.standard_normal((B, P, D), dtype=np.float32))
    snk = rng.standard_normal(H).astype(np.float32) if sink else None
    ds = None
    if docs:
        ds = np.zeros((B, S), dtype=np.int32)
        for b in range(B):
            s0 = int(rng.integers(1, S))
            ds[b, s0:] = s0
    # indices over the whole pool (some non-causal, so masked) plus -1 scattered
    idx = rng.integers(0, P, size=(B, S, K)).astype(np.int32)
    if scatter:
        idx[rng.random((B, S, K)) < 0.25] = -1
    for b in range(B):
        for t in range(S):
            # keep the selected rows distinct
            seen = set()
            for k in range(K):
                if idx[b, t, k] in seen:
                    idx[b, t, k] = -1
                elif idx[b, t, k] >= 0:
                    seen.add(int(idx[b, t, k]))
    return Q, Kw, pool, idx, snk, ds


# ---------------------------------------------------------------- window_lse

def test_window_single_key_is_the_logit():
    """W = 1: the window is the token itself, so the log-mass is its one logit."""
    Q, Kw, *_ = _rand_problem(1, B=2, S=16, H=3, D=16)
    scale = 0.25
    wl = oracle.window_lse(Q, Kw, None, 1, scale)
    q, k = _f64(Q), _f64(Kw)
    expect = scale * np.einsum("bthd,btd->bth", q, k).reshape(-1, 3)
    np.testing.assert_allclose(wl, expect, rtol=0, atol=1e-13)


@pytest.mark.parametrize("W", [1, 3, 7, 40])
def test_window_zero_queries_counts_keys(W):
    """q = 0: every logit is 0, so the log-mass is log(number of window keys),
    min(W, t - d0 + 1) with the document start d0."""
    S, H, D = 24, 2, 8
    Q = np.zeros((2, S, H, D), dtype=np.uint16)
    Kw = synth.bf16_bits(np.random.default_rng(2).standard_normal((2, S, D), dtype=np.float32))
    ds = np.zeros((2, S), dtype=np.int32)
    ds[1, 9:] = 9
    wl = oracle.window_lse(Q, Kw, ds, W, 0.5).reshape(2, S, H)
    for b in range(2):
        for t in range(S):
            d0 = ds[b, t]
            n = min(W, t - d0 + 1)
            assert wl[b, t, 0] == pytest.approx(math.log(n), abs=1e-14)
            assert wl[b, t, 1] == pytest.approx(math.log(n), abs=1e-14)


def test_window_covering_sequence_is_causal_lse():
    """W >= S: the window is the whole causal prefix; compare with scipy's
    logsumexp over the masked matmul logits."""
    Q, Kw, *_ = _rand_problem(3, B=1, S=20, H=2, D=8)
    scale = 0.3
    wl = oracle.window_lse(Q, Kw, None, 64, scale).reshape(20, 2)
    q, k = _f64(Q)[0], _f64(Kw)[0]
    z = scale * np.einsum("thd,sd->ths", q, k)
    for t in range(20):
        np.testing.assert_allclose(wl[t], logsumexp(z[t, :, :t + 1], axis=1), rtol=0, atol=1e-12)


def test_window_batches_are_independent():
    """Two identical batch rows give identical results (batch offset b*S)."""
    Q, Kw, *_ = _rand_problem(4, B=1, S=12, H=2, D=8)
    Q2, K2 = np.concatenate([Q, Q]), np.concatenate([Kw, Kw])
    wl = oracle.window_lse(Q2, K2, None, 4, 0.5).reshape(2, 12, 2)
    np.testing.assert_array_equal(wl[0], wl[1])


def test_window_token_sample_matches_full():
    Q, Kw, *_ = _rand_problem(5, B=2, S=16, H=2, D=8)
    full = oracle.window_lse(Q, Kw, None, 5, 0.5)
    tok = np.array([0, 3, 17, 31])
    np.testing.assert_array_equal(oracle.window_lse(Q, Kw, None, 5, 0.5, tok), full[tok])


# ------------------------------------------------------------ distill_target

def test_causal_block_rule_golden():
    """MaxText page: with t=4 and compress rate 4, block 0 is allowed and
    block 1 masked. With q = 0 the target is uniform over allowed slots."""
    g = _gold("causal_block_t4_cr4.json")
    t, cr = g["t"], g["cr"]
    S, H, D, K = 8, 1, 8, 2
    Q = np.zeros((1, S, H, D), dtype=np.uint16)
    Kw = np.zeros((1, S, D), dtype=np.uint16)
    pool = np.zeros((1, S // cr, D), dtype=np.uint16)
    idx = np.tile(np.array([0, 1], dtype=np.int32), (1, S, 1))
    wl = oracle.window_lse(Q, Kw, None, 4, 1.0)
    p, bad = oracle.distill_target(Q, pool, idx, wl, None, None, cr, 1.0)
    p = p.reshape(S, K)
    assert bad == 0
    assert (p[t, 0] > 0) == g["allowed"]["0"]
    assert (p[t, 1] > 0) == g["allowed"]["1"]
    assert p[t, 0] == 1.0 and p[t, 1] == 0.0


def test_zero_queries_give_uniform_target():
    """q = 0: all logits tie, so p = 1/n_sel on the allowed slots and 0 on
    masked ones, where n_sel counts slots with 0<=idx<P, (idx+1)*cr-1<=t and
    idx*cr >= document start."""
    Q, Kw, pool, idx, snk, ds = _rand_problem(6, B=2, S=32, H=3, D=8, K=7, docs=True)
    Q[:] = 0
    wl = oracle.window_lse(Q, Kw, ds, 5, 0.5)
    p, bad = oracle.distill_target(Q, pool, idx, wl, snk, ds, 4, 0.5)
    p = p.reshape(2, 32, 7)
    for b in range(2):
        for t in range(32):
            d0 = ds[b, t]
            j = idx[b, t].astype(int)
            ok = (j >= 0) & (j < 8) & ((j + 1) * 4 - 1 <= t) & (j * 4 >= d0)
            n = ok.sum()
            if n == 0:
                assert np.all(p[b, t] == 0)
            else:
                np.testing.assert_allclose(p[b, t][ok], 1.0 / n, rtol=1e-15)
                assert np.all(p[b, t][~ok] == 0)


@pytest.mark.parametrize("seed,docs,sink,W", [(10, False, True, 5), (11, True, True, 3),
                                              (12, False, False, 9), (13, True, False, 1)])
def test_target_matches_joint_softmax_long_way(seed, docs, sink, W):
    Q, Kw, pool, idx, snk, ds = _rand_problem(seed, B=2, S=32, H=3, D=16, K=6, W=W, docs=docs, sink=sink)
    scale = 1 / 4
    wl = oracle.window_lse(Q, Kw, ds, W, scale)
    p, bad = oracle.distill_target(Q, pool, idx, wl, snk, ds, 4, scale)
    ref = target_long_way(Q, Kw, pool, idx, snk, ds, W, 4, scale)
    np.testing.assert_allclose(p, ref, rtol=0, atol=1e-12)


def test_target_long_way_on_tiny_workload():
    w = synth.make("tiny")
    wl = oracle.window_lse(w.Q, w.Kw, w.doc_start, w.W, w.scale)
    p, bad = oracle.distill_target(w.Q, w.pool, w.idx, wl, w.sink, w.doc_start, w.cr, w.scale)
    ref = target_long_way(w.Q, w.Kw, w.pool, w.idx, w.sink, w.doc_start, w.W, w.cr, w.scale)
    assert bad == 0
    np.testing.assert_allclose(p, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("docs", [False, True])
def test_dense_mode_is_every_causal_block(docs):
    """Dense warm-up (idx omitted): slot k is compressed block k. The target
    equals the joint softmax computed term by term over the explicit
    index row 0..P-1, puts exactly zero on blocks a token cannot see (the
    MaxText page's rule: with t=4, cr=4 block 0 visible, block 1 masked), and
    with every block visible equals the sparse target that selects them all."""
    S, H, D, cr, W = 32, 3, 16, 4, 5
    Q, Kw, pool, _, snk, ds = _rand_problem(40, B=1, S=S, H=H, D=D, K=6, cr=cr, docs=docs)
    P = S // cr
    scale = 0.25
    wl = oracle.window_lse(Q, Kw, ds, W, scale)
    p, bad = oracle.distill_target(Q, pool, None, wl, snk, ds, cr, scale)
    assert bad == 0 and p.shape == (S, P)
    arange = np.broadcast_to(np.arange(P, dtype=np.int32), (1, S, P)).copy()
    ref = target_long_way(Q, Kw, pool, arange, snk, ds, W, cr, scale)
    np.testing.assert_allclose(p, ref, rtol=0, atol=1e-12)
    t = 4
    assert p[t, 0] > 0 and np.all(p[t, 1:] == 0)
    for t in range(S):
        d0 = 0 if ds is None else min(max(int(ds[0, t]), 0), t)
        for j in range(P):
            if (j + 1) * cr - 1 > t or j * cr < d0:
                assert p[t, j] == 0.0
    if not docs:
        t = S - 1
        idx = np.full((1, S, P), -1, dtype=np.int32)
        idx[0, t] = np.arange(P)[::-1]                 # all blocks, another slot order
        ps, _ = oracle.distill_target(Q, pool, idx, wl, snk, None, cr, scale)
        np.testing.assert_allclose(ps[t][::-1], p[t], rtol=1e-13, atol=0)


def test_target_long_way_on_small_workload_sample():
    """The local-branch-dominates workload (sink +8, q aligned to the key)."""
    w = synth.make("small")
    tok = synth.sample_tokens(w.B, w.S, 48)
    wl = oracle.window_lse(w.Q, w.Kw, w.doc_start, w.W, w.scale, tok)
    p, bad = oracle.distill_target(w.Q, w.pool, w.idx, wl, w.sink, w.doc_start, w.cr, w.scale, tok)
    ref = target_long_way(w.Q, w.Kw, w.pool, w.idx, w.sink, w.doc_start, w.W, w.cr, w.scale, tok)
    np.testing.assert_allclose(p, ref, rtol=0, atol=1e-12)


def test_target_per_branch_limit_is_maxtext_formula():
    """With no sink and a window whose logits are pushed to -200, the joint
    target reduces to the MaxText page's per-branch formula
    L1_Normalize(Sum_h Softmax_k(z)), computed here with scipy's softmax."""
    from scipy.special import softmax
    Q, Kw, pool, idx, _, _ = _rand_problem(20, B=1, S=32, H=3, D=16, K=6, scatter=False)
    # window keys = -c * q of head 0 direction makes every window logit very
    # negative only for a single-key window whose key opposes every head: use
    # one shared direction for all heads and keys.
    rng = np.random.default_rng(21)
    v = rng.standard_normal(16).astype(np.float32)
    v /= np.linalg.norm(v)
    qf = np.abs(rng.standard_normal((1, 32, 3, 1))).astype(np.float32) + 1.0
    Qx = synth.bf16_bits(qf * v[None, None, None, :] * 8)
    Kx = synth.bf16_bits(np.tile(-v * 200.0, (1, 32, 1)))
    scale = 1.0
    wl = oracle.window_lse(Qx, Kx, None, 1, scale)
    assert wl.max() < -100
    p, _ = oracle.distill_target(Qx, pool, idx, wl, None, None, 4, scale)
    q, pl = _f64(Qx)[0], _f64(pool)[0]
    for t in range(32):
        j = idx[0, t].astype(int)
        ok = (j >= 0) & ((j + 1) * 4 - 1 <= t)
        if not ok.any():
            continue
        z = scale * q[t] @ pl[j[ok]].T                 # [H, n]
        ref = softmax(z, axis=1).sum(axis=0)
        ref = ref / ref.sum()
        np.testing.assert_allclose(p.reshape(32, 6)[t][ok], ref, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("seed,docs", [(30, False), (31, True)])
def test_per_branch_mode_is_maxtext_formula(seed, docs):
    """The per-branch mode is the MaxText page's formula as printed:
    L1_Normalize(Sum_h Softmax_k(z)) over the selected entries, computed here
    with scipy's softmax from the same inputs; window and sink play no part."""
    from scipy.special import softmax
    S, H, D, K, cr = 32, 3, 16, 6, 4
    Q, _, pool, idx, snk, ds = _rand_problem(seed, B=1, S=S, H=H, D=D, K=K, cr=cr, docs=docs)
    scale = 0.3
    p, bad = oracle.distill_target(Q, pool, idx, None, None, ds, cr, scale, per_branch=True)
    assert bad == 0
    q, pl = _f64(Q)[0], _f64(pool)[0]
    p = p.reshape(S, K)
    for t in range(S):
        d0 = 0 if ds is None else min(max(int(ds[0, t]), 0), t)
        j = idx[0, t].astype(int)
        ok = (j >= 0) & ((j + 1) * cr - 1 <= t) & (j * cr >= d0)
        if not ok.any():
            assert np.all(p[t] == 0.0)
            continue
        z = scale * q[t] @ pl[j[ok]].T                 # [H, n]
        ref = softmax(z, axis=1).sum(axis=0)
        ref = ref / ref.sum()
        np.testing.assert_allclose(p[t][ok], ref, rtol=1e-12, atol=1e-15)
        assert np.all(p[t][~ok] == 0.0)


def test_per_branch_mode_ignores_window_and_sink_and_sums_to_one():
    """Changing the window log-mass or the sink cannot move the per-branch
    target, while it does move the joint one; every non-empty row sums to 1
    (each head contributes a full distribution, so the 1e-10 floor is idle)."""
    Q, Kw, pool, idx, snk, _ = _rand_problem(32, B=1, S=32, H=3, D=16, K=6)
    wl = oracle.window_lse(Q, Kw, None, 5, 0.25)
    p1, _ = oracle.distill_target(Q, pool, idx, wl, snk, None, 4, 0.25, per_branch=True)
    p2, _ = oracle.distill_target(Q, pool, idx, wl + 5.0, snk * 0 + 30.0, None, 4, 0.25, per_branch=True)
    np.testing.assert_array_equal(p1, p2)
    j1, _ = oracle.distill_target(Q, pool, idx, wl, snk, None, 4, 0.25)
    j2, _ = oracle.distill_target(Q, pool, idx, wl + 5.0, snk, None, 4, 0.25)
    assert np.abs(j1 - j2).max() > 1e-3
    rows = p1.sum(axis=1)
    nonempty = rows > 0
    np.testing.assert_allclose(rows[nonempty], 1.0, rtol=1e-12)


@pytest.mark.parametrize("seed,docs,sink,W", [(50, False, True, 5), (51, True, True, 3), (52, True, False, 7)])
def test_full_lse_mode_with_joint_lse_is_joint_target(seed, docs, sink, W):
    """Handing the target the joint softmax's own log-normaliser (the LSE a
    CSA attention forward over window, selected rows and sink returns,
    computed here the long way) reproduces the joint target written out term
    by term; the sink is inside that LSE and must not be added again."""
    Q, Kw, pool, idx, snk, ds = _rand_problem(seed, B=2, S=32, H=3, D=16, K=6, W=W, docs=docs, sink=sink)
    scale = 1 / 4
    lf = joint_lse_long_way(Q, Kw, pool, idx, snk, ds, W, 4, scale)
    p, bad = oracle.distill_target(Q, pool, idx, lf, snk, ds, 4, scale, full_lse=True)
    assert bad == 0
    ref = target_long_way(Q, Kw, pool, idx, snk, ds, W, 4, scale)
    np.testing.assert_allclose(p, ref, rtol=0, atol=1e-12)
    p_nosink, _ = oracle.distill_target(Q, pool, idx, lf, None, ds, 4, scale, full_lse=True)
    np.testing.assert_array_equal(p, p_nosink)


def test_full_lse_mode_is_shift_invariant():
    """A common offset c on every head's LSE scales every u_k by exp(-c), so
    the L1-normalised p does not move (the floor stays idle here); an offset
    on one head alone re-weights that head and does move p."""
    Q, Kw, pool, idx, snk, ds = _rand_problem(53, B=1, S=32, H=3, D=16, K=6, docs=True)
    scale = 0.3
    lf = joint_lse_long_way(Q, Kw, pool, idx, snk, ds, 5, 4, scale)
    p0, _ = oracle.distill_target(Q, pool, idx, lf, None, ds, 4, scale, full_lse=True)
    p1, _ = oracle.distill_target(Q, pool, idx, lf + 3.7, None, ds, 4, scale, full_lse=True)
    np.testing.assert_allclose(p1, p0, rtol=1e-12, atol=1e-15)
    lf2 = lf.copy()
    lf2[:, 1] += 3.0
    p2, _ = oracle.distill_target(Q, pool, idx, lf2, None, ds, 4, scale, full_lse=True)
    assert np.abs(p2 - p0).max() > 1e-3


def test_full_lse_mode_with_compressed_lse_is_per_branch():
    """With each head's own compressed LSE as the given normaliser every head
    contributes a full distribution over its selected rows: the per-branch
    target (its 1e-10 floor is idle, the row mass being H)."""
    Q, Kw, pool, idx, snk, ds = _rand_problem(54, B=2, S=32, H=4, D=16, K=6, docs=True)
    scale = 0.25
    lc = compressed_lse_long_way(Q, pool, idx, ds, 4, scale)
    lc = np.where(np.isfinite(lc), lc, 0.0)   # tokens with nothing selected: p is 0 regardless
    p, _ = oracle.distill_target(Q, pool, idx, lc, None, ds, 4, scale, full_lse=True)
    pb, _ = oracle.distill_target(Q, pool, idx, None, None, ds, 4, scale, per_branch=True)
    np.testing.assert_allclose(p, pb, rtol=0, atol=1e-13)


def _topk_golden_inputs():
    g = _gold("indexer_topk_small.json")
    B, S, cr, K = g["B"], g["S"], g["cr"], g["K"]
    sc = np.zeros((B, S, S // cr), dtype=np.float32)
    sc[:] = -np.inf                                    # blocks a row does not list
    for r in g["rows"]:
        v = [float(x) for x in r["scores"]]
        sc[r["b"], r["t"], :len(v)] = np.array(v, dtype=np.float32)
    ds = np.zeros((B, S), dtype=np.int32)
    ds[1, g["doc_start_batch1_from_t8"]:] = g["doc_start_batch1_from_t8"]
    return g, sc, ds


def test_topk_golden_hand_rows():
    """Rows worked by hand from the selection rules: the largest scores, a
    boundary tie to the lower block, +0 == -0, NaN and -inf never selected,
    the causal block rule and the document rule, -1 padding."""
    g, sc, ds = _topk_golden_inputs()
    assert np.signbit(sc[0, 29, 0]) and not np.signbit(sc[0, 29, 2])
    toks = [r["b"] * g["S"] + r["t"] for r in g["rows"]]
    idx, sel, valid = oracle.indexer_topk(sc, ds, g["cr"], g["K"], tokens=toks)
    for i, r in enumerate(g["rows"]):
        assert idx[i].tolist() == r["idx"], (r["note"], idx[i].tolist())
        for k, j in enumerate(r["idx"]):
            assert valid[i, k] == (1 if j >= 0 else 0)
            want = sc[r["b"], r["t"], j] if j >= 0 else 0.0
            assert sel[i, k] == want or (np.isinf(want) and sel[i, k] == want)


@pytest.mark.parametrize("seed,docs,K,step", [(60, False, 5, 0.5), (61, True, 3, 0.25), (62, True, 8, 0.0)])
def test_topk_selection_properties(seed, docs, K, step):
    """On random scores (rounded to a coarse grid so that ties are common),
    every row satisfies the definition: min(K, candidates) slots filled in
    ascending block order then -1; no unselected candidate scores above a
    selected one; on the boundary score the lowest blocks are taken."""
    rng = np.random.default_rng(seed)
    B, S, cr = 2, 64, 4
    P = S // cr
    sc = rng.standard_normal((B, S, P)).astype(np.float32)
    if step:
        sc = (np.round(sc / step) * step).astype(np.float32)
    sc[rng.random((B, S, P)) < 0.05] = -np.inf
    ds = None
    if docs:
        ds = np.zeros((B, S), dtype=np.int32)
        for b in range(B):
            s0 = int(rng.integers(1, S))
            ds[b, s0:] = s0
    idx, sel, valid = oracle.indexer_topk(sc, ds, cr, K)
    idx = idx.reshape(B, S, K)
    for b in range(B):
        for t in range(S):
            d0 = 0 if ds is None else min(int(ds[b, t]), t)
            j = np.arange(P)
            cand = ((j + 1) * cr - 1 <= t) & (j * cr >= d0) & ~np.isnan(sc[b, t]) & (sc[b, t] != -np.inf)
            n = min(K, int(cand.sum()))
            row = idx[b, t]
            assert np.all(row[n:] == -1) and np.all(row[:n] >= 0)
            chosen = row[:n]
            assert np.all(np.diff(chosen) > 0)
            assert np.all(cand[chosen])
            if n == 0:
                continue
            rest = cand.copy()
            rest[chosen] = False
            lo = sc[b, t, chosen].min()
            if rest.any():
                assert sc[b, t][rest].max() <= lo
                tied_rest = np.nonzero(rest & (sc[b, t] == lo))[0]
                tied_in = chosen[sc[b, t, chosen] == lo]
                if tied_rest.size:
                    assert tied_in.max() < tied_rest.min()
    flat = idx.reshape(-1, K)
    assert np.array_equal(valid, (flat >= 0).astype(np.uint8))
    rows = np.arange(B * S)[:, None]
    want = np.where(flat >= 0, sc.reshape(B * S, P)[rows, np.maximum(flat, 0)], 0.0).astype(np.float32)
    assert np.array_equal(sel, want)


def test_target_invariants():
    Q, Kw, pool, idx, snk, ds = _rand_problem(30, B=2, S=32, H=4, D=16, K=8, docs=True)
    scale = 0.25
    wl = oracle.window_lse(Q, Kw, ds, 6, scale)
    p, _ = oracle.distill_target(Q, pool, idx, wl, snk, ds, 4, scale)
    p = p.reshape(2, 32, 8)
    assert np.all(np.isfinite(p)) and np.all(p >= 0) and np.all(p <= 1)
    sums = p.sum(-1)
    nonempty = sums > 0
    np.testing.assert_allclose(sums[nonempty], 1.0, rtol=0, atol=1e-13)
    # slot permutation permutes p
    perm = np.random.default_rng(31).permutation(8)
    p2, _ = oracle.distill_target(Q, pool, idx[..., perm], wl, snk, ds, 4, scale)
    np.testing.assert_allclose(p2.reshape(2, 32, 8), p[..., perm], rtol=0, atol=1e-15)
    # head permutation (queries, sink and window log-mass together) leaves p
    hp = np.array([2, 0, 3, 1])
    wl2 = oracle.window_lse(Q[:, :, hp], Kw, ds, 6, scale)
    np.testing.assert_array_equal(wl2, wl[:, hp])
    p3, _ = oracle.distill_target(Q[:, :, hp], pool, idx, wl2, snk[hp], ds, 4, scale)
    np.testing.assert_allclose(p3.reshape(2, 32, 8), p, rtol=0, atol=1e-14)


def test_target_empty_row_and_bad_indices():
    Q, Kw, pool, idx, snk, ds = _rand_problem(40, B=1, S=16, H=2, D=8, K=4)
    idx[0, 5] = -1                 # empty row
    idx[0, 9, 0] = 4               # == P: out of range
    idx[0, 9, 1] = -7              # below -1: out of range
    wl = oracle.window_lse(Q, Kw, ds, 4, 0.5)
    p, bad = oracle.distill_target(Q, pool, idx, wl, snk, ds, 4, 0.5)
    p = p.reshape(16, 4)
    assert bad == 2
    assert np.all(p[5] == 0)
    assert p[9, 0] == 0 and p[9, 1] == 0
    assert np.all(np.isfinite(p))


@pytest.mark.parametrize("sink_val", [8.0, 40.0, 200.0])
def test_target_local_branch_dominates(sink_val):
    """A head whose sink and window carry almost all its attention leaves a
    compressed mass far below 1 (about e^-40 for sink=+40, below float32 tiny
    for sink=+200). The target stays finite, non-negative and sums to at most
    1. At sink=+40 the mass lies between float32 tiny and the old 1e-10 floor,
    so the row must still sum to 1: the Primus page moved the floor because
    1e-10 would clip exactly such an almost entirely local query."""
    Q, Kw, pool, idx, snk, ds = _rand_problem(50, B=1, S=32, H=2, D=16, K=6, scatter=False)
    kf = _f64(Kw)
    Qa = synth.bf16_bits((kf[:, :, None, :] + 0.1 * np.random.default_rng(51).standard_normal((1, 32, 2, 16))).astype(np.float32))
    snk = np.full(2, sink_val, dtype=np.float32)
    scale = 0.25
    wl = oracle.window_lse(Qa, Kw, None, 4, scale)
    p, _ = oracle.distill_target(Qa, pool, idx, wl, snk, None, 4, scale)
    ref = target_long_way(Qa, Kw, pool, idx, snk, None, 4, 4, scale)
    assert np.all(np.isfinite(p)) and np.all(p >= 0)
    assert np.all(p.sum(-1) <= 1 + 1e-12)
    np.testing.assert_allclose(p, ref, rtol=0, atol=1e-12)
    if sink_val == 200.0:
        assert p.sum(-1).max() < 1e-6
    if sink_val == 40.0:
        rows = p.sum(-1) > 0
        np.testing.assert_allclose(p.sum(-1)[rows], 1.0, rtol=0, atol=1e-12)


def test_floor_value_golden():
    g = _gold("float32_tiny.json")
    assert FLT_MIN == g["float32_tiny"]
    assert float(np.finfo(np.float32).tiny) == g["float32_tiny"]


# ----------------------------------------------------------------- distill_kl

def test_kl_two_slot_closed_form():
    """p = (1/2, 1/2), scores (0, log 3): q = (1/4, 3/4),
    KL = 1/2 log 2 + 1/2 log(2/3) = 1/2 log(4/3); dscores = coeff (q - p)."""
    p = np.array([[0.5, 0.5]])
    s = np.array([[0.0, math.log(3.0)]], dtype=np.float32)
    v = np.ones((1, 2), dtype=np.uint8)
    loss, ds, klr = oracle.distill_kl(p, s, v, 0.01)
    q1 = 1.0 / (1.0 + math.exp(float(s[0, 1])))
    assert klr[0] == pytest.approx(0.5 * math.log(0.5 / q1) + 0.5 * math.log(0.5 / (1 - q1)), rel=1e-14)
    assert klr[0] == pytest.approx(0.5 * math.log(4.0 / 3.0), rel=1e-7)
    assert loss == pytest.approx(0.01 * klr[0], rel=1e-15)
    np.testing.assert_allclose(ds[0], 0.01 * np.array([q1 - 0.5, (1 - q1) - 0.5]), rtol=1e-13)


def test_kl_zero_when_scores_match_target():
    rng = np.random.default_rng(60)
    p = rng.random((5, 9)) + 0.05
    p /= p.sum(1, keepdims=True)
    s = (np.log(p) + rng.standard_normal((5, 1)))  # any per-row shift
    v = np.ones((5, 9), dtype=np.uint8)
    # fp32 scores carry rounding; evaluate the oracle on exactly those scores
    s32 = s.astype(np.float32)
    pe = np.exp(s32.astype(np.float64))
    pe /= pe.sum(1, keepdims=True)
    loss, ds, _ = oracle.distill_kl(pe, s32, v, 0.01)
    assert abs(loss) < 1e-15
    assert np.abs(ds).max() < 1e-15


def test_kl_gradient_matches_finite_differences():
    rng = np.random.default_rng(70)
    R, K = 4, 7
    p = rng.random((R, K))
    p[0, 2] = 0.0
    p /= p.sum(1, keepdims=True)
    s = rng.standard_normal((R, K)) * 1.4
    v = (rng.random((R, K)) > 0.2).astype(np.uint8)
    v[3] = 0                                     # a row with no valid slot
    coeff = 0.01

    def loss_at(sv):
        # fp64 scores through the float32 interface would lose the step, so
        # the step is applied to values exactly representable in float32
        l, _, _ = oracle.distill_kl(p, sv.astype(np.float32), v, coeff)
        return l

    s = s.astype(np.float32).astype(np.float64)
    _, ds, _ = oracle.distill_kl(p, s.astype(np.float32), v, coeff)
    h = 2.0 ** -12
    for r in range(R):
        for k in range(K):
            sp, sm = s.copy(), s.copy()
            sp[r, k] += h
            sm[r, k] -= h
            fd = (loss_at(sp) - loss_at(sm)) / (2 * h)
            assert fd == pytest.approx(ds[r, k], rel=1e-6, abs=1e-12)
    assert np.all(ds[3] == 0)
    assert np.all(ds[v == 0] == 0)


def test_kl_masked_rows_do_not_count():
    rng = np.random.default_rng(80)
    p = rng.random((3, 4)); p /= p.sum(1, keepdims=True)
    s = rng.standard_normal((3, 4)).astype(np.float32)
    v = np.ones((3, 4), dtype=np.uint8)
    v[1] = 0
    loss3, ds3, klr = oracle.distill_kl(p, s, v, 1.0)
    keep = [0, 2]
    loss2, ds2, _ = oracle.distill_kl(p[keep], s[keep], v[keep], 1.0)
    assert klr[1] == 0.0
    assert loss3 == pytest.approx(loss2, rel=1e-15)
    np.testing.assert_allclose(ds3[keep], ds2, rtol=1e-15)


def test_kl_single_slot_is_zero():
    p = np.array([[1.0], [0.0]])
    s = np.array([[3.0], [-2.0]], dtype=np.float32)
    v = np.ones((2, 1), dtype=np.uint8)
    loss, ds, _ = oracle.distill_kl(p, s, v, 0.01)
    assert loss == 0.0
    assert ds[0, 0] == 0.0


def test_kl_gradient_sums_to_zero_when_target_normalised():
    rng = np.random.default_rng(90)
    p = rng.random((6, 10)); p /= p.sum(1, keepdims=True)
    s = rng.standard_normal((6, 10)).astype(np.float32)
    v = np.ones((6, 10), dtype=np.uint8)
    _, ds, _ = oracle.distill_kl(p, s, v, 0.01)
    np.testing.assert_allclose(ds.sum(1), 0.0, atol=1e-17)


# ------------------------------------------------------------- the workloads

def test_workload_shapes_and_indices():
    g = _gold("v4_flash_gather.json")
    sp = synth.CONFIGS["flash"]
    gathered = sp.B * sp.S * sp.K * sp.D * g["dtype_bytes"]
    assert round(gathered / 1e9, 1) == g["gathered_bytes_GB"]
    for name in ("tiny", "small"):
        w = synth.make(name)
        P = w.S // w.cr
        for b in range(w.B):
            for t in range(w.S):
                row = w.idx[b, t]
                sel = row[row >= 0]
                assert len(set(sel.tolist())) == len(sel)
                assert np.all((sel + 1) * w.cr - 1 <= t)
                assert len(sel) == min(w.K, (t + 1) // w.cr)
                assert np.all(row[len(sel):] == -1)


def test_end_to_end_oracle_finite_on_tiny():
    w = synth.make("tiny")
    wl, p, loss, ds, bad = oracle.run_all(w)
    assert bad == 0
    assert np.isfinite(loss) and loss > 0
    assert np.all(np.isfinite(ds))
