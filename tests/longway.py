"""The distillation target computed term by term (numpy, fp64).

The Primus page ("perf(deepseek-v4): fuse and enable the indexer distillation
loss", second commit message and "Test plan") checks its fused target against
the joint softmax computed term by term. This is that check in our own form:
for every (token, head) build ONE logit vector that
concatenates the window logits, the selected compressed logits and the sink,
take a softmax over it, keep the compressed part, sum it over heads and
L1-renormalise with the float32-tiny floor.

It deliberately shares nothing with the oracle's decomposition into window,
compressed and sink log-sum-exps: here the window and compressed scores come
from numpy matmuls and the softmax is taken over the concatenated vector.
"""
from __future__ import annotations

import numpy as np

FLT_MIN = float(np.finfo(np.float32).tiny)


def _f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def selected_mask(idx_row: np.ndarray, t: int, cr: int, P: int, d0: int) -> np.ndarray:
    j = idx_row.astype(np.int64)
    return (j >= 0) & (j < P) & ((j + 1) * cr - 1 <= t) & (j * cr >= d0)


def target_long_way(Q, Kw, pool, idx, sink, doc_start, W, cr, scale, tokens=None):
    B, S, H, D = Q.shape
    K = idx.shape[-1]
    P = pool.shape[1]
    Qf, Kf, Pf = _f64(Q), _f64(Kw), _f64(pool)
    toks = range(B * S) if tokens is None else [int(g) for g in tokens]
    out = []
    for g in toks:
        b, t = divmod(g, S)
        d0 = 0 if doc_start is None else min(max(int(doc_start[b, t]), 0), t)
        lo = max(d0, t - W + 1)
        q = Qf[b, t]                                   # [H, D]
        win = scale * (q @ Kf[b, lo:t + 1].T)          # [H, nw]
        sel = selected_mask(idx[b, t], t, cr, P, d0)
        rows = idx[b, t][sel].astype(np.int64)
        comp = scale * (q @ Pf[b, rows].T)             # [H, n_sel]
        parts = [win, comp]
        if sink is not None:
            parts.append(sink.astype(np.float64)[:, None])
        logits = np.concatenate(parts, axis=1)         # the joint vector per head
        mx = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - mx)
        soft = e / e.sum(axis=1, keepdims=True)
        share = soft[:, win.shape[1]:win.shape[1] + comp.shape[1]]  # compressed part
        mass = share.sum(axis=0)                       # head sum, [n_sel]
        m = mass.sum()
        row = np.zeros(K)
        row[np.nonzero(sel)[0]] = mass / max(m, FLT_MIN)
        out.append(row)
    return np.array(out).reshape(-1, K)


def joint_lse_long_way(Q, Kw, pool, idx, sink, doc_start, W, cr, scale):
    """[B*S, H]: log of the joint softmax's denominator per (token, head), i.e.
    the log-normaliser a CSA attention forward over the window keys, the
    selected compressed rows and the sink reports, from the same concatenated
    logit vector as target_long_way."""
    B, S, H, D = Q.shape
    P = pool.shape[1]
    Qf, Kf, Pf = _f64(Q), _f64(Kw), _f64(pool)
    out = np.empty((B * S, H))
    for g in range(B * S):
        b, t = divmod(g, S)
        d0 = 0 if doc_start is None else min(max(int(doc_start[b, t]), 0), t)
        lo = max(d0, t - W + 1)
        q = Qf[b, t]
        sel = selected_mask(idx[b, t], t, cr, P, d0)
        parts = [scale * (q @ Kf[b, lo:t + 1].T), scale * (q @ Pf[b, idx[b, t][sel].astype(np.int64)].T)]
        if sink is not None:
            parts.append(sink.astype(np.float64)[:, None])
        logits = np.concatenate(parts, axis=1)
        mx = logits.max(axis=1)
        out[g] = mx + np.log(np.exp(logits - mx[:, None]).sum(axis=1))
    return out


def compressed_lse_long_way(Q, pool, idx, doc_start, cr, scale):
    """[B*S, H]: log-sum-exp of each head's selected compressed logits (-inf
    where a token selects nothing)."""
    B, S, H, D = Q.shape
    P = pool.shape[1]
    Qf, Pf = _f64(Q), _f64(pool)
    out = np.full((B * S, H), -np.inf)
    for g in range(B * S):
        b, t = divmod(g, S)
        d0 = 0 if doc_start is None else min(max(int(doc_start[b, t]), 0), t)
        sel = selected_mask(idx[b, t], t, cr, P, d0)
        if sel.any():
            z = scale * (Qf[b, t] @ Pf[b, idx[b, t][sel].astype(np.int64)].T)
            mx = z.max(axis=1)
            out[g] = mx + np.log(np.exp(z - mx[:, None]).sum(axis=1))
    return out
