"""fp64 CPU oracle for the CSA indexer distillation loss (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` leg may import this package; the product path
(``sparse_attention_indexer_window_b200``) never does. The arithmetic lives in
``oracle.c``; this file only builds it with gcc and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP, IEEE fp64)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int64
        Dd = ctypes.c_double
        lib.orc_window_lse.argtypes = [P, P, P, I, I, I, I, I, Dd, P, I, P]
        lib.orc_window_lse.restype = None
        lib.orc_distill_target.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, Dd, P, I, ctypes.c_int, P]
        lib.orc_distill_target.restype = I
        lib.orc_count_valid_rows.argtypes = [P, I, I]
        lib.orc_count_valid_rows.restype = I
        lib.orc_distill_kl.argtypes = [P, P, P, I, I, Dd, I, P, P, P]
        lib.orc_distill_kl.restype = None
        lib.orc_indexer_topk.argtypes = [P, P, I, I, I, I, P, I, P, P, P]
        lib.orc_indexer_topk.restype = None
        lib.orc_num_threads.argtypes = []
        lib.orc_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use."""
    return int(_load().orc_num_threads())


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _tokens(tokens, B, S):
    if tokens is None:
        return None, B * S
    t = np.ascontiguousarray(tokens, dtype=np.int64)
    return t, t.size


def window_lse(Q, Kw, doc_start, W: int, scale: float, tokens=None) -> np.ndarray:
    """[n, H] fp64 window log-mass for the flat token ids in ``tokens``."""
    B, S, H, D = Q.shape
    Q = _c(Q, np.uint16); Kw = _c(Kw, np.uint16); ds = _c(doc_start, np.int32)
    tk, n = _tokens(tokens, B, S)
    out = np.empty((n, H), dtype=np.float64)
    _load().orc_window_lse(_ptr(Q), _ptr(Kw), _ptr(ds), B, S, H, D, W, float(scale),
                           _ptr(tk), n, _ptr(out))
    return out


def distill_target(Q, pool, idx, wl, sink, doc_start, cr: int, scale: float, tokens=None,
                   per_branch: bool = False, full_lse: bool = False):
    """(p [n, K] fp64, bad_index_count) for the flat token ids in ``tokens``.

    per_branch selects the earlier per-branch target (every head normalised
    over the selected entries alone, floor 1e-10); wl and sink are then
    unused and may be None. full_lse says that wl already holds lse_full,
    the per-head log-normaliser of the whole attention row (window, selected
    entries and sink) as a CSA attention forward returns it; sink is then
    unused. idx=None is the dense warm-up stage: slot k is compressed block k
    for every token (K = S/cr)."""
    B, S, H, D = Q.shape
    if idx is None:
        idx = np.broadcast_to(np.arange(S // cr, dtype=np.int32), (B, S, S // cr))
    K = idx.shape[-1]
    Q = _c(Q, np.uint16); pool = _c(pool, np.uint16); idx = _c(idx, np.int32)
    wl = _c(wl, np.float64); sink = _c(sink, np.float32); ds = _c(doc_start, np.int32)
    tk, n = _tokens(tokens, B, S)
    assert not (per_branch and full_lse)
    mode = 1 if per_branch else (2 if full_lse else 0)
    if per_branch:
        wl = None
    else:
        assert wl.shape == (n, H)
    if per_branch or full_lse:
        sink = None
    p = np.empty((n, K), dtype=np.float64)
    bad = _load().orc_distill_target(_ptr(Q), _ptr(pool), _ptr(idx), _ptr(wl), _ptr(sink), _ptr(ds),
                                     B, S, H, D, K, cr, float(scale), _ptr(tk), n, mode,
                                     _ptr(p))
    return p, int(bad)


def count_valid_rows(valid) -> int:
    v = _c(valid, np.uint8)
    K = v.shape[-1]
    return int(_load().orc_count_valid_rows(_ptr(v), v.size // K, K))


def distill_kl(p, scores, valid, coeff: float, n_norm: int = -1):
    """(loss, dscores [rows, K], kl_rows [rows]) in fp64."""
    K = scores.shape[-1]
    p = _c(p, np.float64).reshape(-1, K)
    s = _c(scores, np.float32).reshape(-1, K)
    v = _c(valid, np.uint8).reshape(-1, K)
    rows = s.shape[0]
    loss = np.zeros(1, dtype=np.float64)
    ds = np.empty((rows, K), dtype=np.float64)
    klr = np.empty(rows, dtype=np.float64)
    _load().orc_distill_kl(_ptr(p), _ptr(s), _ptr(v), rows, K, float(coeff), int(n_norm),
                           _ptr(loss), _ptr(ds), _ptr(klr))
    return float(loss[0]), ds, klr


def run_all(w, tokens=None):
    """The whole path on a workload: (wl, p, loss, dscores) for the token list
    (all tokens when None). With a token sample, the loss is not formed (it
    needs every row); dscores use the batch-wide valid-token count."""
    wl = window_lse(w.Q, w.Kw, w.doc_start, w.W, w.scale, tokens)
    p, bad = distill_target(w.Q, w.pool, w.idx, wl, w.sink, w.doc_start, w.cr, w.scale, tokens)
    K = w.K
    if tokens is None:
        loss, ds, _ = distill_kl(p, w.scores, w.valid, w.coeff)
    else:
        n_all = count_valid_rows(w.valid)
        loss = None
        _, ds, _ = distill_kl(p, w.scores.reshape(-1, K)[tokens], w.valid.reshape(-1, K)[tokens],
                              w.coeff, n_norm=n_all)
    return wl, p, loss, ds, bad


def indexer_topk(scores, doc_start, cr: int, K: int, tokens=None):
    """(idx [n, K] int32, sel [n, K] fp32, valid [n, K] uint8): the top-K
    candidate blocks of each token by indexer score, in ascending block
    order with a -1 tail; ``scores`` is [B, S, S/cr] fp32."""
    B, S, P = scores.shape
    assert P * cr == S and 1 <= K <= P
    sc = _c(scores, np.float32); ds = _c(doc_start, np.int32)
    tk, n = _tokens(tokens, B, S)
    idx = np.empty((n, K), dtype=np.int32)
    sel = np.empty((n, K), dtype=np.float32)
    valid = np.empty((n, K), dtype=np.uint8)
    _load().orc_indexer_topk(_ptr(sc), _ptr(ds), B, S, cr, K, _ptr(tk), n, _ptr(idx), _ptr(sel), _ptr(valid))
    return idx, sel, valid
