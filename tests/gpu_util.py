"""Helpers shared by the GPU tests: move a synth workload to the device and run
the three C-ABI calls through the Python binding."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances. p, loss and dscores: the benchmark spec's bounds. window_lse: the
# window stage feeds p only through exp(window_lse - lse_full), so a relative
# change of 1e-5 in the window mass (|d wl| <= 1e-5, scaled for large |wl|)
# keeps p inside its own 1e-5 bound.
TOL_P = 1e-5
TOL_LOSS_REL = 1e-4
TOL_DS = 1e-6
TOL_DS_REL_MAX = 1e-3


def tol_wl(ref: np.ndarray) -> np.ndarray:
    return 1e-5 * np.maximum(1.0, np.abs(ref))


def to_dev(w, dev="cuda"):
    t = {}
    t["Q"] = torch.from_numpy(w.Q.view(np.int16)).to(dev).view(torch.bfloat16)
    t["Kw"] = torch.from_numpy(w.Kw.view(np.int16)).to(dev).view(torch.bfloat16)
    t["pool"] = torch.from_numpy(w.pool.view(np.int16)).to(dev).view(torch.bfloat16)
    t["idx"] = torch.from_numpy(w.idx).to(dev)
    t["sink"] = None if w.sink is None else torch.from_numpy(w.sink).to(dev)
    t["doc_start"] = None if w.doc_start is None else torch.from_numpy(w.doc_start).to(dev)
    t["scores"] = torch.from_numpy(w.scores).to(dev)
    t["valid"] = torch.from_numpy(w.valid).to(dev)
    return t


def run_chain(sai, w, t, err=None):
    """window_lse -> distill_target -> distill_kl on the device; outputs are
    pre-filled with NaN so a slot the kernels forget to write shows up."""
    B, S, H, K = w.B, w.S, w.H, w.K
    dev = t["Q"].device
    wl = torch.full((B, S, H), float("nan"), device=dev)
    p = torch.full((B, S, K), float("nan"), device=dev)
    ds = torch.full((B, S, K), float("nan"), device=dev)
    loss = torch.full((1,), float("nan"), device=dev)
    sai.window_lse(t["Q"], t["Kw"], w.W, w.scale, t["doc_start"], out=wl)
    sai.distill_target(t["Q"], t["pool"], t["idx"], wl, w.cr, w.scale, sink=t["sink"],
                       doc_start=t["doc_start"], err=err, out=p)
    sai.distill_kl(p, t["scores"], t["valid"], w.coeff, loss=loss, dscores=ds)
    torch.cuda.synchronize()
    return wl, p, loss, ds


def assert_close(name, got, ref, atol):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    err = np.abs(got - ref)
    bad = err > atol
    if np.any(bad):
        i = np.unravel_index(np.argmax(err - atol), err.shape)
        raise AssertionError(f"{name}: {bad.sum()} elements out of tolerance; worst at {i}: "
                             f"got {got[i]!r} ref {ref[i]!r} |err| {err[i]:.3e}")
