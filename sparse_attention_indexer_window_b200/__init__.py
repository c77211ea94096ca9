"""Thin Python binding of libsai (CSA indexer distillation loss, sm_100a).

Every function marshals torch CUDA tensors into the C ABI of ``include/sai.h``
and raises ``SaiError`` on a non-zero status. There is no computation and no
fallback here: if ``libsai.so`` is missing the import fails.

    window_lse(Q, Kw, W, scale, doc_start=None)                -> [B,S,H] fp32
    distill_target(Q, pool, idx, wl, cr, scale, sink=None, doc_start=None, err=None) -> [B,S,K] fp32
    distill_kl(p, scores, valid, coeff, want_grad=True, workspace=None, n_rows=None) -> (loss[1], dscores)
    distill_target_window(Q, Kw, pool, idx, W, cr, scale, ...) -> [B,S,K] fp32 (window band inside, Q read once)

The token-range calls (window_lse_range, distill_target_range,
count_valid_rows) serve a batch split across GPUs by sequence position; see
shard.py for the call sequence.

bf16 tensors may be passed as torch.bfloat16 or as int16/uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import importlib.util
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsai.so")


def _builder():
    spec = importlib.util.spec_from_file_location("_sai_build", os.path.join(_HERE, "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


# Rebuild when a source is newer than the library (a no-op otherwise).
try:
    _builder().build()
except Exception as exc:  # no nvcc here: only an existing, current library will do
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libsai.so is not built ({LIB_PATH}) and cannot be built: {exc}") from exc

_lib = ctypes.CDLL(LIB_PATH)
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_lib.sai_window_lse.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _P]
_lib.sai_window_lse.restype = _I
_lib.sai_distill_target.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P]
_lib.sai_distill_target.restype = _I
_lib.sai_distill_target_ex.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, ctypes.c_uint,
                                       _P, _P, _P]
_lib.sai_distill_target_ex.restype = _I
TARGET_PER_BRANCH = 1   # flag of sai_distill_target_ex: the earlier per-branch target
TARGET_FULL_LSE = 2     # flag of sai_distill_target_ex: window_lse holds the full per-head LSE
_lib.sai_distill_target_kl_workspace_bytes.argtypes = [_I, _I, _I]
_lib.sai_distill_target_kl_workspace_bytes.restype = ctypes.c_size_t
_lib.sai_distill_target_kl.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, ctypes.c_uint,
                                       _P, _P, _F, _P, _P, _P, _P, ctypes.c_size_t, _P, _P]
_lib.sai_distill_target_kl.restype = _I
_lib.sai_distill_kl_workspace_bytes.argtypes = [_I, _I, _I]
_lib.sai_distill_kl_workspace_bytes.restype = ctypes.c_size_t
_lib.sai_distill_kl.argtypes = [_P, _P, _P, _I, _I, _I, _F, _P, _P, _P, ctypes.c_size_t, _P]
_lib.sai_distill_kl.restype = _I
_lib.sai_window_lse_range.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P]
_lib.sai_window_lse_range.restype = _I
_lib.sai_distill_target_range.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F,
                                          ctypes.c_uint, _P, _P, _P]
_lib.sai_distill_target_range.restype = _I
_lib.sai_distill_target_workspace_bytes.argtypes = [_I, _I, _I, _I, _I]
_lib.sai_distill_target_workspace_bytes.restype = ctypes.c_size_t
_lib.sai_distill_target_ws.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F,
                                       ctypes.c_uint, _P, _P, _P, ctypes.c_size_t, _P]
_lib.sai_distill_target_ws.restype = _I
_lib.sai_distill_target_window.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P,
                                           _P, ctypes.c_size_t, _P]
_lib.sai_distill_target_window.restype = _I
_lib.sai_distill_target_window_range.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                                                 _F, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.sai_distill_target_window_range.restype = _I
_lib.sai_count_valid_rows.argtypes = [_P, _I, _I, _I, _P, _P]
_lib.sai_count_valid_rows.restype = _I
_lib.sai_distill_kl_ex.argtypes = [_P, _P, _P, _I, _I, _I, _F, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.sai_distill_kl_ex.restype = _I
_lib.sai_distill_kl_noalloc.argtypes = [_P, _P, _P, _I, _I, _I, _F, _P, _P, _P]
_lib.sai_distill_kl_noalloc.restype = _I
_lib.sai_distill_kl_noalloc_max_scratch_bytes.argtypes = []
_lib.sai_distill_kl_noalloc_max_scratch_bytes.restype = ctypes.c_size_t
_lib.sai_status_string.argtypes = [_I]
_lib.sai_status_string.restype = ctypes.c_char_p
_lib.sai_indexer_topk.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P]
_lib.sai_indexer_topk.restype = _I
_lib.sai_version.argtypes = []
_lib.sai_version.restype = _I

SAI_ERR_INDEX = 5
SAI_ERR_TIMEOUT = 8


class SaiError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.sai_status_string(status).decode()}")


def lib() -> ctypes.CDLL:
    return _lib


def version() -> int:
    return int(_lib.sai_version())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _check(st: int, where: str):
    if st != 0:
        raise SaiError(st, where)


def _call(fn, dev: torch.device, *args) -> int:
    """Run one C entry point with the tensors' device current: the library
    takes its device (SM count, TMA encoding, the allocation-free call's
    scratch array) from the current device, and the stream passed is that
    device's current stream."""
    with torch.cuda.device(dev):
        return fn(*args, _stream(dev))


def _bf16_bits(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype in (torch.bfloat16, torch.int16, torch.uint16):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        return t
    raise TypeError(f"{name} must be bfloat16 (or its int16/uint16 bit pattern), got {t.dtype}")


def _want(t: Optional[torch.Tensor], name: str, dtype, shape=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def window_lse(Q: torch.Tensor, Kw: torch.Tensor, W: int, scale: float,
               doc_start: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    B, S, H, D = Q.shape
    Q = _bf16_bits(Q, "Q")
    Kw = _bf16_bits(Kw, "Kw")
    if tuple(Kw.shape) != (B, S, D):
        raise ValueError("Kw must be [B,S,D]")
    _want(doc_start, "doc_start", torch.int32, (B, S))
    if out is None:
        out = torch.empty((B, S, H), dtype=torch.float32, device=Q.device)
    _want(out, "out", torch.float32, (B, S, H))
    st = _call(_lib.sai_window_lse, Q.device, _ptr(Q), _ptr(Kw), _ptr(doc_start), B, S, H, D, int(W),
               float(scale), _ptr(out))
    _check(st, "sai_window_lse")
    return out


def window_lse_range(Q: torch.Tensor, Kw: torch.Tensor, W: int, scale: float, t_begin: int, kw_lead: int,
                     doc_start: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """window_lse for sequence positions t_begin .. t_begin+S-1, through
    sai_window_lse_range. Q is the range's [B,S,H,D]; Kw [B,S+kw_lead,D] holds
    the keys from position t_begin-kw_lead on (the range and its halo)."""
    B, S, H, D = Q.shape
    Q = _bf16_bits(Q, "Q")
    Kw = _bf16_bits(Kw, "Kw")
    if tuple(Kw.shape) != (B, S + kw_lead, D):
        raise ValueError(f"Kw must be [B,S+kw_lead,D] = {(B, S + kw_lead, D)}, got {tuple(Kw.shape)}")
    _want(doc_start, "doc_start", torch.int32, (B, S))
    if out is None:
        out = torch.empty((B, S, H), dtype=torch.float32, device=Q.device)
    _want(out, "out", torch.float32, (B, S, H))
    st = _call(_lib.sai_window_lse_range, Q.device, _ptr(Q), _ptr(Kw), _ptr(doc_start), B, S, H, D, int(W),
               int(t_begin), int(kw_lead), float(scale), _ptr(out))
    _check(st, "sai_window_lse_range")
    return out


def _target_inputs(Q, pool, idx, wl, cr, sink, doc_start, err, per_branch, full_lse, S_seq=None,
                   wl_from_kw=False):
    """Checked arguments shared by the target entry points:
    (Q bits, pool bits, K, wl, sink, flags). wl_from_kw: the window log-mass
    is formed from Kw inside the kernel (wl is not an input)."""
    B, S, H, D = Q.shape
    S_seq = S if S_seq is None else S_seq
    K = idx.shape[-1] if idx is not None else S_seq // cr
    Q = _bf16_bits(Q, "Q")
    pool = _bf16_bits(pool, "pool")
    if tuple(pool.shape) != (B, S_seq // cr, D):
        raise ValueError("pool must be [B,S_seq/cr,D]")
    _want(idx, "idx", torch.int32, (B, S, K))
    if per_branch and full_lse:
        raise ValueError("per_branch and full_lse exclude each other")
    if per_branch:
        wl, sink = None, None
    elif wl is None and not wl_from_kw:
        raise ValueError("window_lse (the full LSE with full_lse=True) is required unless per_branch")
    if full_lse:
        sink = None   # already inside the given LSE
    _want(wl, "window_lse", torch.float32, (B, S, H))
    if sink is not None:
        # The Primus page: a sink must hold one value per head (else ValueError).
        if sink.numel() != H:
            raise ValueError(f"sink needs one logit per head: expected {H} values, found {sink.numel()}")
        _want(sink, "sink", torch.float32)
    _want(doc_start, "doc_start", torch.int32, (B, S))
    _want(err, "err", torch.int32)
    flags = (TARGET_PER_BRANCH if per_branch else 0) | (TARGET_FULL_LSE if full_lse else 0)
    return Q, pool, K, wl, sink, flags


def target_workspace_bytes(B: int, S: int, H: int, D: int, K: int, device=None) -> int:
    """Bytes of the raw-score spill sai_distill_target_ws uses for tokens of
    more than one TMEM group (0 when it needs none), on `device`."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(_lib.sai_distill_target_workspace_bytes(B, S, H, D, K))


def _target_workspace(dev: torch.device, B: int, S: int, H: int, D: int, K: int,
                      given: Optional[torch.Tensor] = None):
    """The spill workspace: the caller's (uint8, on dev, large enough), else a
    new one when the shape needs it."""
    nb = target_workspace_bytes(B, S, H, D, K, dev)
    if nb == 0:
        return None, 0
    if given is not None:
        _want(given, "workspace", torch.uint8)
        if given.numel() < nb:
            raise ValueError(f"workspace holds {given.numel()} bytes, {nb} needed")
        return given, given.numel()
    return torch.empty(nb, dtype=torch.uint8, device=dev), nb


def distill_target(Q: torch.Tensor, pool: torch.Tensor, idx: Optional[torch.Tensor], wl: Optional[torch.Tensor], cr: int,
                   scale: float, sink: Optional[torch.Tensor] = None, doc_start: Optional[torch.Tensor] = None,
                   err: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                   per_branch: bool = False, full_lse: bool = False,
                   workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """p[B,S,K] through sai_distill_target_ws (with its spill workspace, so
    tokens of more than one TMEM group are gathered and multiplied once).
    per_branch=True selects the
    earlier per-branch target; wl and sink are then not used (may be None).
    full_lse=True says wl already holds lse_full, each head's log-normaliser
    over the window, the selected entries and the sink, as a CSA attention
    forward returns it; sink is then not used. idx=None is the dense warm-up
    stage: every compressed block is a slot (K = S/cr, slot k = block k)."""
    B, S, H, D = Q.shape
    Q, pool, K, wl, sink, flags = _target_inputs(Q, pool, idx, wl, cr, sink, doc_start, err, per_branch, full_lse)
    if out is None:
        out = torch.empty((B, S, K), dtype=torch.float32, device=Q.device)
    _want(out, "out", torch.float32, (B, S, K))
    ws, nb = _target_workspace(Q.device, B, S, H, D, K, workspace)
    st = _call(_lib.sai_distill_target_ws, Q.device, _ptr(Q), _ptr(pool), _ptr(idx), _ptr(wl), _ptr(sink),
               _ptr(doc_start), B, S, S, 0, H, D, K, int(cr), float(scale), flags, _ptr(out), _ptr(err), _ptr(ws), nb)
    _check(st, "sai_distill_target_ws")
    return out


def distill_target_range(Q: torch.Tensor, pool: torch.Tensor, idx: Optional[torch.Tensor],
                         wl: Optional[torch.Tensor], cr: int, scale: float, S_seq: int, t_begin: int,
                         sink: Optional[torch.Tensor] = None, doc_start: Optional[torch.Tensor] = None,
                         err: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                         per_branch: bool = False, full_lse: bool = False) -> torch.Tensor:
    """p for sequence positions t_begin .. t_begin+S-1 of sequences of S_seq
    tokens, through sai_distill_target_ws: Q, idx, wl and doc_start are the
    range's rows, pool is the whole sequence's [B,S_seq/cr,D]."""
    B, S, H, D = Q.shape
    Q, pool, K, wl, sink, flags = _target_inputs(Q, pool, idx, wl, cr, sink, doc_start, err, per_branch,
                                                 full_lse, S_seq=S_seq)
    if out is None:
        out = torch.empty((B, S, K), dtype=torch.float32, device=Q.device)
    _want(out, "out", torch.float32, (B, S, K))
    ws, nb = _target_workspace(Q.device, B, S, H, D, K)
    st = _call(_lib.sai_distill_target_ws, Q.device, _ptr(Q), _ptr(pool), _ptr(idx), _ptr(wl), _ptr(sink),
               _ptr(doc_start), B, S, int(S_seq), int(t_begin), H, D, K, int(cr), float(scale), flags,
               _ptr(out), _ptr(err), _ptr(ws), nb)
    _check(st, "sai_distill_target_ws")
    return out


def distill_target_window(Q: torch.Tensor, Kw: torch.Tensor, pool: torch.Tensor, idx: Optional[torch.Tensor],
                          W: int, cr: int, scale: float, sink: Optional[torch.Tensor] = None,
                          doc_start: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None,
                          out: Optional[torch.Tensor] = None, wl_out: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """p[B,S,K] through sai_distill_target_window: the window log-mass is
    formed from Kw [B,S,D] inside the target kernel (W <= 128), so Q is read
    once. wl_out [B,S,H] fp32, if given, receives the window log-mass."""
    B, S, H, D = Q.shape
    Kw = _bf16_bits(Kw, "Kw")
    if tuple(Kw.shape) != (B, S, D):
        raise ValueError("Kw must be [B,S,D]")
    Q, pool, K, _, sink, _ = _target_inputs(Q, pool, idx, None, cr, sink, doc_start, err, False, False,
                                            wl_from_kw=True)
    if out is None:
        out = torch.empty((B, S, K), dtype=torch.float32, device=Q.device)
    _want(out, "out", torch.float32, (B, S, K))
    _want(wl_out, "wl_out", torch.float32, (B, S, H))
    ws, nb = _target_workspace(Q.device, B, S, H, D, K, workspace)
    st = _call(_lib.sai_distill_target_window, Q.device, _ptr(Q), _ptr(Kw), _ptr(pool), _ptr(idx), _ptr(sink),
               _ptr(doc_start), B, S, H, D, K, int(cr), int(W), float(scale), _ptr(out), _ptr(wl_out), _ptr(err),
               _ptr(ws), nb)
    _check(st, "sai_distill_target_window")
    return out


def distill_target_window_range(Q: torch.Tensor, Kw: torch.Tensor, pool: torch.Tensor,
                                idx: Optional[torch.Tensor], W: int, cr: int, scale: float, S_seq: int,
                                t_begin: int, kw_lead: int, sink: Optional[torch.Tensor] = None,
                                doc_start: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None,
                                out: Optional[torch.Tensor] = None, wl_out: Optional[torch.Tensor] = None,
                                workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """p for sequence positions t_begin .. t_begin+S-1 of sequences of S_seq
    tokens through sai_distill_target_window_range: Q, idx and doc_start are
    the range's rows, Kw [B,S+kw_lead,D] the range's keys and its halo, pool
    the whole sequence's [B,S_seq/cr,D]."""
    B, S, H, D = Q.shape
    Kw = _bf16_bits(Kw, "Kw")
    if tuple(Kw.shape) != (B, S + kw_lead, D):
        raise ValueError(f"Kw must be [B,S+kw_lead,D] = {(B, S + kw_lead, D)}, got {tuple(Kw.shape)}")
    Q, pool, K, _, sink, _ = _target_inputs(Q, pool, idx, None, cr, sink, doc_start, err, False, False,
                                            S_seq=S_seq, wl_from_kw=True)
    if out is None:
        out = torch.empty((B, S, K), dtype=torch.float32, device=Q.device)
    _want(out, "out", torch.float32, (B, S, K))
    _want(wl_out, "wl_out", torch.float32, (B, S, H))
    ws, nb = _target_workspace(Q.device, B, S, H, D, K, workspace)
    st = _call(_lib.sai_distill_target_window_range, Q.device, _ptr(Q), _ptr(Kw), _ptr(pool), _ptr(idx),
               _ptr(sink), _ptr(doc_start), B, S, int(S_seq), int(t_begin), int(kw_lead), H, D, K, int(cr), int(W),
               float(scale), _ptr(out), _ptr(wl_out), _ptr(err), _ptr(ws), nb)
    _check(st, "sai_distill_target_window_range")
    return out


def count_valid_rows(valid: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """N, the rows of valid [B,S,K] with a valid slot, as a device int32 [1]
    (sai_count_valid_rows); nothing is read back to the host."""
    B, S, K = valid.shape
    if valid.dtype == torch.bool:
        valid = valid.view(torch.uint8)
    _want(valid, "valid", torch.uint8, (B, S, K))
    if out is None:
        out = torch.empty(1, dtype=torch.int32, device=valid.device)
    _want(out, "out", torch.int32, (1,))
    st = _call(_lib.sai_count_valid_rows, valid.device, _ptr(valid), B, S, K, _ptr(out))
    _check(st, "sai_count_valid_rows")
    return out


def target_kl_workspace_bytes(B: int, S: int, K: int) -> int:
    return int(_lib.sai_distill_target_kl_workspace_bytes(B, S, K))


def distill_target_kl(Q: torch.Tensor, pool: torch.Tensor, idx: Optional[torch.Tensor], wl: Optional[torch.Tensor],
                      cr: int, scale: float, scores: torch.Tensor, valid: torch.Tensor, coeff: float,
                      sink: Optional[torch.Tensor] = None, doc_start: Optional[torch.Tensor] = None,
                      err: Optional[torch.Tensor] = None, p: Optional[torch.Tensor] = None,
                      per_branch: bool = False, workspace: Optional[torch.Tensor] = None,
                      loss: Optional[torch.Tensor] = None, dscores: Optional[torch.Tensor] = None,
                      full_lse: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """(loss, dscores) through sai_distill_target_kl: the target and the KL
    stage in one call. p (optional [B,S,K] fp32 output) receives the target
    when given; without it the target never leaves the GPU's on-chip memory
    where the fused route applies. per_branch and full_lse as for
    distill_target."""
    B, S, H, D = Q.shape
    Q, pool, K, wl, sink, flags = _target_inputs(Q, pool, idx, wl, cr, sink, doc_start, err, per_branch, full_lse)
    _want(scores, "scores", torch.float32, (B, S, K))
    if valid.dtype == torch.bool:
        valid = valid.view(torch.uint8)
    _want(valid, "valid", torch.uint8, (B, S, K))
    _want(p, "p", torch.float32, (B, S, K))
    need = target_kl_workspace_bytes(B, S, K)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    if loss is None:
        loss = torch.empty(1, dtype=torch.float32, device=Q.device)
    if dscores is None:
        dscores = torch.empty((B, S, K), dtype=torch.float32, device=Q.device)
    _want(dscores, "dscores", torch.float32, (B, S, K))
    st = _call(_lib.sai_distill_target_kl, Q.device, _ptr(Q), _ptr(pool), _ptr(idx), _ptr(wl), _ptr(sink),
               _ptr(doc_start), B, S, H, D, K, int(cr), float(scale), flags,
               _ptr(scores), _ptr(valid), float(coeff), _ptr(p), _ptr(loss), _ptr(dscores),
               _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(err))
    _check(st, "sai_distill_target_kl")
    return loss, dscores


def kl_workspace_bytes(B: int, S: int, K: int) -> int:
    return int(_lib.sai_distill_kl_workspace_bytes(B, S, K))


def distill_kl(p: torch.Tensor, scores: torch.Tensor, valid: torch.Tensor, coeff: float,
               want_grad: bool = True, workspace: Optional[torch.Tensor] = None,
               loss: Optional[torch.Tensor] = None, dscores: Optional[torch.Tensor] = None,
               n_rows: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """(loss[1], dscores) through sai_distill_kl_ex. n_rows (device int32 [1],
    optional) is the batch-wide N when the batch is split across GPUs; the
    loss is then this call's share of the batch loss."""
    B, S, K = scores.shape
    _want(n_rows, "n_rows", torch.int32, (1,))
    _want(p, "p", torch.float32, (B, S, K))
    _want(scores, "scores", torch.float32, (B, S, K))
    if valid.dtype == torch.bool:
        valid = valid.view(torch.uint8)
    _want(valid, "valid", torch.uint8, (B, S, K))
    need = kl_workspace_bytes(B, S, K)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=scores.device)
    if loss is None:
        loss = torch.empty(1, dtype=torch.float32, device=scores.device)
    if want_grad and dscores is None:
        dscores = torch.empty((B, S, K), dtype=torch.float32, device=scores.device)
    if not want_grad:
        dscores = None
    st = _call(_lib.sai_distill_kl_ex, scores.device, _ptr(p), _ptr(scores), _ptr(valid), B, S, K, float(coeff),
               _ptr(n_rows), _ptr(loss), _ptr(dscores), _ptr(workspace),
               workspace.numel() * workspace.element_size())
    _check(st, "sai_distill_kl_ex")
    return loss, dscores


def distill_kl_noalloc(p: torch.Tensor, scores: torch.Tensor, valid: torch.Tensor, coeff: float,
                       loss: torch.Tensor, dscores: Optional[torch.Tensor] = None) -> None:
    """sai_distill_kl_noalloc: the KL call for callers that cannot allocate.

    Writes into the caller's ``loss`` (and ``dscores``, if given) without any
    workspace: the library keeps its scratch in a fixed device array. Calls
    running at the same time on one GPU share that array and race."""
    B, S, K = scores.shape
    _want(p, "p", torch.float32, (B, S, K))
    _want(scores, "scores", torch.float32, (B, S, K))
    if valid.dtype == torch.bool:
        valid = valid.view(torch.uint8)
    _want(valid, "valid", torch.uint8, (B, S, K))
    _want(loss, "loss", torch.float32)
    _want(dscores, "dscores", torch.float32, (B, S, K))
    st = _call(_lib.sai_distill_kl_noalloc, scores.device, _ptr(p), _ptr(scores), _ptr(valid), B, S, K,
               float(coeff), _ptr(loss), _ptr(dscores))
    _check(st, "sai_distill_kl_noalloc")


def distill_loss(Q, Kw, pool, idx, scores, valid, *, W: int, cr: int, scale: float, coeff: float,
                 sink=None, doc_start=None, err=None, workspace=None, fused_window: bool = False):
    """The whole path on the current stream: window_lse -> distill_target ->
    distill_kl, or with fused_window=True distill_target_window ->
    distill_kl (the window band inside the target kernel, Q read once; the
    window log-mass is still returned). Returns (loss, dscores, p, wl)."""
    if fused_window:
        B, S, H, _ = Q.shape
        wl = torch.empty((B, S, H), dtype=torch.float32, device=Q.device)
        p = distill_target_window(Q, Kw, pool, idx, W, cr, scale, sink=sink, doc_start=doc_start, err=err,
                                  wl_out=wl)
    else:
        wl = window_lse(Q, Kw, W, scale, doc_start)
        p = distill_target(Q, pool, idx, wl, cr, scale, sink=sink, doc_start=doc_start, err=err)
    loss, ds = distill_kl(p, scores, valid, coeff, workspace=workspace)
    return loss, ds, p, wl


def indexer_topk(index_scores: torch.Tensor, cr: int, K: int, doc_start: Optional[torch.Tensor] = None,
                 idx: Optional[torch.Tensor] = None, sel_scores: Optional[torch.Tensor] = None,
                 valid: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """(idx, sel_scores, valid) through sai_indexer_topk: each token's K
    candidate blocks with the largest indexer scores, in ascending block
    order with a -1 tail, the scores of those blocks and the valid flags."""
    B, S, P = index_scores.shape
    if P * cr != S:
        raise ValueError("index_scores must be [B,S,S/cr]")
    _want(index_scores, "index_scores", torch.float32, (B, S, P))
    _want(doc_start, "doc_start", torch.int32, (B, S))
    dev = index_scores.device
    if idx is None:
        idx = torch.empty((B, S, K), dtype=torch.int32, device=dev)
    if sel_scores is None:
        sel_scores = torch.empty((B, S, K), dtype=torch.float32, device=dev)
    if valid is None:
        valid = torch.empty((B, S, K), dtype=torch.uint8, device=dev)
    _want(idx, "idx", torch.int32, (B, S, K))
    _want(sel_scores, "sel_scores", torch.float32, (B, S, K))
    _want(valid, "valid", torch.uint8, (B, S, K))
    st = _call(_lib.sai_indexer_topk, dev, _ptr(index_scores), _ptr(doc_start), B, S, int(cr), int(K),
               _ptr(idx), _ptr(sel_scores), _ptr(valid))
    _check(st, "sai_indexer_topk")
    return idx, sel_scores, valid
