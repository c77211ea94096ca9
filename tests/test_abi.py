"""The C-ABI library: it builds for sm_100a, loads, exports every symbol that
include/sai.h declares, and rejects bad arguments on the host before touching
the GPU (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sai.h")


@pytest.fixture(scope="module")
def sai():
    import sparse_attention_indexer_window_b200 as m
    return m


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(sai_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("sai_window_lse", "sai_distill_target", "sai_distill_kl", "sai_distill_kl_workspace_bytes",
              "sai_status_string", "sai_version"):
        assert n in names


def test_library_exports_every_declared_symbol(sai):
    lib = ctypes.CDLL(sai.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_status_strings(sai):
    lib = sai.lib()
    for code in range(0, 9):
        s = lib.sai_status_string(code).decode()
        assert s.startswith("SAI_")
    assert b"unknown" in lib.sai_status_string(99)


def test_workspace_size(sai):
    lib = sai.lib()
    assert lib.sai_distill_kl_workspace_bytes(0, 1, 1) == 0
    n = lib.sai_distill_kl_workspace_bytes(1, 4096, 512)
    assert 16 < n < 1 << 20 and n % 16 == 0


FAKE = 1 << 20          # a 16-byte aligned non-NULL address; never dereferenced
FAKE_MIS = FAKE + 4     # misaligned for 16-byte tensors


def test_window_lse_host_errors(sai):
    lib = sai.lib()
    ok = dict(B=1, S=64, H=4, D=32, W=16)
    f = lib.sai_window_lse
    assert f(None, FAKE, None, 1, 64, 4, 32, 16, 0.1, FAKE, None) == 1          # NULL Q
    assert f(FAKE, FAKE, None, 0, 64, 4, 32, 16, 0.1, FAKE, None) == 2          # B = 0
    assert f(FAKE, FAKE, None, 1, 64, 4, 30, 16, 0.1, FAKE, None) == 2          # D % 8
    assert f(FAKE, FAKE, None, 1, 64, 4, 32, 0, 0.1, FAKE, None) == 2           # W = 0
    assert f(FAKE, FAKE, None, 1, 64, 4, 32, 16, float("nan"), FAKE, None) == 2
    assert f(FAKE_MIS, FAKE, None, 1, 64, 4, 32, 16, 0.1, FAKE, None) == 7      # misaligned Q


def test_distill_target_host_errors(sai):
    f = sai.lib().sai_distill_target
    a = [FAKE] * 4
    assert f(None, FAKE, FAKE, FAKE, None, None, 1, 64, 4, 32, 8, 4, 0.1, FAKE, None, None) == 1
    assert f(*a, None, None, 1, 64, 4, 32, 8, 3, 0.1, FAKE, None, None) == 2     # S % cr
    assert f(*a, None, None, 1, 64, 4, 32, 17, 4, 0.1, FAKE, None, None) == 2    # K > S/cr
    assert f(*a, None, None, 1, 64, 4, 32, 0, 4, 0.1, FAKE, None, None) == 2     # K = 0
    assert f(FAKE, FAKE_MIS, FAKE, FAKE, None, None, 1, 64, 4, 32, 8, 4, 0.1, FAKE, None, None) == 7


def test_distill_target_ex_host_errors(sai):
    """The flags variant: unknown flag bits and the two modes at once are
    refused; the joint target (flags 0) and the given-LSE target need
    window_lse. Only paths that return before any launch."""
    f = sai.lib().sai_distill_target_ex
    args = lambda wl, flags: (FAKE, FAKE, FAKE, wl, None, None, 1, 64, 4, 32, 8, 4, 0.1, flags, FAKE, None, None)
    assert f(*args(FAKE, 4)) == 3                     # unknown flag bit
    assert f(*args(FAKE, 0x80000000)) == 3
    assert f(*args(FAKE, 3)) == 3                     # per-branch and full LSE together
    assert f(*args(None, 0)) == 1                     # joint target without window_lse
    assert f(*args(None, 2)) == 1                     # full-LSE target without its LSE
    assert f(*args(FAKE, 1)[:6], 1, 64, 4, 32, 8, 3, 0.1, 1, FAKE, None, None) == 2   # S % cr, per-branch


def test_distill_target_ws_host_errors_and_size(sai):
    """The spill-workspace variant: a misaligned workspace is refused before
    anything else; NULL workspace is allowed (the two-sweep path); the usual
    argument checks apply. No spill is needed at K=512, H=64 (one TMEM group)
    or below H=64; sizes the kernel does not take report 0."""
    lib = sai.lib()
    f = lib.sai_distill_target_ws
    args = lambda ws, nb, S=64, K=8, cr=4: (FAKE, FAKE, FAKE, FAKE, None, None, 1, S, S, 0, 4, 32, K, cr, 0.1, 0,
                                             FAKE, None, ws, nb, None)
    assert f(*args(FAKE_MIS, 1 << 20)) == 7          # SAI_ERR_ALIGN: workspace
    assert f(*args(None, 0, cr=3)) == 2              # S % cr, no workspace
    assert f(*args(FAKE, 1 << 20, K=17)) == 2        # K > S/cr
    sz = lib.sai_distill_target_workspace_bytes
    assert sz(1, 4096, 64, 512, 512) == 0             # one group of four tiles
    assert sz(1, 4096, 32, 512, 2048) == 0            # below H = 64: the two-sweep path only
    assert sz(1, 4096, 64, 500, 2048) == 0            # D % 64 != 0: not the tensor-core kernel
    assert sz(0, 4096, 64, 512, 2048) == 0


def test_distill_target_window_host_errors(sai):
    """The window-fused target: a misaligned workspace is refused first; Kw
    is required; 1 <= W <= 128 (a longer window is unsupported, not a shape
    error); the target's own shape checks; Kw and the window_lse output
    aligned. Only paths that return before any launch."""
    f = sai.lib().sai_distill_target_window
    args = lambda Kw=FAKE, W=16, ws=None, K=8, cr=4, wlo=FAKE: (FAKE, Kw, FAKE, FAKE, None, None, 1, 64, 4, 32, K,
                                                                 cr, W, 0.1, FAKE, wlo, None, ws, 0, None)
    assert f(*args(ws=FAKE_MIS)) == 7                # SAI_ERR_ALIGN: workspace
    assert f(*args(Kw=None)) == 1                    # SAI_ERR_NULL: Kw
    assert f(*args(W=0)) == 2
    assert f(*args(W=129)) == 3                      # the window band is one 128-row tile
    assert f(*args(cr=3)) == 2                       # S % cr
    assert f(*args(K=17)) == 2                       # K > S/cr
    assert f(*args(Kw=FAKE_MIS)) == 7
    assert f(*args(wlo=FAKE + 2)) == 7               # window_lse out not 4-byte aligned


def test_distill_target_window_range_host_errors(sai):
    """The range form of the window-fused target: a halo shorter than the
    window needs, or a range outside the sequence, is a shape error."""
    f = sai.lib().sai_distill_target_window_range
    args = lambda S=32, S_seq=64, t0=32, lead=15, W=16: (FAKE, FAKE, FAKE, FAKE, None, None, 1, S, S_seq, t0, lead,
                                                         4, 32, 8, 4, W, 0.1, FAKE, None, None, None, 0, None)
    assert f(*args(lead=10)) == 2                    # 10 halo keys, W - 1 = 15 needed
    assert f(*args(lead=33)) == 2                    # more halo than positions before the range
    assert f(*args(t0=40)) == 2                      # t_begin + S > S_seq
    assert f(*args(W=129, lead=32)) == 3


def test_distill_target_kl_host_errors(sai):
    """The fused target + KL call refuses missing KL buffers and a short or
    misaligned workspace before launching anything."""
    lib = sai.lib()
    f = lib.sai_distill_target_kl
    need = lib.sai_distill_target_kl_workspace_bytes(1, 64, 8)
    assert need > lib.sai_distill_kl_workspace_bytes(1, 64, 8)
    head = (FAKE, FAKE, FAKE, FAKE, None, None, 1, 64, 4, 32, 8, 4, 0.1, 0)
    assert f(*head, None, FAKE, 0.01, None, FAKE, FAKE, FAKE, need, None, None) == 1    # no scores
    assert f(*head, FAKE, FAKE, 0.01, None, FAKE, None, FAKE, need, None, None) == 1    # no dscores
    assert f(*head, FAKE, FAKE, 0.01, None, FAKE, FAKE, FAKE, need - 1, None, None) == 6
    assert f(*head, FAKE, FAKE, 0.01, None, FAKE, FAKE, FAKE_MIS, need, None, None) == 6
    assert f(*head, FAKE_MIS, FAKE, 0.01, None, FAKE, FAKE, FAKE, need, None, None) == 7
    assert f(*head[:13], 2, FAKE, FAKE, 0.01, None, FAKE, FAKE, FAKE, need, None, None) == 3   # bad flag


def test_distill_kl_host_errors(sai):
    f = sai.lib().sai_distill_kl
    need = sai.lib().sai_distill_kl_workspace_bytes(1, 64, 8)
    assert f(None, FAKE, FAKE, 1, 64, 8, 0.01, FAKE, FAKE, FAKE, need, None) == 1
    assert f(FAKE, FAKE, FAKE, 1, 0, 8, 0.01, FAKE, FAKE, FAKE, need, None) == 2
    assert f(FAKE, FAKE, FAKE, 1, 64, 8, 0.01, FAKE, FAKE, FAKE, need - 1, None) == 6   # short workspace
    assert f(FAKE, FAKE, FAKE, 1, 64, 8, 0.01, FAKE, FAKE, None, need, None) == 6       # no workspace
    assert f(FAKE, FAKE, FAKE, 1, 64, 8, 0.01, FAKE, FAKE, FAKE_MIS, need, None) == 6   # misaligned
    assert f(FAKE_MIS, FAKE, FAKE, 1, 64, 8, 0.01, FAKE, FAKE, FAKE, need, None) == 7


def test_python_sink_length_check(sai):
    """The Primus page's rule: a sink must hold one value per head."""
    import torch
    Q = torch.zeros((1, 8, 4, 8), dtype=torch.bfloat16)
    with pytest.raises((ValueError, TypeError)):
        sai.distill_target(Q, torch.zeros((1, 2, 8), dtype=torch.bfloat16), torch.zeros((1, 8, 2), dtype=torch.int32),
                           torch.zeros((1, 8, 4)), 4, 0.1, sink=torch.zeros(3))


def test_indexer_topk_host_errors(sai):
    """Refusals that return before any launch: missing pointers, S % cr,
    K outside [1, P], too many blocks per row."""
    f = sai.lib().sai_indexer_topk
    assert f(None, None, 1, 64, 4, 8, FAKE, None, None, None) == 1     # no scores
    assert f(FAKE, None, 1, 64, 4, 8, None, None, None, None) == 1     # no idx
    assert f(FAKE, None, 1, 66, 4, 8, FAKE, None, None, None) == 2     # S % cr
    assert f(FAKE, None, 1, 64, 4, 17, FAKE, None, None, None) == 2    # K > P
    assert f(FAKE, None, 1, 64, 4, 0, FAKE, None, None, None) == 2     # K < 1
    assert f(FAKE, None, 1, 40000, 1, 8, FAKE, None, None, None) == 3  # P > 32768
