"""sai_distill_kl_noalloc: the KL call for callers that cannot allocate device
memory (no workspace argument; scratch lives in a fixed array inside the
library). Checked through the C ABI against sai_distill_kl on two calls in a
row, so a stale scratch word left by the first call would show up in the
second, then a larger grid followed by a smaller one on the shared array,
the forward-only form through the Python wrapper, and the loss against the
fp64 oracle. This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    import sparse_attention_indexer_window_b200 as m
    return m.lib()


def _case(seed, B, S, K):
    rng = np.random.default_rng(seed)
    p = rng.random((B, S, K)).astype(np.float32)
    valid = (rng.random((B, S, K)) < 0.8).astype(np.uint8)
    valid[0, :3] = 0
    p *= valid
    s = p.sum(-1, keepdims=True)
    p = np.where(s > 0, p / np.where(s > 0, s, 1), 0).astype(np.float32)
    scores = (rng.standard_normal((B, S, K)) * np.sqrt(2)).astype(np.float32)
    return [torch.from_numpy(x).cuda() for x in (p, scores, valid)]


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("shape", [(2, 300, 64), (1, 4096, 512)])
def test_noalloc_matches_workspace_call_twice(lib, shape):
    B, S, K = shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.sai_distill_kl_noalloc_max_scratch_bytes() >= lib.sai_distill_kl_workspace_bytes(B, S, K)
    for call, seed in enumerate((11, 12)):
        p, scores, valid = _case(seed, B, S, K)
        ws = torch.empty(lib.sai_distill_kl_workspace_bytes(B, S, K), dtype=torch.uint8, device="cuda")
        loss_ref = torch.full((1,), float("nan"), device="cuda")
        ds_ref = torch.full((B, S, K), float("nan"), device="cuda")
        st = lib.sai_distill_kl(_ptr(p), _ptr(scores), _ptr(valid), B, S, K, ctypes.c_float(0.01), _ptr(loss_ref),
                                _ptr(ds_ref), _ptr(ws), ws.numel(), stream)
        assert st == 0
        loss = torch.full((1,), float("nan"), device="cuda")
        ds = torch.full((B, S, K), float("nan"), device="cuda")
        st = lib.sai_distill_kl_noalloc(_ptr(p), _ptr(scores), _ptr(valid), B, S, K, ctypes.c_float(0.01),
                                        _ptr(loss), _ptr(ds), stream)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        lr, lg = float(loss_ref.item()), float(loss.item())
        assert abs(lg - lr) <= 1e-4 * abs(lr), (call, lg, lr)
        assert torch.max(torch.abs(ds - ds_ref)).item() <= 1e-6
        assert bool(torch.isfinite(ds).all())


def test_noalloc_large_grid_then_small_and_forward_only():
    """The flash shape (the most KL blocks) fills the shared array first; a
    small shape after it must not read the large call's leftovers. The second
    call goes through the Python wrapper without dscores (forward only)."""
    import oracle
    import sparse_attention_indexer_window_b200 as sai
    for B, S, K, seed in ((1, 4096, 512, 21), (2, 75, 96, 22)):
        p, scores, valid = _case(seed, B, S, K)
        loss = torch.full((1,), float("nan"), device="cuda")
        ds = torch.full((B, S, K), float("nan"), device="cuda") if S == 4096 else None
        sai.distill_kl_noalloc(p, scores, valid, 0.01, loss, ds)
        torch.cuda.synchronize()
        ol, ods, _ = oracle.distill_kl(p.cpu().numpy().astype(np.float64), scores.cpu().numpy(),
                                       valid.cpu().numpy(), 0.01)
        assert abs(float(loss.item()) - ol) <= 1e-4 * abs(ol)
        if ds is not None:
            assert np.abs(ds.cpu().numpy().reshape(-1, K) - ods).max() <= 1e-6
