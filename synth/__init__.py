"""Seeded synthetic workloads for the CSA indexer distillation loss.

This module only draws inputs. It holds none of the loss arithmetic: no
logits, no softmax, no log-sum-exp. Both the CUDA path and the CPU oracle read
the same arrays from here, so they see identical bytes.

The five workloads follow the shapes and value distributions named for the
DeepSeek-V4 CSA layer on the source pages ("perf(deepseek-v4): fuse and enable
the indexer distillation loss", Summary and "Why the target was wrong"; the
MaxText "Add Indexer Loss [Deepseek v4]" page for the causal block rule):

  tiny    B=1  S=64    H=4  D=32  cr=4 K=8    W=16
  small   B=2  S=512   H=16 D=128 cr=4 K=64   W=64   (half the heads local)
  flash   B=1  S=4096  H=64 D=512 cr=4 K=512  W=128  (V4-Flash CSA width)
  packed  B=4  S=4096  H=64 D=512 cr=4 K=512  W=128  (2 documents per row)
  long    B=1  S=16384 H=64 D=512 cr=4 K=2048 W=128

Arrays are numpy. bf16 tensors are carried as uint16 bit patterns produced by
round-to-nearest-even from float32 draws.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

__all__ = ["Workload", "CONFIGS", "make", "bf16_bits", "bf16_to_f32", "config_dims"]


@dataclasses.dataclass(frozen=True)
class Spec:
    name: str
    B: int
    S: int
    H: int
    D: int
    cr: int
    K: int
    W: int
    seed: int
    idx_mode: str          # "random" (distinct, random order) or "topk_sorted"
    local_heads: bool = False
    docs: int = 1
    coeff: float = 1e-2


CONFIGS: Dict[str, Spec] = {
    "tiny": Spec("tiny", 1, 64, 4, 32, 4, 8, 16, 1001, "random"),
    "small": Spec("small", 2, 512, 16, 128, 4, 64, 64, 1002, "random", local_heads=True),
    "flash": Spec("flash", 1, 4096, 64, 512, 4, 512, 128, 1003, "topk_sorted"),
    "packed": Spec("packed", 4, 4096, 64, 512, 4, 512, 128, 1004, "topk_sorted", docs=2),
    "long": Spec("long", 1, 16384, 64, 512, 4, 2048, 128, 1005, "random"),
}


@dataclasses.dataclass
class Workload:
    """One seeded problem instance. All arrays are C-contiguous numpy arrays."""

    name: str
    B: int
    S: int
    H: int
    D: int
    cr: int
    K: int
    W: int
    scale: float
    coeff: float
    Q: np.ndarray            # [B,S,H,D] uint16 (bf16 bits)
    Kw: np.ndarray           # [B,S,D]   uint16 (bf16 bits), window keys
    pool: np.ndarray         # [B,P,D]   uint16 (bf16 bits), compressed entries
    idx: np.ndarray          # [B,S,K]   int32, -1 padded
    sink: Optional[np.ndarray]       # [H] float32 or None
    doc_start: Optional[np.ndarray]  # [B,S] int32 or None
    scores: np.ndarray       # [B,S,K] float32, indexer logits
    valid: np.ndarray        # [B,S,K] uint8

    @property
    def P(self) -> int:
        return self.S // self.cr

    def nbytes(self) -> int:
        tot = 0
        for a in (self.Q, self.Kw, self.pool, self.idx, self.sink, self.doc_start, self.scores, self.valid):
            if a is not None:
                tot += a.nbytes
        return tot


def config_dims(name: str) -> Spec:
    return CONFIGS[name]


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern, round to nearest even (finite inputs)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # finite inputs: the sum stays below 2^32
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit pattern -> float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    flat = out.reshape(-1)
    n = flat.size
    step = 1 << 24
    for i in range(0, n, step):
        m = min(step, n - i)
        flat[i:i + m] = bf16_bits(rng.standard_normal(m, dtype=np.float32))
    return out


def _doc_starts(rng: np.random.Generator, B: int, S: int, docs: int) -> Optional[np.ndarray]:
    if docs <= 1:
        return None
    assert docs == 2
    ds = np.zeros((B, S), dtype=np.int32)
    for b in range(B):
        s0 = int(rng.integers(1, S))  # split position, uniform in [1, S-1]
        ds[b, s0:] = s0
    return ds


def _block_ok(S: int, cr: int, doc_start: Optional[np.ndarray], b: int):
    """Boolean [S, P] table of blocks a token may select: the block lies wholly
    before or at the token (causal) and inside the token's document."""
    P = S // cr
    t = np.arange(S)[:, None]
    j = np.arange(P)[None, :]
    ok = (j + 1) * cr - 1 <= t
    if doc_start is not None:
        ok &= j * cr >= doc_start[b][:, None]
    return ok


def _idx_random(rng, S, cr, K, doc_start, b) -> np.ndarray:
    """Distinct allowed blocks chosen uniformly, in random slot order, -1 tail."""
    P = S // cr
    out = np.empty((S, K), dtype=np.int32)
    rows = 2048
    for t0 in range(0, S, rows):
        t1 = min(S, t0 + rows)
        ok = _block_ok(S, cr, doc_start, b)[t0:t1]
        keys = rng.random((t1 - t0, P), dtype=np.float32)
        keys[~ok] = 2.0
        kk = min(K, P)
        part = np.argpartition(keys, kk - 1, axis=1)[:, :kk] if kk < P else np.tile(np.arange(P), (t1 - t0, 1))
        pk = np.take_along_axis(keys, part, axis=1)
        order = np.argsort(pk, axis=1, kind="stable")
        sel = np.take_along_axis(part, order, axis=1).astype(np.int32)
        selk = np.take_along_axis(pk, order, axis=1)
        sel[selk >= 2.0] = -1
        blk = np.full((t1 - t0, K), -1, dtype=np.int32)
        blk[:, :kk] = sel
        out[t0:t1] = blk
    return out


def _idx_topk_sorted(rng, S, cr, K, doc_start, b) -> np.ndarray:
    """Top-K of a random score over allowed blocks, ascending, -1 tail."""
    P = S // cr
    out = np.empty((S, K), dtype=np.int32)
    rows = 2048
    for t0 in range(0, S, rows):
        t1 = min(S, t0 + rows)
        ok = _block_ok(S, cr, doc_start, b)[t0:t1]
        sc = rng.standard_normal((t1 - t0, P), dtype=np.float32)
        sc[~ok] = -np.inf
        kk = min(K, P)
        part = np.argpartition(-sc, kk - 1, axis=1)[:, :kk] if kk < P else np.tile(np.arange(P), (t1 - t0, 1))
        ps = np.take_along_axis(sc, part, axis=1)
        big = np.int64(1) << 40
        key = np.where(np.isfinite(ps), part.astype(np.int64), big)
        key.sort(axis=1)
        sel = np.where(key >= big, -1, key).astype(np.int32)
        blk = np.full((t1 - t0, K), -1, dtype=np.int32)
        blk[:, :kk] = sel
        out[t0:t1] = blk
    return out


def make(name: str, *, seed: Optional[int] = None, with_sink: bool = True,
         S: Optional[int] = None, B: Optional[int] = None, K: Optional[int] = None,
         W: Optional[int] = None, H: Optional[int] = None, D: Optional[int] = None) -> Workload:
    """Draw the named workload. ``S``/``B``/``K``/``W``/``H``/``D`` override the
    sizes (same recipe and value distributions; H=128 is the V4-Pro head
    count)."""
    sp = CONFIGS[name]
    B_ = B if B is not None else sp.B
    S_ = S if S is not None else sp.S
    H = sp.H if H is None else H
    D = sp.D if D is None else D
    cr = sp.cr
    K = sp.K if K is None else K
    W = sp.W if W is None else W
    assert K <= S_ // cr
    assert S_ % cr == 0
    P = S_ // cr
    rng = np.random.Generator(np.random.PCG64(sp.seed if seed is None else seed))

    Q = _normal_bf16(rng, (B_, S_, H, D))
    Kw = _normal_bf16(rng, (B_, S_, D))
    pool = _normal_bf16(rng, (B_, P, D))
    sink = rng.standard_normal(H, dtype=np.float32) if with_sink else None
    doc_start = _doc_starts(rng, B_, S_, sp.docs)

    if sp.local_heads:
        # Heads h < H/2 attend locally: q = k_t + 0.1 * noise and a +8 sink.
        hl = H // 2
        kf = bf16_to_f32(Kw)                                  # [B,S,D]
        noise = rng.standard_normal((B_, S_, hl, D), dtype=np.float32)
        Q[:, :, :hl, :] = bf16_bits(kf[:, :, None, :] + np.float32(0.1) * noise)
        if sink is not None:
            sink[:hl] = 8.0

    idx = np.empty((B_, S_, K), dtype=np.int32)
    for b in range(B_):
        if sp.idx_mode == "random":
            idx[b] = _idx_random(rng, S_, cr, K, doc_start, b)
        else:
            idx[b] = _idx_topk_sorted(rng, S_, cr, K, doc_start, b)

    scores = (rng.standard_normal((B_, S_, K), dtype=np.float32) * np.float32(math.sqrt(2.0))).astype(np.float32)
    valid = (idx >= 0).astype(np.uint8)

    return Workload(name=name, B=B_, S=S_, H=H, D=D, cr=cr, K=K, W=W,
                    scale=1.0 / math.sqrt(D), coeff=sp.coeff,
                    Q=Q, Kw=Kw, pool=pool, idx=idx, sink=sink, doc_start=doc_start,
                    scores=scores, valid=valid)


def index_scores(B: int, S: int, cr: int, seed: int) -> np.ndarray:
    """[B, S, S/cr] fp32 indexer scores over every compressed block, N(0,1)
    (the flash workload's random causal score; which blocks a token may
    select is left to the selection)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal((B, S, S // cr), dtype=np.float32)


def sample_tokens(B: int, S: int, n: int, seed: int = 7) -> np.ndarray:
    """A sorted, seeded sample of flat token ids b*S+t that always includes the
    first and last token of every row (the lightest and heaviest)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    must = []
    for b in range(B):
        must += [b * S, b * S + S - 1]
    extra = rng.choice(B * S, size=max(0, min(n, B * S) - len(must)), replace=False)
    return np.unique(np.concatenate([np.array(must, dtype=np.int64), extra.astype(np.int64)]))
