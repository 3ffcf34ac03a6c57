"""Seeded synthetic decode workloads (shared by the tests, the bench and the oracle checks).

This module only draws random numbers and lays them out.  It holds none of the
method's arithmetic (no rotation, no bucketing, no distances, no attention), so
it may serve both the CUDA path and the CPU oracle.

Workload shapes follow the long-context decode settings that the ADAMAS sparse
attention article (lnwmold.com/news/826806) measures on: Llama-2-7B-class heads
(§2.2, §5.2: 32 heads of width 128, 32K-128K contexts, budgets 64..1024), plus a
GQA batch shaped like Llama-3-8B and a 1M-token layer shaped like the attention
layers of a Llama-3.2-3B hybrid.  No model weights or dataset items are used:
K, V and q are N(0, 1) with a few channels scaled x20 (activation outliers, §2.1)
and planted "needle" keys K_i = 2 q* + 0.1 N(0, 1) that a good selector must keep.

Recipe (all values rounded to bf16 with round-to-nearest-even):
  * every (layer, b, kv head) block draws from its own PCG64 stream keyed by
    SeedSequence([seed, layer, b, kvh, tag]) so any head can be regenerated alone;
  * 4 outlier channels per (layer, kv head), chosen without replacement, scaled x20
    in K and q (workload 1) or in K and V (workloads 2-5);
  * per query head a needle query q*_h ~ N(0, 1) (with the K outlier channels x20
    in workload 1); needle j of kv head g targets query head g*G + (j mod G);
  * needle positions are stratified: floor((j + u_j) / n * len) for u_j ~ U[0, 1);
  * decode step s uses q* when s % 10 == 0, else a fresh q ~ N(0, 1);
  * per-sequence lengths are Nmax, or U[lo, hi] inclusive for workload 4.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence, Tuple

import numpy as np

HEAD_DIM = 128

# stream tags for SeedSequence keys
_TAG_K, _TAG_V, _TAG_Q, _TAG_NEEDLE, _TAG_LENS, _TAG_OUTLIER, _TAG_QSTAR, _TAG_POS = range(8)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode workload (shapes, budgets, value recipe)."""

    name: str
    B: int
    Hq: int
    Hkv: int
    Nmax: int
    budgets: Tuple[int, ...]
    seed: int
    n_needles: int                   # per kv head
    outliers_in_q: bool              # True: outliers in K and q; False: in K and V
    len_range: Optional[Tuple[int, int]] = None   # None: every sequence is Nmax long
    d: int = HEAD_DIM
    n_outliers: int = 4
    outlier_scale: float = 20.0
    needle_gain: float = 2.0
    needle_noise: float = 0.1

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def scaled(self, **kw) -> "Workload":
        """Same recipe at other sizes (parity cases the oracle finishes quickly)."""
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    1: Workload("single_head_4k", B=1, Hq=1, Hkv=1, Nmax=4096, budgets=(64,), seed=1001,
                n_needles=3, outliers_in_q=True),
    2: Workload("mha32_32k", B=1, Hq=32, Hkv=32, Nmax=32768, budgets=(128, 256, 1024), seed=1002,
                n_needles=8, outliers_in_q=False),
    3: Workload("mha32_128k", B=1, Hq=32, Hkv=32, Nmax=131072, budgets=(64, 128, 1024), seed=1003,
                n_needles=8, outliers_in_q=False),
    4: Workload("gqa8x4_b8_32k", B=8, Hq=32, Hkv=8, Nmax=32768, budgets=(256,), seed=1004,
                n_needles=4, outliers_in_q=False, len_range=(16384, 32768)),
    5: Workload("gqa8x3_1m", B=1, Hq=24, Hkv=8, Nmax=1048576, budgets=(1024,), seed=1005,
                n_needles=16, outliers_in_q=False),
}


# ---------------------------------------------------------------- bf16 helpers
def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32 (exact)."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------- streams
def _rng(w: Workload, layer: int, b: int, h: int, tag: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, layer, b, h, tag])))


def seq_lens(w: Workload) -> np.ndarray:
    """Per-sequence context lengths, int32[B]."""
    if w.len_range is None:
        return np.full(w.B, w.Nmax, dtype=np.int32)
    lo, hi = w.len_range
    r = _rng(w, 0, 0, 0, _TAG_LENS)
    return r.integers(lo, hi + 1, size=w.B).astype(np.int32)


def outlier_channels(w: Workload, kvh: int, layer: int = 0) -> np.ndarray:
    r = _rng(w, layer, 0, kvh, _TAG_OUTLIER)
    return np.sort(r.choice(w.d, size=w.n_outliers, replace=False))


def needle_query_f32(w: Workload, b: int, hq: int, layer: int = 0) -> np.ndarray:
    """q*_h before bf16 rounding, float32[d]."""
    r = _rng(w, layer, b, hq, _TAG_QSTAR)
    q = r.standard_normal(w.d, dtype=np.float32)
    if w.outliers_in_q:
        ch = outlier_channels(w, hq // w.G, layer)
        q[ch] *= np.float32(w.outlier_scale)
    return q


def needle_positions(w: Workload, b: int, kvh: int, length: int, layer: int = 0) -> np.ndarray:
    """Stratified needle positions in [0, length), int64[n] (distinct when length >= n)."""
    n = w.n_needles
    if n == 0 or length == 0:
        return np.zeros(0, dtype=np.int64)
    u = _rng(w, layer, b, kvh, _TAG_POS).random(n)
    pos = np.floor((np.arange(n) + u) / n * length).astype(np.int64)
    return np.minimum(pos, length - 1)


def needle_targets(w: Workload, kvh: int) -> np.ndarray:
    """Query head targeted by each needle of kv head kvh."""
    return kvh * w.G + (np.arange(w.n_needles) % w.G)


def head_kv(w: Workload, b: int, kvh: int, layer: int = 0,
            rows: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """K and V of one (b, kv head) as bf16 bits, uint16[rows, d] each (rows defaults to Nmax).

    Rows at or beyond the sequence length hold the same distribution (never read
    by a correct implementation)."""
    n = w.Nmax if rows is None else rows
    d = w.d
    ch = outlier_channels(w, kvh, layer)
    K = _rng(w, layer, b, kvh, _TAG_K).standard_normal((n, d), dtype=np.float32)
    V = _rng(w, layer, b, kvh, _TAG_V).standard_normal((n, d), dtype=np.float32)
    K[:, ch] *= np.float32(w.outlier_scale)
    if not w.outliers_in_q:
        V[:, ch] *= np.float32(w.outlier_scale)
    length = int(seq_lens(w)[b])
    pos = needle_positions(w, b, kvh, min(length, n), layer)
    if pos.size:
        noise = _rng(w, layer, b, kvh, _TAG_NEEDLE).standard_normal((pos.size, d), dtype=np.float32)
        for j, (p, hq) in enumerate(zip(pos, needle_targets(w, kvh))):
            qs = bf16_to_f32(bf16_round(needle_query_f32(w, b, int(hq), layer)))
            K[p] = np.float32(w.needle_gain) * qs + np.float32(w.needle_noise) * noise[j]
    return bf16_round(K), bf16_round(V)


def query(w: Workload, step: int = 0, layer: int = 0) -> np.ndarray:
    """Decode query for one step, bf16 bits uint16[B, Hq, d]."""
    q = np.empty((w.B, w.Hq, w.d), dtype=np.float32)
    for b in range(w.B):
        for hq in range(w.Hq):
            if step % 10 == 0:
                q[b, hq] = needle_query_f32(w, b, hq, layer)
            else:
                q[b, hq] = _rng(w, layer * 1_000_003 + step, b, hq, _TAG_Q).standard_normal(
                    w.d, dtype=np.float32)
    return bf16_round(q)


def make_inputs(w: Workload, layer: int = 0, step: int = 0,
                kv_heads: Optional[Sequence[Tuple[int, int]]] = None):
    """Full arrays for a workload: dict(K, V [B,Hkv,Nmax,d] u16, q [B,Hq,d] u16, lens [B] i32).

    kv_heads, if given, restricts generation to those (b, kvh) blocks; the others
    are left zero (used to sample large workloads)."""
    K = np.zeros((w.B, w.Hkv, w.Nmax, w.d), dtype=np.uint16)
    V = np.zeros_like(K)
    blocks = kv_heads if kv_heads is not None else [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    for b, h in blocks:
        K[b, h], V[b, h] = head_kv(w, b, h, layer)
    return dict(K=K, V=V, q=query(w, step, layer), lens=seq_lens(w))
