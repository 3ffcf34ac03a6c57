"""Byte accounting for the KV cache and for one ADAMAS decode step (host arithmetic only).

KV-cache size follows the formula of the compressed-sparse-attention comparison
article (cloud.baidu.com/article/9429012, part 3.1 "architecture and memory"):
    bytes = L_ctx * N_layers * N_kvheads * (d_K + d_V) * bytes_per_value.

Algorithmic bytes of one decode step (one attention layer, whole batch) are what
the method must move at least once: the packed key codes it scores (d/4 bytes per
cached token and kv head, ADAMAS article §3.1 and §2.3), the K and V rows of the
kept tokens (ADAMAS article §5.2 token budget) and the query.  Output writes are
reported separately and are not part of the roofline numerator.
"""
from __future__ import annotations

from typing import Iterable, Optional


def kv_cache_bytes(l_ctx: int, n_layers: int, n_kv_heads: int, d_k: int, d_v: int,
                   bytes_per_value: int = 2) -> int:
    return l_ctx * n_layers * n_kv_heads * (d_k + d_v) * bytes_per_value


def code_bytes_per_token(d: int = 128) -> int:
    """Packed 2-bit codes: four per byte."""
    return d // 4


def encode_bytes_per_vector(d: int = 128, in_bytes: int = 2) -> int:
    """Bytes the key encoder moves per (token, kv head): the bf16 key in, the codes out."""
    return d * in_bytes + code_bytes_per_token(d)


def decode_step_bytes(lens: Iterable[int], Hq: int, Hkv: int, budget: int, d: int = 128,
                      unique_rows: Optional[int] = None) -> dict:
    """Algorithmic bytes of one decode step.

    lens: per-sequence context lengths.  Rows are counted per query head
    (min(budget, len) each) unless unique_rows gives the number of distinct
    (b, kv head, token) rows actually gathered."""
    lens = [int(x) for x in lens]
    B = len(lens)
    codes = sum(Hkv * n * code_bytes_per_token(d) for n in lens)
    rows = sum(Hq * min(budget, n) for n in lens) if unique_rows is None else unique_rows
    kv_rows = rows * 2 * d * 2
    q = B * Hq * d * 2
    out = B * Hq * d * 4 + B * Hq * budget * 4
    return dict(codes=codes, kv_rows=kv_rows, q=q, total=codes + kv_rows + q, writes=out)
