"""NumPy front end of the CPU oracle (adamas_oracle.c) -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package smoke check and the bench's CPU-baseline leg may
import this module.  The product path never does.

The C source follows the ADAMAS long-context sparse attention article
(lnwmold.com/news/826806): §2.1 Hadamard rotation, §2.2 dynamic 2-bit bucketing,
§3.1 packing of the code cache, §2.3 Manhattan-distance scoring, §5.2 token budget,
followed by exact attention over the kept rows.  Parity unpinned: the page's own
activation statistics and accuracy tables (they need model weights and datasets).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "adamas_oracle.c")
LIBRARY = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile adamas_oracle.c into liboracle.so next to it (gcc, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(LIBRARY) or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE):
        tmp = LIBRARY + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, SOURCE, "-lm"], check=True)
        os.replace(tmp, LIBRARY)
    return LIBRARY


def lib():
    global _lib
    with _lock:
        if _lib is None:
            l = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64, I32 = ctypes.c_int64, ctypes.c_int
            l.oracle_rotate.argtypes = [P, I64, I32, P]
            l.oracle_bucket_pack.argtypes = [P, I64, I32, P]
            l.oracle_encode.argtypes = [P, I64, I32, P]
            l.oracle_distance.argtypes = [P, P, I64, I32, P]
            l.oracle_select.argtypes = [P, I64, I64, P]
            l.oracle_attend.argtypes = [P, P, P, P, I64, I32, P]
            l.oracle_decode_step.argtypes = [P, P, P, P, P, I32, I32, I32, I64, I32, I32, P, P, P, I32]
            for f in (l.oracle_rotate, l.oracle_bucket_pack, l.oracle_encode, l.oracle_distance,
                      l.oracle_select, l.oracle_attend, l.oracle_decode_step):
                f.restype = ctypes.c_int
            _lib = l
        return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc: int, name: str):
    if rc != 0:
        raise ValueError(f"oracle: {name} rejected its arguments")


def rotate(x_bf16: np.ndarray) -> np.ndarray:
    """fp32 Hadamard-rotated values of bf16 vectors [..., 128] -> float32 [..., 128]."""
    x = _c(x_bf16, np.uint16)
    y = np.empty(x.shape, dtype=np.float32)
    _check(lib().oracle_rotate(_p(x), x.size // 128, x.shape[-1], _p(y)), "rotate")
    return y


def bucket_pack(y: np.ndarray) -> np.ndarray:
    """Packed codes of already-rotated fp32 vectors [..., 128] -> uint8 [..., 32]."""
    y = _c(y, np.float32)
    out = np.empty(y.shape[:-1] + (32,), dtype=np.uint8)
    _check(lib().oracle_bucket_pack(_p(y), y.size // 128, y.shape[-1], _p(out)), "bucket_pack")
    return out


def encode(x_bf16: np.ndarray) -> np.ndarray:
    """Packed 2-bit codes of bf16 vectors [..., 128] -> uint8 [..., 32]."""
    x = _c(x_bf16, np.uint16)
    out = np.empty(x.shape[:-1] + (32,), dtype=np.uint8)
    _check(lib().oracle_encode(_p(x), x.size // 128, x.shape[-1], _p(out)), "encode")
    return out


def distance(qcode: np.ndarray, kcodes: np.ndarray) -> np.ndarray:
    """L1 distances of one packed query code [32] to packed keys [n, 32] -> int32 [n]."""
    q = _c(qcode, np.uint8).reshape(32)
    k = _c(kcodes, np.uint8).reshape(-1, 32)
    D = np.empty(k.shape[0], dtype=np.int32)
    _check(lib().oracle_distance(_p(q), _p(k), k.shape[0], 128, _p(D)), "distance")
    return D


def select(D: np.ndarray, k: int) -> np.ndarray:
    """Token indices of the k smallest (D, index), -1 past len(D) -> int32 [k]."""
    D = _c(D, np.int32)
    idx = np.empty(max(k, 1), dtype=np.int32)
    _check(lib().oracle_select(_p(D), D.size, k, _p(idx)), "select")
    return idx[:k]


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """float64 attention of one bf16 query [128] over bf16 rows K/V [n, 128] picked by idx."""
    q = _c(q, np.uint16).reshape(128)
    K = _c(K, np.uint16).reshape(-1, 128)
    V = _c(V, np.uint16).reshape(-1, 128)
    idx = _c(idx, np.int32).reshape(-1)
    if idx.size and int(idx.max(initial=-1)) >= K.shape[0]:
        raise ValueError("oracle: idx out of range")
    out = np.empty(128, dtype=np.float64)
    _check(lib().oracle_attend(_p(q), _p(K), _p(V), _p(idx), idx.size, 128, _p(out)), "attend")
    return out


def decode_step(q, K, V, codes, seq_lens, budget: int, nthreads: int = 1, want_dist: bool = False):
    """Whole decode step.  q [B,Hq,128], K/V [B,Hkv,Nmax,128] bf16 bits, codes
    [B,Hkv,Nmax,32] (from encode), seq_lens int32 [B].
    Returns (out float64 [B,Hq,128], idx int32 [B,Hq,budget], dist int32 [B,Hq,Nmax] or None)."""
    q = _c(q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    codes = _c(codes, np.uint8)
    lens = _c(seq_lens, np.int32)
    B, Hq, d = q.shape
    _, Hkv, Nmax, _ = K.shape
    if V.shape != K.shape or codes.shape != (B, Hkv, Nmax, 32) or lens.shape != (B,):
        raise ValueError("oracle: inconsistent shapes")
    out = np.empty((B, Hq, d), dtype=np.float64)
    idx = np.empty((B, Hq, max(budget, 1)), dtype=np.int32)
    dist = np.empty((B, Hq, Nmax), dtype=np.int32) if want_dist else None
    rc = lib().oracle_decode_step(_p(q), _p(K), _p(V), _p(codes), _p(lens), B, Hq, Hkv, Nmax, d,
                                  budget, _p(out), _p(idx), _p(dist) if want_dist else None,
                                  nthreads)
    _check(rc, "decode_step")
    return out, idx[:, :, :budget], dist


def decode_step_group_shared(q, K, V, codes, seq_lens, budget: int):
    """Group-shared selection for grouped-query attention (a reading for grouped
    heads of the ADAMAS article's §2.3 scoring and §5.2 token budget, which the
    article states per head only): for every (b, kv head) the L1 distances of
    its G query heads are summed per token, the k_eff = min(budget, len) tokens
    of smallest (summed distance, index) are kept once, and each query head of
    the group runs exact attention over those rows.

    q [B,Hq,128], K/V [B,Hkv,Nmax,128] bf16 bits, codes [B,Hkv,Nmax,32] (from
    encode), seq_lens int32 [B].  Returns (out float64 [B,Hq,128], idx int32
    [B,Hkv,budget] with -1 past k_eff)."""
    q = _c(q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    codes = _c(codes, np.uint8)
    lens = _c(seq_lens, np.int32)
    B, Hq, d = q.shape
    _, Hkv, Nmax, _ = K.shape
    if Hq % Hkv or V.shape != K.shape or codes.shape != (B, Hkv, Nmax, 32) or lens.shape != (B,):
        raise ValueError("oracle: inconsistent shapes")
    G = Hq // Hkv
    qcodes = encode(q.reshape(-1, d)).reshape(B, Hq, 32)
    out = np.zeros((B, Hq, d), dtype=np.float64)
    idx = np.full((B, Hkv, budget), -1, dtype=np.int32)
    for b in range(B):
        n = int(lens[b])
        if n < 0 or n > Nmax:
            raise ValueError("oracle: sequence length outside [0, Nmax]")
        keff = min(budget, n)
        for h in range(Hkv):
            if keff == 0:
                continue
            D = np.zeros(n, dtype=np.int64)
            for g in range(G):
                D += distance(qcodes[b, h * G + g], codes[b, h, :n])
            kept = select(D.astype(np.int32), keff)
            idx[b, h, :keff] = kept
            for g in range(G):
                out[b, h * G + g] = attend(q[b, h * G + g], K[b, h, :n], V[b, h, :n], kept)
    return out, idx


def decode_step_forced(q, K, V, codes, seq_lens, budget: int, n_sink: int, n_recent: int):
    """Per-head decode step with forced rows: the first n_sink tokens (attention
    sinks) and the last n_recent tokens of each sequence (the recent window)
    rank ahead of every scored token, as if their distance were -1; the rest is
    the per-head step (k_eff = min(budget, len) tokens of smallest (D, index)).
    Forced rows therefore come first in idx, in index order, and when there are
    more of them than k_eff the lowest indices win.  (A reading of the ADAMAS
    article's §3.2 / §6 tuning advice -- some tokens keep full attention -- for
    the sink and window the other pages describe; the article gives no rule.)

    Shapes as decode_step.  Returns (out float64 [B,Hq,128], idx int32 [B,Hq,budget])."""
    q = _c(q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    codes = _c(codes, np.uint8)
    lens = _c(seq_lens, np.int32)
    B, Hq, d = q.shape
    _, Hkv, Nmax, _ = K.shape
    if Hq % Hkv or V.shape != K.shape or codes.shape != (B, Hkv, Nmax, 32) or lens.shape != (B,):
        raise ValueError("oracle: inconsistent shapes")
    if n_sink < 0 or n_recent < 0:
        raise ValueError("oracle: negative forced-row counts")
    G = Hq // Hkv
    qcodes = encode(q.reshape(-1, d)).reshape(B, Hq, 32)
    out = np.zeros((B, Hq, d), dtype=np.float64)
    idx = np.full((B, Hq, budget), -1, dtype=np.int32)
    for b in range(B):
        n = int(lens[b])
        if n < 0 or n > Nmax:
            raise ValueError("oracle: sequence length outside [0, Nmax]")
        keff = min(budget, n)
        if keff == 0:
            continue
        t = np.arange(n)
        forced = (t < n_sink) | (t >= n - n_recent)
        for hq in range(Hq):
            h = hq // G
            D = distance(qcodes[b, hq], codes[b, h, :n])
            D[forced] = -1
            kept = select(D, keff)
            idx[b, hq, :keff] = kept
            out[b, hq] = attend(q[b, hq], K[b, h, :n], V[b, h, :n], kept)
    return out, idx


def decode_step_paged(q, K_pages, V_pages, code_pages, block_table, seq_lens, budget: int):
    """Per-head decode step over a paged cache: token t of sequence b lives in
    physical page block_table[b, t // P] at slot t % P (P = page size).  Pages are
    laid out with every kv head's rows of a page contiguous: K_pages/V_pages
    [n_pages, Hkv, P, 128] bf16 bits, code_pages [n_pages, Hkv, P, 32], block_table
    int32 [B, max_pages].  The tokens are read through the table into sequence
    order and the plain step runs on them.  Returns (out float64 [B,Hq,128], idx
    int32 [B,Hq,budget])."""
    K, V, codes, lens = paged_to_contiguous(K_pages, V_pages, code_pages, block_table, seq_lens)
    out, idx, _ = decode_step(q, K, V, codes, lens, budget)
    return out, idx


def paged_to_contiguous(K_pages, V_pages, code_pages, block_table, seq_lens):
    """The contiguous cache [B, Hkv, max_pages * P, ...] that a paged cache describes
    (positions past each sequence's length are zero).  Raises on a table entry
    outside [0, n_pages) within a sequence."""
    K_pages = _c(K_pages, np.uint16)
    V_pages = _c(V_pages, np.uint16)
    code_pages = _c(code_pages, np.uint8)
    table = _c(block_table, np.int32)
    lens = _c(seq_lens, np.int32)
    n_pages, Hkv, P, d = K_pages.shape
    B, max_pages = table.shape
    if V_pages.shape != K_pages.shape or code_pages.shape != (n_pages, Hkv, P, 32) or lens.shape != (B,):
        raise ValueError("oracle: inconsistent shapes")
    Nmax = max_pages * P
    K = np.zeros((B, Hkv, Nmax, d), dtype=np.uint16)
    V = np.zeros_like(K)
    codes = np.zeros((B, Hkv, Nmax, 32), dtype=np.uint8)
    for b in range(B):
        n = int(lens[b])
        if n < 0 or n > Nmax:
            raise ValueError("oracle: sequence length outside the table")
        for t in range(n):
            page = int(table[b, t // P])
            if not 0 <= page < n_pages:
                raise ValueError("oracle: block table entry out of range")
            K[b, :, t] = K_pages[page, :, t % P]
            V[b, :, t] = V_pages[page, :, t % P]
            codes[b, :, t] = code_pages[page, :, t % P]
    return K, V, codes, lens


def decode_step_general(q, K, V, codes, seq_lens, budget: int, n_sink: int = 0, n_recent: int = 0,
                        group_shared: bool = False):
    """Decode step with forced rows and/or group-shared selection together (the
    rules of decode_step_forced and decode_step_group_shared combined): per token
    the ranking distance is -1 for a forced row, else its L1 distance (summed over
    the group's query heads when group_shared); k_eff = min(budget, len) tokens of
    smallest (distance, index) are kept, per query head or once per kv head.
    Returns (out float64 [B,Hq,128], idx int32 [B,Hq or Hkv,budget])."""
    q = _c(q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    codes = _c(codes, np.uint8)
    lens = _c(seq_lens, np.int32)
    B, Hq, d = q.shape
    _, Hkv, Nmax, _ = K.shape
    if Hq % Hkv or V.shape != K.shape or codes.shape != (B, Hkv, Nmax, 32) or lens.shape != (B,):
        raise ValueError("oracle: inconsistent shapes")
    if n_sink < 0 or n_recent < 0:
        raise ValueError("oracle: negative forced-row counts")
    G = Hq // Hkv
    qcodes = encode(q.reshape(-1, d)).reshape(B, Hq, 32)
    out = np.zeros((B, Hq, d), dtype=np.float64)
    idx = np.full((B, Hkv if group_shared else Hq, budget), -1, dtype=np.int32)
    for b in range(B):
        n = int(lens[b])
        if n < 0 or n > Nmax:
            raise ValueError("oracle: sequence length outside [0, Nmax]")
        keff = min(budget, n)
        if keff == 0:
            continue
        t = np.arange(n)
        forced = (t < n_sink) | (t >= n - n_recent)
        for h in range(Hkv):
            Ds = [distance(qcodes[b, h * G + g], codes[b, h, :n]).astype(np.int64) for g in range(G)]
            if group_shared:
                D = np.sum(Ds, axis=0)
                D[forced] = -1
                kept = select(D.astype(np.int32), keff)
                idx[b, h, :keff] = kept
                for g in range(G):
                    out[b, h * G + g] = attend(q[b, h * G + g], K[b, h, :n], V[b, h, :n], kept)
            else:
                for g in range(G):
                    D = Ds[g].copy()
                    D[forced] = -1
                    kept = select(D.astype(np.int32), keff)
                    idx[b, h * G + g, :keff] = kept
                    out[b, h * G + g] = attend(q[b, h * G + g], K[b, h, :n], V[b, h, :n], kept)
    return out, idx
