"""Python binding of libadamas.so (C ABI in include/adamas.h).

Argument marshalling only: every step of the method runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors; calls are enqueued on the current torch
stream.  The library must have been built (compressed_sparse_kv_fp32_b200.build);
there is no fallback of any kind.

Method: ADAMAS long-context sparse attention article (lnwmold.com/news/826806),
§2.1 Hadamard rotation, §2.2 dynamic 2-bit bucketing, §3.1 packed code cache,
§2.3 Manhattan-distance scoring, §5.2 token budget.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

from .build import LIBRARY

HEAD_DIM = 128
DEVERR_SEQLEN = 0x1
DEVERR_TIMEOUT = 0x2

_lock = threading.Lock()
_lib = None

SYMBOLS = (
    "adamas_status_string", "adamas_version", "adamas_last_error_string", "adamas_workspace_bytes", "adamas_workspace_init",
    "adamas_encode_keys", "adamas_decode_step", "adamas_score", "adamas_get_device_error",
    "adamas_decode_step_static", "adamas_decode_step_append", "adamas_decode_step_ex",
    "adamas_static_device_error", "adamas_debug_withhold_stage",
    "adamas_shard_workspace_bytes", "adamas_shard_score", "adamas_shard_attend", "adamas_merge_partials",
)

SELECT_PER_HEAD = 0
SELECT_GROUP_SHARED = 1
DEVERR_INTERNAL = 0x4
DEVERR_TABLE = 0x8


class DecodeArgs(ctypes.Structure):
    """Mirror of adamas_decode_args (include/adamas.h), field for field."""

    _fields_ = [
        ("q", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("K", ctypes.c_void_p), ("V", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
        ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("Nmax", ctypes.c_int64),
        ("d", ctypes.c_int), ("budget", ctypes.c_int),
        ("out", ctypes.c_void_p), ("idx", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("append_pos", ctypes.c_void_p), ("k_new", ctypes.c_void_p), ("v_new", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p), ("n_pages", ctypes.c_int64), ("page_size", ctypes.c_int),
        ("max_pages", ctypes.c_int), ("n_sink", ctypes.c_int), ("n_recent", ctypes.c_int), ("policy", ctypes.c_int),
    ]


class AdamasError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = f": {load().adamas_last_error_string().decode()}" if status == -4 else ""
        super().__init__(f"{where}: {status_string(status)} ({status}){detail}")


def load(path: str = LIBRARY) -> ctypes.CDLL:
    """Load libadamas.so and declare its signatures (raises if it was not built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: build it with `python -m compressed_sparse_kv_fp32_b200.build`")
        l = ctypes.CDLL(path)
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        l.adamas_status_string.argtypes = [I]
        l.adamas_status_string.restype = ctypes.c_char_p
        l.adamas_version.argtypes = []
        l.adamas_version.restype = I
        l.adamas_last_error_string.argtypes = []
        l.adamas_last_error_string.restype = ctypes.c_char_p
        l.adamas_workspace_bytes.argtypes = [I, I, I, I64, I, I]
        l.adamas_workspace_bytes.restype = SZ
        l.adamas_workspace_init.argtypes = [P, SZ, P]
        l.adamas_workspace_init.restype = I
        l.adamas_encode_keys.argtypes = [P, P, P, I, I, I, I64, I, P]
        l.adamas_encode_keys.restype = I
        l.adamas_decode_step.argtypes = [P, P, P, P, P, I, I, I, I64, I, I, P, P, P, SZ, P]
        l.adamas_decode_step.restype = I
        l.adamas_score.argtypes = [P, P, P, I, I, I, I64, I, P, P]
        l.adamas_score.restype = I
        l.adamas_get_device_error.argtypes = [P, SZ, ctypes.POINTER(ctypes.c_uint32), P]
        l.adamas_get_device_error.restype = I
        l.adamas_decode_step_static.argtypes = [P, P, P, P, P, I, I, I, I64, I, I, P, P, P]
        l.adamas_decode_step_static.restype = I
        l.adamas_decode_step_append.argtypes = [P, P, P, P, P, P, I, I, I, I64, I, I, P, P, P, SZ, P]
        l.adamas_decode_step_append.restype = I
        l.adamas_decode_step_ex.argtypes = [ctypes.POINTER(DecodeArgs), P]
        l.adamas_decode_step_ex.restype = I
        l.adamas_static_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), P]
        l.adamas_static_device_error.restype = I
        l.adamas_shard_workspace_bytes.argtypes = [I, I, I, I64, I, I]
        l.adamas_shard_workspace_bytes.restype = SZ
        l.adamas_shard_score.argtypes = [P, P, P, I, I, I, I64, I, I, P, P, SZ, P]
        l.adamas_shard_score.restype = I
        l.adamas_shard_attend.argtypes = [P, P, P, P, I, I, I, I64, I, I, P, I, I, P, P, P, SZ, P]
        l.adamas_shard_attend.restype = I
        l.adamas_merge_partials.argtypes = [P, I, I, I, P, P]
        l.adamas_merge_partials.restype = I
        l.adamas_debug_withhold_stage.argtypes = [I]
        l.adamas_debug_withhold_stage.restype = None
        _lib = l
        return l


def status_string(status: int) -> str:
    return load().adamas_status_string(int(status)).decode()


def _check(rc: int, where: str):
    if rc != 0:
        raise AdamasError(rc, where)


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape: Optional[tuple] = None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def workspace_bytes(B: int, Hq: int, Hkv: int, Nmax: int, budget: int, d: int = HEAD_DIM) -> int:
    n = load().adamas_workspace_bytes(B, Hq, Hkv, Nmax, d, budget)
    if n == 0:
        raise AdamasError(-2, "adamas_workspace_bytes")
    return int(n)


def shard_workspace_bytes(B: int, Hq: int, Hkv: int, Nmax: int, budget: int, d: int = HEAD_DIM) -> int:
    n = load().adamas_shard_workspace_bytes(B, Hq, Hkv, Nmax, d, budget)
    if n == 0:
        raise AdamasError(-2, "adamas_shard_workspace_bytes")
    return int(n)


class Workspace:
    """Device workspace of adamas_decode_step (or, with sharded=True, of the
    sequence-sharded step's two halves), zero-filled on creation."""

    def __init__(self, B: int, Hq: int, Hkv: int, Nmax: int, budget: int, device=None,
                 stream: Optional[torch.cuda.Stream] = None, sharded: bool = False):
        self.nbytes = (shard_workspace_bytes if sharded else workspace_bytes)(B, Hq, Hkv, Nmax, budget)
        self.buffer = torch.empty(self.nbytes, dtype=torch.uint8,
                                  device=device if device is not None else "cuda")
        self.reset(stream)

    def reset(self, stream: Optional[torch.cuda.Stream] = None):
        _check(load().adamas_workspace_init(self.buffer.data_ptr(), self.nbytes, _stream(stream)),
               "adamas_workspace_init")

    def device_error(self, stream: Optional[torch.cuda.Stream] = None) -> int:
        """Synchronise the stream and return the device error word (DEVERR_* bits)."""
        word = ctypes.c_uint32(0)
        rc = load().adamas_get_device_error(self.buffer.data_ptr(), self.nbytes, ctypes.byref(word),
                                            _stream(stream))
        if rc not in (0, -5):
            raise AdamasError(rc, "adamas_get_device_error")
        return int(word.value)


def encode_keys(K: torch.Tensor, codes: torch.Tensor, pos_begin: Optional[torch.Tensor] = None,
                count: Optional[int] = None, stream: Optional[torch.cuda.Stream] = None):
    """Encode K [B,Hkv,Nmax,128] bf16 into codes [B,Hkv,Nmax,32] uint8 at positions
    [pos_begin[b], pos_begin[b] + count) (all positions by default)."""
    _need(K, "K", torch.bfloat16)
    if K.dim() != 4 or K.shape[-1] != HEAD_DIM:
        raise ValueError("K must be [B, Hkv, Nmax, 128]")
    B, Hkv, Nmax, d = K.shape
    _need(codes, "codes", torch.uint8, (B, Hkv, Nmax, d // 4))
    if pos_begin is not None:
        _need(pos_begin, "pos_begin", torch.int32, (B,))
    n = Nmax if count is None else int(count)
    _check(load().adamas_encode_keys(K.data_ptr(), codes.data_ptr(), _ptr(pos_begin), n, B, Hkv, Nmax, d,
                                     _stream(stream)), "adamas_encode_keys")
    return codes


def _decode_args(q, codes, K, V, seq_lens, budget, out, idx):
    _need(q, "q", torch.bfloat16)
    if q.dim() != 3:
        raise ValueError("q must be [B, Hq, 128]")
    B, Hq, d = q.shape
    _need(K, "K", torch.bfloat16)
    if K.dim() != 4:
        raise ValueError("K must be [B, Hkv, Nmax, 128]")
    _, Hkv, Nmax, _ = K.shape
    _need(K, "K", torch.bfloat16, (B, Hkv, Nmax, d))
    _need(V, "V", torch.bfloat16, (B, Hkv, Nmax, d))
    _need(codes, "codes", torch.uint8, (B, Hkv, Nmax, d // 4))
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty((B, Hq, budget), dtype=torch.int32, device=q.device)
    _need(out, "out", torch.float32, (B, Hq, d))
    _need(idx, "idx", torch.int32, (B, Hq, budget))
    return B, Hq, Hkv, Nmax, d, out, idx


def decode_step(q: torch.Tensor, codes: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                seq_lens: torch.Tensor, budget: int, workspace: Workspace,
                out: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One decode step: returns (out [B,Hq,128] fp32, idx [B,Hq,budget] int32)."""
    B, Hq, Hkv, Nmax, d, out, idx = _decode_args(q, codes, K, V, seq_lens, budget, out, idx)
    rc = load().adamas_decode_step(q.data_ptr(), codes.data_ptr(), K.data_ptr(), V.data_ptr(),
                                   seq_lens.data_ptr(), B, Hq, Hkv, Nmax, d, budget, out.data_ptr(),
                                   idx.data_ptr() if budget > 0 else None,
                                   workspace.buffer.data_ptr(), workspace.nbytes, _stream(stream))
    _check(rc, "adamas_decode_step")
    return out, idx


def decode_step_append(q: torch.Tensor, codes: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                       seq_lens: torch.Tensor, append_pos: torch.Tensor, budget: int, workspace: Workspace,
                       out: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                       stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """encode_keys of the key at append_pos[b] (int32 [B]; out of [0, Nmax): none)
    followed by decode_step, in one launch; codes is updated in place."""
    B, Hq, Hkv, Nmax, d, out, idx = _decode_args(q, codes, K, V, seq_lens, budget, out, idx)
    _need(append_pos, "append_pos", torch.int32, (B,))
    rc = load().adamas_decode_step_append(q.data_ptr(), codes.data_ptr(), K.data_ptr(), V.data_ptr(),
                                          seq_lens.data_ptr(), append_pos.data_ptr(), B, Hq, Hkv, Nmax, d,
                                          budget, out.data_ptr(), idx.data_ptr() if budget > 0 else None,
                                          workspace.buffer.data_ptr(), workspace.nbytes, _stream(stream))
    _check(rc, "adamas_decode_step_append")
    return out, idx


def score(q: torch.Tensor, codes: torch.Tensor, seq_lens: torch.Tensor, Hkv: Optional[int] = None,
          stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """L1 code distances [B,Hq,Nmax] (uint16 values in an int16 tensor; 0xFFFF past each length)."""
    _need(q, "q", torch.bfloat16)
    B, Hq, d = q.shape
    _need(codes, "codes", torch.uint8)
    _, Hkv, Nmax, _ = codes.shape
    _need(codes, "codes", torch.uint8, (B, Hkv, Nmax, d // 4))
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    dist = torch.empty((B, Hq, Nmax), dtype=torch.int16, device=q.device)
    _check(load().adamas_score(q.data_ptr(), codes.data_ptr(), seq_lens.data_ptr(), B, Hq, Hkv, Nmax, d,
                               dist.data_ptr(), _stream(stream)), "adamas_score")
    return dist


def decode(q: torch.Tensor, codes: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_lens: torch.Tensor,
           budget: int, workspace: Workspace, *, append_pos: Optional[torch.Tensor] = None,
           k_new: Optional[torch.Tensor] = None, v_new: Optional[torch.Tensor] = None,
           block_table: Optional[torch.Tensor] = None, n_sink: int = 0, n_recent: int = 0,
           policy: int = SELECT_PER_HEAD, out: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
           stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """adamas_decode_step_ex: the decode step with every option.

    Contiguous cache: codes [B,Hkv,Nmax,32], K/V [B,Hkv,Nmax,128].  Paged cache
    (block_table int32 [B, max_pages]): codes [n_pages,Hkv,P,32], K/V
    [n_pages,Hkv,P,128] with P the page size.  append_pos int32 [B] encodes the key
    at that position first; k_new/v_new bf16 [B,Hkv,128] are also written into the
    cache there by the launch.  n_sink/n_recent force the first/last tokens of each
    sequence into the kept set.  policy SELECT_GROUP_SHARED keeps one budget per kv
    head (idx [B,Hkv,budget]).  Returns (out [B,Hq,128] fp32, idx)."""
    _need(q, "q", torch.bfloat16)
    if q.dim() != 3:
        raise ValueError("q must be [B, Hq, 128]")
    B, Hq, d = q.shape
    _need(K, "K", torch.bfloat16)
    if K.dim() != 4:
        raise ValueError("K must be 4-dimensional")
    paged = block_table is not None
    if paged:
        n_pages, Hkv, page_size, _ = K.shape
        _need(block_table, "block_table", torch.int32)
        if block_table.dim() != 2 or block_table.shape[0] != B:
            raise ValueError("block_table must be [B, max_pages]")
        max_pages = block_table.shape[1]
        Nmax = max_pages * page_size
        _need(K, "K", torch.bfloat16, (n_pages, Hkv, page_size, d))
        _need(V, "V", torch.bfloat16, (n_pages, Hkv, page_size, d))
        _need(codes, "codes", torch.uint8, (n_pages, Hkv, page_size, d // 4))
    else:
        _, Hkv, Nmax, _ = K.shape
        n_pages = page_size = max_pages = 0
        _need(K, "K", torch.bfloat16, (B, Hkv, Nmax, d))
        _need(V, "V", torch.bfloat16, (B, Hkv, Nmax, d))
        _need(codes, "codes", torch.uint8, (B, Hkv, Nmax, d // 4))
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    rows = Hkv if policy == SELECT_GROUP_SHARED else Hq
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty((B, rows, budget), dtype=torch.int32, device=q.device)
    _need(out, "out", torch.float32, (B, Hq, d))
    _need(idx, "idx", torch.int32, (B, rows, budget))
    if append_pos is not None:
        _need(append_pos, "append_pos", torch.int32, (B,))
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    if k_new is not None:
        _need(k_new, "k_new", torch.bfloat16, (B, Hkv, d))
        _need(v_new, "v_new", torch.bfloat16, (B, Hkv, d))
    a = DecodeArgs(q.data_ptr(), codes.data_ptr(), K.data_ptr(), V.data_ptr(), seq_lens.data_ptr(),
                   B, Hq, Hkv, Nmax, d, budget, out.data_ptr(), idx.data_ptr() if budget > 0 else None,
                   workspace.buffer.data_ptr(), workspace.nbytes, _ptr(append_pos), _ptr(k_new), _ptr(v_new),
                   _ptr(block_table), n_pages, page_size, max_pages, n_sink, n_recent, policy)
    _check(load().adamas_decode_step_ex(ctypes.byref(a), _stream(stream)), "adamas_decode_step_ex")
    return out, idx


# ---------------------------------------------------------------- sequence-sharded step
HIST_STRIDE = 388      # ADAMAS_HIST_STRIDE: uint32 bins per (b, query head) of an exchanged histogram
PARTIAL_FLOATS = 132   # ADAMAS_PARTIAL_FLOATS: fp32 per (b, query head) of a softmax state


def _shard_shapes(q, codes_or_K, seq_lens):
    _need(q, "q", torch.bfloat16)
    if q.dim() != 3:
        raise ValueError("q must be [B, Hq, 128]")
    B, Hq, d = q.shape
    if codes_or_K.dim() != 4:
        raise ValueError("the cache must be [B, Hkv, Nmax, ...]")
    _, Hkv, Nmax, _ = codes_or_K.shape
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    return B, Hq, Hkv, Nmax, d


def shard_score(q: torch.Tensor, codes: torch.Tensor, seq_lens: torch.Tensor, budget: int, workspace: Workspace,
                hist: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """First half of the sharded step on this GPU's slice: returns its histograms
    [B, Hq, HIST_STRIDE] int32 (uint32 counts), to be all-gathered in rank order."""
    B, Hq, Hkv, Nmax, d = _shard_shapes(q, codes, seq_lens)
    _need(codes, "codes", torch.uint8, (B, Hkv, Nmax, d // 4))
    if hist is None:
        hist = torch.empty((B, Hq, HIST_STRIDE), dtype=torch.int32, device=q.device)
    _need(hist, "hist", torch.int32, (B, Hq, HIST_STRIDE))
    _check(load().adamas_shard_score(q.data_ptr(), codes.data_ptr(), seq_lens.data_ptr(), B, Hq, Hkv, Nmax, d,
                                     budget, hist.data_ptr(), workspace.buffer.data_ptr(), workspace.nbytes,
                                     _stream(stream)), "adamas_shard_score")
    return hist


def shard_attend(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_lens: torch.Tensor, budget: int,
                 hist_all: torch.Tensor, rank: int, workspace: Workspace, partial: Optional[torch.Tensor] = None,
                 idx: Optional[torch.Tensor] = None,
                 stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Second half on this GPU's slice, with hist_all [world, B, Hq, HIST_STRIDE] of
    every slice: returns (partial [B, Hq, PARTIAL_FLOATS] fp32, idx [B, Hq, budget]
    int32 holding the global indices of this slice's kept tokens, -1 elsewhere)."""
    B, Hq, Hkv, Nmax, d = _shard_shapes(q, K, seq_lens)
    _need(K, "K", torch.bfloat16, (B, Hkv, Nmax, d))
    _need(V, "V", torch.bfloat16, (B, Hkv, Nmax, d))
    if hist_all.dim() != 4:
        raise ValueError("hist_all must be [world, B, Hq, HIST_STRIDE]")
    world = hist_all.shape[0]
    _need(hist_all, "hist_all", torch.int32, (world, B, Hq, HIST_STRIDE))
    if partial is None:
        partial = torch.empty((B, Hq, PARTIAL_FLOATS), dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty((B, Hq, budget), dtype=torch.int32, device=q.device)
    _need(partial, "partial", torch.float32, (B, Hq, PARTIAL_FLOATS))
    _need(idx, "idx", torch.int32, (B, Hq, budget))
    _check(load().adamas_shard_attend(q.data_ptr(), K.data_ptr(), V.data_ptr(), seq_lens.data_ptr(), B, Hq, Hkv,
                                      Nmax, d, budget, hist_all.data_ptr(), world, int(rank), partial.data_ptr(),
                                      idx.data_ptr() if budget > 0 else None, workspace.buffer.data_ptr(),
                                      workspace.nbytes, _stream(stream)), "adamas_shard_attend")
    return partial, idx


def merge_partials(partials: torch.Tensor, out: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Attention output [B, Hq, 128] fp32 from the states [n, B, Hq, PARTIAL_FLOATS] of n slices."""
    if partials.dim() != 4:
        raise ValueError("partials must be [n, B, Hq, PARTIAL_FLOATS]")
    n, B, Hq, _ = partials.shape
    _need(partials, "partials", torch.float32, (n, B, Hq, PARTIAL_FLOATS))
    if out is None:
        out = torch.empty((B, Hq, HEAD_DIM), dtype=torch.float32, device=partials.device)
    _need(out, "out", torch.float32, (B, Hq, HEAD_DIM))
    _check(load().adamas_merge_partials(partials.data_ptr(), n, B, Hq, out.data_ptr(), _stream(stream)),
           "adamas_merge_partials")
    return out
