"""CPU stand-in for the three kernels of the sequence-sharded step (test double).

It restates, with NumPy and the oracle's own distance, what the kernels compute
for one slice, so that the exchange protocol (histograms gathered in slice order,
global rank bases, states merged by log-sum-exp) and the host driver can be
checked on CPU against the single-sequence oracle:

  score   hist[b, h, d] = tokens of the slice with L1 code distance d to query head h
  attend  with H = the histograms of all slices summed and B_r the sum over the
          slices before this one, a token of distance d that is the j-th such
          token of the slice (index order) sits at position
              sum_{d' < d} H[d'] + B_r[d] + j
          of the whole sequence's (distance, index) order; it is kept when that
          position is below k_eff = min(budget, total length), and the position is
          its idx slot (ADAMAS long-context sparse attention article,
          lnwmold.com/news/826806, §2.3 scoring and §5.2 token budget);
          its state is m = max s, l = sum 2^(s - m), o = sum 2^(s - m) v with
          s = q.k / sqrt(128) * log2 e over the kept rows.
  merge   out = sum_r 2^(m_r - M) o_r / sum_r 2^(m_r - M) l_r.
"""
from __future__ import annotations

import numpy as np
import torch

HIST_STRIDE = 388
PARTIAL_FLOATS = 132
LOG2E = 1.4426950408889634


def _u16(t) -> np.ndarray:
    a = t.numpy() if isinstance(t, torch.Tensor) else np.asarray(t)
    return a.view(np.uint16) if a.dtype == np.int16 else a


def bf16_to_f64(a_u16: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(a_u16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def slice_inputs(K, V, codes, lens, world: int, cuts=None):
    """Split every sequence b of length lens[b] into `world` contiguous slices; cuts
    (optional, [world + 1] fractions 0..1) places the boundaries, else even.
    Returns per rank (K_r, V_r, codes_r, lens_r) with Nmax_r = the longest slice."""
    B = lens.shape[0]
    bounds = np.zeros((world + 1, B), dtype=np.int64)
    for b in range(B):
        n = int(lens[b])
        for r in range(world + 1):
            f = (r / world) if cuts is None else cuts[r]
            bounds[r, b] = int(round(f * n)) if 0 < r < world else (0 if r == 0 else n)
        bounds[:, b] = np.maximum.accumulate(bounds[:, b])
    out = []
    for r in range(world):
        ln = (bounds[r + 1] - bounds[r]).astype(np.int32)
        nmax = max(1, int(ln.max(initial=0)))
        Kr = np.zeros((B, K.shape[1], nmax, K.shape[3]), dtype=K.dtype)
        Vr = np.zeros_like(Kr)
        Cr = np.zeros((B, codes.shape[1], nmax, codes.shape[3]), dtype=codes.dtype)
        for b in range(B):
            a, e = int(bounds[r, b]), int(bounds[r + 1, b])
            Kr[b, :, :e - a] = K[b, :, a:e]
            Vr[b, :, :e - a] = V[b, :, a:e]
            Cr[b, :, :e - a] = codes[b, :, a:e]
        out.append((Kr, Vr, Cr, ln))
    return out


class OracleShardOps:
    """score / attend / merge of one slice, on CPU tensors (numpy inside)."""

    def __init__(self, orc):
        self.orc = orc
        self._dist = None

    def score(self, q, codes, seq_lens, budget):
        qn = _u16(q)
        cn, lens = codes.numpy(), seq_lens.numpy()
        B, Hq, _ = qn.shape
        Hkv = cn.shape[1]
        G = Hq // Hkv
        qcodes = self.orc.encode(qn.reshape(-1, 128)).reshape(B, Hq, 32)
        hist = np.zeros((B, Hq, HIST_STRIDE), dtype=np.int32)
        self._dist = {}
        for b in range(B):
            n = int(lens[b]) if budget > 0 else 0
            for h in range(Hq):
                D = self.orc.distance(qcodes[b, h], cn[b, h // G, :n]) if n else np.zeros(0, np.int32)
                self._dist[b, h] = D
                hist[b, h, :385] = np.bincount(D, minlength=385)
        return torch.from_numpy(hist)

    def attend(self, q, K, V, seq_lens, budget, hist_all, rank):
        qn, Kn, Vn = _u16(q), _u16(K), _u16(V)
        ha = hist_all.numpy().astype(np.int64)
        B, Hq, _ = qn.shape
        G = Hq // Kn.shape[1]
        idx = np.full((B, Hq, budget), -1, dtype=np.int32)
        part = np.zeros((B, Hq, PARTIAL_FLOATS), dtype=np.float64)
        for b in range(B):
            for h in range(Hq):
                H = ha[:, b, h, :385].sum(0)
                before = ha[:rank, b, h, :385].sum(0)
                keff = min(budget, int(H.sum()))
                ofs = int(before.sum())
                smaller = np.concatenate([[0], np.cumsum(H)[:-1]])
                D = self._dist[b, h]
                seen = np.zeros(385, dtype=np.int64)
                kept = []
                for t, d in enumerate(D):
                    pos = smaller[d] + before[d] + seen[d]
                    seen[d] += 1
                    if pos < keff:
                        idx[b, h, pos] = ofs + t
                        kept.append(t)
                m, l, o = -np.inf, 0.0, np.zeros(128)
                if kept:
                    qf = bf16_to_f64(qn[b, h])
                    k = bf16_to_f64(Kn[b, h // G, kept])
                    v = bf16_to_f64(Vn[b, h // G, kept])
                    s = (k @ qf) / np.sqrt(128.0) * LOG2E
                    m = s.max()
                    w = np.exp2(s - m)
                    l, o = w.sum(), w @ v
                part[b, h, 0], part[b, h, 1], part[b, h, 4:] = m, l, o
        return torch.from_numpy(part), torch.from_numpy(idx)

    def merge(self, partials):
        P = partials.numpy().astype(np.float64)
        m = P[..., 0]
        M = m.max(0)
        out = np.zeros(P.shape[1:3] + (128,), dtype=np.float64)
        ok = np.isfinite(M)
        w = np.where(np.isfinite(m), np.exp2(m - np.where(ok, M, 0.0)), 0.0)
        L = (w * P[..., 1]).sum(0)
        O = (w[..., None] * P[..., 4:]).sum(0)
        out[ok] = O[ok] / L[ok][..., None]
        return torch.from_numpy(out)


def run_emulated(ops_per_rank, inputs_per_rank, q, budget):
    """The sharded step of len(ops_per_rank) slices in one process, phase by phase
    in the order every rank's driver takes them; returns (out, idx) as tensors."""
    world = len(ops_per_rank)
    hists = [ops.score(q, inp[2], inp[3], budget) for ops, inp in zip(ops_per_rank, inputs_per_rank)]
    hist_all = torch.stack(hists, 0)
    states = [ops.attend(q, inp[0], inp[1], inp[3], budget, hist_all, r)
              for r, (ops, inp) in enumerate(zip(ops_per_rank, inputs_per_rank))]
    partials = torch.stack([s[0] for s in states], 0)
    idx = states[0][1]
    for r in range(1, world):
        idx = torch.maximum(idx, states[r][1])
    return ops_per_rank[0].merge(partials), idx
