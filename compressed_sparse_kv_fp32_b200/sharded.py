"""Sequence-sharded decode step: one long sequence split into contiguous slices, one
slice per GPU, for contexts longer than one GPU holds (the 2M-token context blog,
intelliparadigm.com/.../2174157, §5.1: two million tokens need several GPUs or CPU
offloading; the AMD Zebra-HyLo article, yeyulingfeng.com/a/1106654.html, reports
2M-token contexts).

Rank r holds the r-th slice of every sequence (codes, K, V as [B, Hkv, Nmax, ...],
seq_lens[b] the slice's length).  One step exchanges two small messages:

  1. score (kernel): the slice's distance histograms, [B, Hq, 388] uint32;
  2. all-gather of the histograms, in rank order;
  3. attend (kernel): the threshold and rank bases of the whole sequence come from
     the gathered histograms, so every rank keeps exactly its share of the
     sequence's top-k (ties to the lower global index); it writes their global
     indices into idx (-1 elsewhere) and its softmax state (m, l, o) over them;
  4. all-gather of the states, all-reduce (max) of idx;
  5. merge (kernel): out = the states combined by their log-sum-exp weights.

The result is the single-GPU step on the whole sequence.  The kernels are the
library's (adamas.shard_score / shard_attend / merge_partials); this module only
orders them around the collectives.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import adamas


class TorchExchange:
    """The step's collectives over a torch.distributed process group (NCCL between
    GPUs; any backend that has all_gather and a MAX all_reduce for int32)."""

    def __init__(self, group: Optional[dist.ProcessGroup] = None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self._flat = dist.get_backend(group) == "nccl"

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        """[world, *t.shape], rank r's tensor at [r]."""
        out = torch.empty((self.world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        if self._flat:
            dist.all_gather_into_tensor(out, t.contiguous(), group=self.group)
        else:
            dist.all_gather(list(out.unbind(0)), t.contiguous(), group=self.group)
        return out

    def all_reduce_max(self, t: torch.Tensor) -> torch.Tensor:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=self.group)
        return t


class CudaShardOps:
    """The three kernels of the sharded step on this GPU, with their workspace."""

    def __init__(self, B: int, Hq: int, Hkv: int, Nmax: int, budget: int, device=None):
        self.workspace = adamas.Workspace(B, Hq, Hkv, Nmax, budget, device=device, sharded=True)

    def score(self, q, codes, seq_lens, budget):
        return adamas.shard_score(q, codes, seq_lens, budget, self.workspace)

    def attend(self, q, K, V, seq_lens, budget, hist_all, rank):
        return adamas.shard_attend(q, K, V, seq_lens, budget, hist_all, rank, self.workspace)

    def merge(self, partials):
        return adamas.merge_partials(partials)


def decode_step_sharded(q: torch.Tensor, codes: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                        seq_lens: torch.Tensor, budget: int, ops, exchange) -> Tuple[torch.Tensor, torch.Tensor]:
    """One decode step over this rank's slice; returns (out [B, Hq, 128] fp32,
    idx [B, Hq, budget] int32 of global indices), the same on every rank.

    ops: the kernels (CudaShardOps); exchange: the collectives (TorchExchange).
    Every rank makes the same collective calls in the same order."""
    hist = ops.score(q, codes, seq_lens, budget)
    hist_all = exchange.all_gather(hist)
    partial, idx = ops.attend(q, K, V, seq_lens, budget, hist_all, exchange.rank)
    partials = exchange.all_gather(partial)
    exchange.all_reduce_max(idx)
    out = ops.merge(partials)
    return out, idx


def slice_bounds(total_len: int, world: int, rank: int) -> Tuple[int, int]:
    """The contiguous slice [begin, end) of a sequence of total_len tokens that rank
    `rank` of `world` holds when the sequence is split as evenly as possible."""
    if world < 1 or not 0 <= rank < world or total_len < 0:
        raise ValueError("slice_bounds: need world >= 1, 0 <= rank < world, total_len >= 0")
    return total_len * rank // world, total_len * (rank + 1) // world
