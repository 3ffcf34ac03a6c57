"""Sequence-sharded step on the GPU (adamas_shard_score / adamas_shard_attend /
adamas_merge_partials) against the oracle's step on the whole sequence.

The ranks are emulated in one process: every slice has its own cache arrays and
workspace, and the phases run slice by slice in the order each rank's driver takes
them (score, gather the histograms, attend, gather the states and reduce idx,
merge), so no kernel ever waits on another.  idx must equal the oracle's; out
within max-abs 1e-2 / rel-RMS 1e-3.  Then the torch.distributed driver over a
one-rank NCCL group, against the single-GPU step."""
import numpy as np
import pytest
import torch
import torch.distributed as dist

from compressed_sparse_kv_fp32_b200 import adamas, sharded, synth
from helpers import assert_close_out, dev, dev_bf16
from shard_ops_cpu import slice_inputs

pytestmark = pytest.mark.gpu


def _case(B, Hq, Hkv, N, lens, seed, equal_keys=False):
    w = synth.WORKLOADS[4].scaled(B=B, Hq=Hq, Hkv=Hkv, Nmax=N, len_range=None, n_needles=3, seed=seed)
    inp = synth.make_inputs(w)
    inp["lens"] = np.asarray(lens, np.int32)
    if equal_keys:
        inp["K"][:] = inp["K"][:, :, :1]
    return inp


def _gpu_slices(inp, world, cuts):
    dummy = np.zeros(inp["K"].shape[:3] + (32,), np.uint8)  # codes come from the GPU encoder per slice
    out = []
    for Kr, Vr, _, ln in slice_inputs(inp["K"], inp["V"], dummy, inp["lens"], world, cuts):
        K, V = dev_bf16(Kr), dev_bf16(Vr)
        codes = torch.empty(K.shape[:3] + (32,), dtype=torch.uint8, device="cuda")
        adamas.encode_keys(K, codes)
        out.append((K, V, codes, dev(ln)))
    return out


def _run(q, slices, budget):
    B, Hq, _ = q.shape
    Hkv = slices[0][0].shape[1]
    ops = [sharded.CudaShardOps(B, Hq, Hkv, s[0].shape[2], budget) for s in slices]
    hist_all = torch.stack([o.score(q, s[2], s[3], budget) for o, s in zip(ops, slices)], 0)
    states = [o.attend(q, s[0], s[1], s[3], budget, hist_all, r) for r, (o, s) in enumerate(zip(ops, slices))]
    idx = states[0][1].clone()
    for _, i in states[1:]:
        idx = torch.maximum(idx, i)
    out = ops[0].merge(torch.stack([p for p, _ in states], 0))
    torch.cuda.synchronize()
    for o in ops:
        assert o.workspace.device_error() == 0
    return out.cpu().numpy(), idx.cpu().numpy()


@pytest.mark.parametrize("B,Hq,Hkv,N,lens,world,cuts,budgets", [
    (1, 2, 2, 3000, [3000], 2, None, (0, 1, 64, 5000)),
    (2, 4, 2, 3000, [3000, 700], 3, (0.0, 0.1, 0.8, 1.0), (16, 300)),
    (1, 1, 1, 2000, [2000], 4, (0.0, 0.0, 0.5, 0.5, 1.0), (100,)),       # two empty slices
    (3, 3, 1, 1500, [1500, 0, 1], 2, None, (8, 2000)),                  # empty and one-token sequences
    (2, 4, 4, 40000, [40000, 25000], 2, None, (1024,)),                 # several blocks per slice
    (1, 8, 1, 200000, [200000], 3, (0.0, 0.2, 0.7, 1.0), (512,)),      # G = 8, uneven slices
])
def test_emulated_ranks_give_the_whole_sequence_step(orc, B, Hq, Hkv, N, lens, world, cuts, budgets):
    inp = _case(B, Hq, Hkv, N, lens, seed=17 + world)
    slices = _gpu_slices(inp, world, cuts)
    q = dev_bf16(inp["q"])
    codes = orc.encode(inp["K"])
    for budget in budgets:
        out, idx = _run(q, slices, budget)
        want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, inp["lens"], budget)
        assert np.array_equal(idx, want_idx), budget
        assert_close_out(out, want_out)


def test_ties_across_slices_go_to_the_lower_global_index(orc):
    inp = _case(1, 2, 1, 30000, [30000], seed=5, equal_keys=True)
    slices = _gpu_slices(inp, 3, (0.0, 0.3, 0.35, 1.0))
    out, idx = _run(dev_bf16(inp["q"]), slices, 2000)
    assert np.array_equal(idx[0, 0], np.arange(2000))
    want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], orc.encode(inp["K"]), inp["lens"], 2000)
    assert np.array_equal(idx, want_idx)
    assert_close_out(out, want_out)


def test_four_slices_match_the_single_gpu_step_at_512k():
    inp = _case(1, 2, 2, 1 << 19, [1 << 19], seed=29)
    q = dev_bf16(inp["q"])
    K, V = dev_bf16(inp["K"]), dev_bf16(inp["V"])
    codes = torch.empty(K.shape[:3] + (32,), dtype=torch.uint8, device="cuda")
    adamas.encode_keys(K, codes)
    ws = adamas.Workspace(1, 2, 2, 1 << 19, 1024)
    ref_out, ref_idx = adamas.decode_step(q, codes, K, V, dev(inp["lens"]), 1024, ws)
    out, idx = _run(q, _gpu_slices(inp, 4, None), 1024)
    assert np.array_equal(idx, ref_idx.cpu().numpy())
    assert_close_out(out, ref_out.cpu().numpy())


def test_driver_over_a_one_rank_nccl_group():
    inp = _case(2, 4, 2, 5000, [5000, 3000], seed=31)
    (K, V, codes, lens), = _gpu_slices(inp, 1, None)
    q = dev_bf16(inp["q"])
    ws = adamas.Workspace(2, 4, 2, 5000, 256)
    ref_out, ref_idx = adamas.decode_step(q, codes, K, V, lens, 256, ws)
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1)
    try:
        ops = sharded.CudaShardOps(2, 4, 2, 5000, 256)
        out, idx = sharded.decode_step_sharded(q, codes, K, V, lens, 256, ops, sharded.TorchExchange())
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(idx, ref_idx)
    assert_close_out(out.cpu().numpy(), ref_out.cpu().numpy())
