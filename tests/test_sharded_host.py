"""Sequence-sharded step on CPU: the exchange protocol and the torch.distributed driver.

The sequence is split into contiguous slices, one per rank.  With the kernels
replaced by their CPU restatement (shard_ops_cpu.OracleShardOps), the protocol --
histograms gathered in slice order, global rank bases, states merged by their
log-sum-exp weights -- must give exactly the oracle's step on the whole sequence:
the same idx, and out equal up to float64 rounding.  Then the same through
compressed_sparse_kv_fp32_b200.sharded.decode_step_sharded over a gloo process
group of two ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from compressed_sparse_kv_fp32_b200 import sharded, synth
from shard_ops_cpu import OracleShardOps, run_emulated, slice_inputs


def _case(B, Hq, Hkv, N, lens, seed, equal_keys=False):
    w = synth.WORKLOADS[4].scaled(B=B, Hq=Hq, Hkv=Hkv, Nmax=N, len_range=None, n_needles=2, seed=seed)
    inp = synth.make_inputs(w)
    inp["lens"] = np.asarray(lens, np.int32)
    if equal_keys:  # every key the same: every distance ties, so the global index decides
        inp["K"][:] = inp["K"][:, :, :1]
    return inp


def _tensors(sl):
    Kr, Vr, Cr, ln = sl
    return (torch.from_numpy(Kr.view(np.int16)), torch.from_numpy(Vr.view(np.int16)), torch.from_numpy(Cr),
            torch.from_numpy(ln))


CASES = [
    # B, Hq, Hkv, N, lens, world, cuts, budgets
    (1, 2, 2, 3000, [3000], 2, None, (0, 1, 64, 5000)),
    (2, 4, 2, 3000, [3000, 700], 3, (0.0, 0.1, 0.8, 1.0), (16, 300)),
    (1, 1, 1, 2000, [2000], 4, (0.0, 0.0, 0.5, 0.5, 1.0), (100,)),          # two empty slices
    (3, 3, 1, 1500, [1500, 0, 1], 2, None, (8, 2000)),                     # empty and one-token sequences
]


@pytest.mark.parametrize("B,Hq,Hkv,N,lens,world,cuts,budgets", CASES)
def test_protocol_gives_the_whole_sequence_step(orc, B, Hq, Hkv, N, lens, world, cuts, budgets):
    inp = _case(B, Hq, Hkv, N, lens, seed=7 + world)
    codes = orc.encode(inp["K"])
    slices = [_tensors(s) for s in slice_inputs(inp["K"], inp["V"], codes, inp["lens"], world, cuts)]
    q = torch.from_numpy(inp["q"].view(np.int16))
    for budget in budgets:
        ops = [OracleShardOps(orc) for _ in range(world)]
        out, idx = run_emulated(ops, slices, q, budget)
        want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, inp["lens"], budget)
        assert np.array_equal(idx.numpy(), want_idx), budget
        np.testing.assert_allclose(out.numpy(), want_out, rtol=0, atol=1e-9)


def test_ties_across_slices_go_to_the_lower_global_index(orc):
    inp = _case(1, 2, 1, 1200, [1200], seed=3, equal_keys=True)
    codes = orc.encode(inp["K"])
    slices = [_tensors(s) for s in slice_inputs(inp["K"], inp["V"], codes, inp["lens"], 3, (0, 0.3, 0.35, 1))]
    q = torch.from_numpy(inp["q"].view(np.int16))
    out, idx = run_emulated([OracleShardOps(orc) for _ in range(3)], slices, q, 500)
    assert np.array_equal(idx.numpy()[0, 0], np.arange(500))
    want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, inp["lens"], 500)
    assert np.array_equal(idx.numpy(), want_idx)
    np.testing.assert_allclose(out.numpy(), want_out, rtol=0, atol=1e-9)


def test_slice_bounds_cover_the_sequence_in_order():
    for n in (0, 1, 7, 1000, 2 ** 21):
        for world in (1, 2, 3, 8):
            spans = [sharded.slice_bounds(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[r][1] == spans[r + 1][0] for r in range(world - 1))
            assert max(e - a for a, e in spans) - min(e - a for a, e in spans) <= 1
    with pytest.raises(ValueError):
        sharded.slice_bounds(10, 2, 2)


# ---------------------------------------------------------------- two gloo ranks
def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, budget, q_out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        from oracle import oracle as orc
        dist.init_process_group("gloo", rank=rank, world_size=world)
        inp = _case(2, 4, 2, 2500, [2500, 1100], seed=11)
        codes = orc.encode(inp["K"])
        Kr, Vr, Cr, ln = _tensors(slice_inputs(inp["K"], inp["V"], codes, inp["lens"], world)[rank])
        q = torch.from_numpy(inp["q"].view(np.int16))
        ex = sharded.TorchExchange()
        out, idx = sharded.decode_step_sharded(q, Cr, Kr, Vr, ln, budget, OracleShardOps(orc), ex)
        q_out.put((rank, out.numpy(), idx.numpy(), None))
    except Exception as e:  # reported to the parent
        q_out.put((rank, None, None, repr(e)))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_driver_over_two_gloo_ranks(orc):
    world, budget = 2, 200
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, budget, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, out, idx, err = q_out.get(timeout=150)
        assert err is None, err
        res[r] = (out, idx)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    inp = _case(2, 4, 2, 2500, [2500, 1100], seed=11)
    want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], orc.encode(inp["K"]), inp["lens"], budget)
    for r in range(world):  # every rank ends with the whole step's result
        assert np.array_equal(res[r][1], want_idx)
        np.testing.assert_allclose(res[r][0], want_out, rtol=0, atol=1e-9)
