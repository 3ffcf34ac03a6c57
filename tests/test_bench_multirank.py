"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

Under torchrun every rank runs its own replica of the workload (the decode path
has no exchange step between (b, kv head) units); the reported time is the max
over ranks and the value counts the steps of all ranks.  Only rank 0 runs and
prints the reference (oracle) arm."""
import contextlib
import io
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 5.0])
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            if rank != 0:
                bench.run_reference(None, rank, world)  # must return at once, print nothing
        dist.barrier()
        q.put((rank, got, buf.getvalue()))
    except Exception as e:  # reported to the parent
        q.put((rank, repr(e), ""))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_reference_rank0_only():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict((r, (g, out)) for r, g, out in (q.get(timeout=100) for _ in range(world)))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for r in range(world):
        got, out = results[r]
        assert got == [2.0, 10.0, 5.0], got
        assert out == ""


def test_single_rank_identity_and_job_value():
    assert bench.max_over_ranks([3.0, 4.5]) == [3.0, 4.5]
    assert bench.job_value(1, 100, 50.0) == pytest.approx(2000.0)
    assert bench.job_value(4, 100, 50.0) == pytest.approx(8000.0)  # weak scaling: all ranks' steps
