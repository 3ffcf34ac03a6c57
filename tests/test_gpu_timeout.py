"""The bounded waits of the decode step give up, flag the error and let the step end.

A test hook (adamas_debug_withhold_stage) makes the copy warp of every block skip
the bulk copy of one code stage, so that stage never arrives: the workers' wait
for it runs out after about a second, ADAMAS_DEVERR_TIMEOUT is set, and the launch
completes (no copy is left in flight, nothing is read out of bounds).  The call
must return, the error word must carry the timeout bit, and after the hook is
cleared the same workspace, reset, must give the oracle's results again."""
import time

import numpy as np
import pytest
import torch

from compressed_sparse_kv_fp32_b200 import adamas, synth
from helpers import assert_close_out, dev, dev_bf16

pytestmark = pytest.mark.gpu


def test_withheld_stage_times_out_and_the_step_recovers(orc):
    # 3000 tokens over 2 blocks: 2 stages per block, each ring buffer used once
    w = synth.WORKLOADS[2].scaled(Hq=1, Hkv=1, Nmax=3000)
    inp = synth.make_inputs(w)
    K, V, q = dev_bf16(inp["K"]), dev_bf16(inp["V"]), dev_bf16(inp["q"])
    codes = torch.empty((1, 1, w.Nmax, 32), dtype=torch.uint8, device="cuda")
    adamas.encode_keys(K, codes)
    lens = dev(inp["lens"])
    ws = adamas.Workspace(1, 1, 1, w.Nmax, 64)
    lib = adamas.load()
    lib.adamas_debug_withhold_stage(0)
    try:
        t0 = time.perf_counter()
        adamas.decode(q, codes, K, V, lens, 64, ws)
        torch.cuda.synchronize()
        waited = time.perf_counter() - t0
    finally:
        lib.adamas_debug_withhold_stage(-1)
    assert ws.device_error() & adamas.DEVERR_TIMEOUT
    assert 0.3 < waited < 60.0
    ws.reset()
    out, idx = adamas.decode(q, codes, K, V, lens, 64, ws)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], orc.encode(inp["K"]), inp["lens"], 64)
    assert np.array_equal(idx.cpu().numpy(), want_idx)
    assert_close_out(out.cpu().numpy(), want_out)
