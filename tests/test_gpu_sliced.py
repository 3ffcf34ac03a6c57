"""Long contexts over few kv heads: the plain decode step splits every (b, kv head)
into slices inside the GPU (the sequence-sharded kernels with in-launch slices and
a merge of the slices' softmax states), so that more clusters run.  The result is
the same step: indices identical to the oracle's, outputs within max-abs 1e-2 /
rel-RMS 1e-3, the appended key encoded by the launch, ties across slice
boundaries going to the lower index.

Method: ADAMAS long-context sparse attention article (lnwmold.com/news/826806),
§2.3 (L1 scoring), §5.2 (token budget), §3.1 (the cache grows by one row per token)."""
import numpy as np
import pytest
import torch

from compressed_sparse_kv_fp32_b200 import adamas, synth
from helpers import assert_close_out, dev, dev_bf16

pytestmark = pytest.mark.gpu


def _setup(B, Hq, Hkv, N, lens, seed, equal_keys=False):
    w = synth.WORKLOADS[4].scaled(B=B, Hq=Hq, Hkv=Hkv, Nmax=N, len_range=None, n_needles=3, seed=seed)
    inp = synth.make_inputs(w)
    inp["lens"] = np.asarray(lens, np.int32)
    if equal_keys:
        inp["K"][:] = inp["K"][:, :, :1]
    K, V = dev_bf16(inp["K"]), dev_bf16(inp["V"])
    codes = torch.empty(K.shape[:3] + (32,), dtype=torch.uint8, device="cuda")
    adamas.encode_keys(K, codes)
    return inp, K, V, codes


@pytest.mark.parametrize("B,Hq,Hkv,N,lens,budgets", [
    (1, 4, 2, 100000, [100000], (64, 1024, 4096)),
    (2, 3, 1, 70000, [70000, 65541], (256, 70000)),      # ragged; budget above the length: dense
    (1, 8, 1, 200000, [199999], (512,)),                 # G = 8
])
def test_sliced_step_matches_the_oracle(orc, B, Hq, Hkv, N, lens, budgets):
    inp, K, V, codes = _setup(B, Hq, Hkv, N, lens, seed=41)
    ocodes = orc.encode(inp["K"])
    q = dev_bf16(inp["q"])
    for budget in budgets:
        ws = adamas.Workspace(B, Hq, Hkv, N, budget)
        out, idx = adamas.decode_step(q, codes, K, V, dev(inp["lens"]), budget, ws)
        torch.cuda.synchronize()
        assert ws.device_error() == 0
        want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], ocodes, inp["lens"], budget)
        assert np.array_equal(idx.cpu().numpy(), want_idx), budget
        assert_close_out(out.cpu().numpy(), want_out)


def test_sliced_step_with_the_appended_key(orc):
    B, Hq, Hkv, N = 1, 2, 2, 90000
    inp, K, V, codes = _setup(B, Hq, Hkv, N, [N], seed=43)
    codes[:, :, N - 1] = 0                      # the newest key's code is written by the launch
    lens = dev(inp["lens"])
    ws = adamas.Workspace(B, Hq, Hkv, N, 1024)
    out, idx = adamas.decode_step_append(dev_bf16(inp["q"]), codes, K, V, lens, (lens - 1).to(torch.int32), 1024, ws)
    torch.cuda.synchronize()
    ocodes = orc.encode(inp["K"])
    assert np.array_equal(codes.cpu().numpy(), ocodes)
    want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], ocodes, inp["lens"], 1024)
    assert np.array_equal(idx.cpu().numpy(), want_idx)
    assert_close_out(out.cpu().numpy(), want_out)


def test_ties_across_slices_go_to_the_lower_index(orc):
    inp, K, V, codes = _setup(1, 2, 1, 80000, [80000], seed=47, equal_keys=True)
    ws = adamas.Workspace(1, 2, 1, 80000, 3000)
    out, idx = adamas.decode_step(dev_bf16(inp["q"]), codes, K, V, dev(inp["lens"]), 3000, ws)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy()[0, 0], np.arange(3000))
    want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], orc.encode(inp["K"]), inp["lens"], 3000)
    assert np.array_equal(idx.cpu().numpy(), want_idx)
    assert_close_out(out.cpu().numpy(), want_out)
