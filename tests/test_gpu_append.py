"""Fused append + decode step against the two-launch sequence and the oracle.

adamas_decode_step_append encodes the key at append_pos[b] into the code cache
and runs the decode step over the cache in one launch.  Its codes, indices and
output must be bit-identical to adamas_encode_keys of that one position followed
by adamas_decode_step, and its indices equal to the oracle's.

Method: ADAMAS long-context sparse attention article (lnwmold.com/news/826806),
§3.1 (the code cache grows by one row per generated token), §2.3 and §5.2 (the
step scores and selects over the whole cache)."""
import numpy as np
import pytest
import torch

from compressed_sparse_kv_fp32_b200 import adamas, synth
from helpers import assert_close_out, dev, dev_bf16, host_u16  # noqa: F401

pytestmark = pytest.mark.gpu

CASES = [
    # B, Hq, Hkv, Nmax, lens, append_pos, budget
    (1, 1, 1, 64, [64], [63], 8),            # the last token of the sequence
    (2, 4, 2, 50, [50, 13], [10, 12], 16),   # inside the sequence
    (2, 4, 2, 50, [40, 13], [45, -1], 16),   # past the sequence (encoded, not scored); none
    (3, 6, 3, 40, [0, 40, 7], [0, 39, 50], 5),  # empty sequence; out-of-range position
    (1, 8, 1, 3000, [3000], [2047], 64),     # first row of the second stage
    (2, 2, 2, 40000, [5, 40000], [4, 20001], 16),  # a middle block of the cluster
    (1, 1, 1, 40000, [39999], [39998], 0),   # budget 0: appended, nothing scored
    (1, 8, 1, 200000, [200000], [199999], 512),  # distances in the workspace
]


@pytest.mark.parametrize("B,Hq,Hkv,N,lens,apos,budget", CASES)
def test_append_matches_two_launches(orc, B, Hq, Hkv, N, lens, apos, budget):
    w = synth.WORKLOADS[4].scaled(B=B, Hq=Hq, Hkv=Hkv, Nmax=N, len_range=None, n_needles=2)
    inp = synth.make_inputs(w)
    K, V, q = dev_bf16(inp["K"]), dev_bf16(inp["V"]), dev_bf16(inp["q"])
    seq = dev(np.asarray(lens, np.int32))
    ap = dev(np.asarray(apos, np.int32))
    ws = adamas.Workspace(B, Hq, Hkv, N, budget)

    full = torch.empty((B, Hkv, N, 32), dtype=torch.uint8, device="cuda")
    adamas.encode_keys(K, full)
    # the cache before the step: the appended rows hold stale bytes
    stale = full.clone()
    for b, a in enumerate(apos):
        if 0 <= a < N:
            stale[b, :, a] = 0xA5

    ref_codes = stale.clone()
    adamas.encode_keys(K, ref_codes, pos_begin=ap.clamp(0, N - 1), count=1)
    for b, a in enumerate(apos):  # positions out of range append nothing
        if not 0 <= a < N:
            ref_codes[b] = stale[b]
    ref_out, ref_idx = adamas.decode_step(q, ref_codes, K, V, seq, budget, ws)

    codes = stale.clone()
    out, idx = adamas.decode_step_append(q, codes, K, V, seq, ap, budget, ws)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    assert torch.equal(codes, ref_codes)
    assert torch.equal(idx, ref_idx)
    assert torch.equal(out.view(torch.int32), ref_out.view(torch.int32))

    if all(0 <= a < N for a in apos):
        assert torch.equal(codes, full)
    # against the oracle: the appended rows are the freshly encoded ones
    want_codes = orc.encode(inp["K"])
    lens_np = np.asarray(lens, np.int32)
    for b, a in enumerate(apos):
        if not 0 <= a < N:
            want_codes[b] = stale[b].cpu().numpy()
    assert np.array_equal(codes.cpu().numpy(), want_codes)
    want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], want_codes, lens_np, budget,
                                            nthreads=8)
    assert np.array_equal(idx.cpu().numpy(), want_idx)
    assert_close_out(out.cpu().numpy(), want_out)


def test_append_rejects_missing_positions():
    w = synth.WORKLOADS[4].scaled(B=1, Hq=1, Hkv=1, Nmax=64, len_range=None, n_needles=2)
    inp = synth.make_inputs(w)
    K, V, q = dev_bf16(inp["K"]), dev_bf16(inp["V"]), dev_bf16(inp["q"])
    codes = torch.zeros((1, 1, 64, 32), dtype=torch.uint8, device="cuda")
    ws = adamas.Workspace(1, 1, 1, 64, 8)
    rc = adamas.load().adamas_decode_step_append(
        q.data_ptr(), codes.data_ptr(), K.data_ptr(), V.data_ptr(), dev(np.array([64], np.int32)).data_ptr(),
        None, 1, 1, 1, 64, 128, 8, torch.empty((1, 1, 128), device="cuda").data_ptr(),
        torch.empty((1, 1, 8), dtype=torch.int32, device="cuda").data_ptr(), ws.buffer.data_ptr(), ws.nbytes, None)
    assert rc == -1  # ADAMAS_ERR_INVALID_ARG
