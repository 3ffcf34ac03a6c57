"""adamas_decode_step_static: the decode step for callers that cannot allocate
device memory where they decode (an allocator that must not be re-entered from
the decode loop, a hook that runs with allocation forbidden, a program that only
receives pointers to memory someone else owns).  It keeps its scratch in a fixed
array inside the library instead of a caller workspace.

Checked through the C ABI against adamas_decode_step on the same inputs, for two
calls in a row (the second call starts from the first call's leftovers in the
shared scratch), within the float tolerance the other parity tests use.  This
file is collected last so that a failure here stops a -x run only after every
other test has run."""
import ctypes

import numpy as np
import pytest
import torch

from compressed_sparse_kv_fp32_b200 import adamas, synth
from helpers import MAX_ABS, REL_RMS, assert_close_out, dev, dev_bf16

pytestmark = pytest.mark.gpu


def _inputs(w):
    inp = synth.make_inputs(w)
    K, V = dev_bf16(inp["K"]), dev_bf16(inp["V"])
    codes = torch.empty(K.shape[:-1] + (32,), dtype=torch.uint8, device="cuda")
    adamas.encode_keys(K, codes)
    return inp, K, V, codes


def _static_call(lib, q, codes, K, V, lens, budget, out, idx):
    B, Hq, d = q.shape
    _, Hkv, N, _ = K.shape
    return lib.adamas_decode_step_static(q.data_ptr(), codes.data_ptr(), K.data_ptr(), V.data_ptr(),
                                         lens.data_ptr(), B, Hq, Hkv, N, d, budget, out.data_ptr(),
                                         idx.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("wid,kw,budget", [(2, dict(Hq=8, Hkv=8, Nmax=20000), 256),
                                           (4, dict(B=3, Nmax=5000, len_range=(100, 5000)), 64),
                                           # G = 8 over 200K tokens: the distances spill into the scratch
                                           (5, dict(B=1, Hq=8, Hkv=1, Nmax=200000, len_range=None), 512)])
def test_matches_workspace_entry_point_twice(wid, kw, budget):
    lib = adamas.load()
    w = synth.WORKLOADS[wid].scaled(**kw)
    inp, K, V, codes = _inputs(w)
    lens = dev(inp["lens"])
    ws = adamas.Workspace(w.B, w.Hq, w.Hkv, w.Nmax, budget)  # the static call checks its own 4 MiB bound
    for step in (0, 1):                      # two calls in a row on the shared scratch
        q = dev_bf16(synth.query(w, step))
        ref_out, ref_idx = adamas.decode_step(q, codes, K, V, lens, budget, ws)
        out = torch.full((w.B, w.Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
        idx = torch.full((w.B, w.Hq, budget), -7, dtype=torch.int32, device="cuda")
        assert _static_call(lib, q, codes, K, V, lens, budget, out, idx) == 0
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), ref_idx.cpu().numpy())
        assert_close_out(out.cpu().numpy(), ref_out.cpu().numpy())
        word = ctypes.c_uint32(7)
        assert lib.adamas_static_device_error(ctypes.byref(word), torch.cuda.current_stream().cuda_stream) == 0
        assert word.value == 0


def test_device_errors_of_the_static_path_can_be_read_back():
    lib = adamas.load()
    w = synth.WORKLOADS[2].scaled(Hq=2, Hkv=2, Nmax=3000)
    inp, K, V, codes = _inputs(w)
    q = dev_bf16(inp["q"])
    out = torch.empty((1, 2, 128), dtype=torch.float32, device="cuda")
    idx = torch.empty((1, 2, 64), dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    word = ctypes.c_uint32(0)
    bad = dev(np.array([w.Nmax + 5], np.int32))      # beyond the cache: clamped and flagged
    assert _static_call(lib, q, codes, K, V, bad, 64, out, idx) == 0
    rc = lib.adamas_static_device_error(ctypes.byref(word), st)
    assert rc == -5 and word.value & adamas.DEVERR_SEQLEN  # ADAMAS_ERR_DEVICE
    good = dev(np.array([w.Nmax], np.int32))          # the next call clears the word
    assert _static_call(lib, q, codes, K, V, good, 64, out, idx) == 0
    assert lib.adamas_static_device_error(ctypes.byref(word), st) == 0 and word.value == 0


def test_sizes_beyond_the_fixed_scratch_are_rejected():
    lib = adamas.load()
    # 1M-token context over 8 kv heads needs far more than 4 MiB of scratch
    need = adamas.workspace_bytes(1, 24, 8, 1 << 20, 1024)
    assert need > 4 << 20
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced: the call fails its size check first
    rc = lib.adamas_decode_step_static(fake, fake, fake, fake, fake, 1, 24, 8, 1 << 20, 128, 1024,
                                       fake, fake, None)
    assert rc == -3
    assert "workspace" in adamas.status_string(rc)
    assert (MAX_ABS, REL_RMS) == (1e-2, 1e-3)
