"""GPU decode step against the CPU oracle, through the C ABI.

Selected indices must be identical (same (D, index) order, -1 padding); the fp32
output must lie within max-abs 1e-2 / relative-RMS 1e-3 of the oracle's float64
attention over the same rows.

Method: ADAMAS long-context sparse attention article (lnwmold.com/news/826806),
§2.1-§2.3 (rotation, bucketing, L1 scoring), §5.2 (token budget)."""
import numpy as np
import pytest
import torch

from compressed_sparse_kv_fp32_b200 import adamas, synth
from helpers import assert_close_out, dev, dev_bf16

pytestmark = pytest.mark.gpu


class Gpu:
    """Device copy of one workload's inputs with its codes encoded on the GPU."""

    def __init__(self, inp, budget_max):
        self.K = dev_bf16(inp["K"])
        self.V = dev_bf16(inp["V"])
        B, Hkv, N, _ = self.K.shape
        self.codes = torch.empty((B, Hkv, N, 32), dtype=torch.uint8, device="cuda")
        adamas.encode_keys(self.K, self.codes)
        self.Hq = inp["q"].shape[1]
        self.ws = adamas.Workspace(B, self.Hq, Hkv, N, budget_max)

    def step(self, q_u16, lens, budget):
        out, idx = adamas.decode_step(dev_bf16(q_u16), self.codes, self.K, self.V,
                                      dev(np.asarray(lens, np.int32)), budget, self.ws)
        torch.cuda.synchronize()
        return out.cpu().numpy(), idx.cpu().numpy()


def compare(orc, inp, lens, budget, gpu=None, nthreads=8):
    g = gpu or Gpu(inp, budget)
    out, idx = g.step(inp["q"], lens, budget)
    codes = orc.encode(inp["K"])
    want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, lens, budget,
                                            nthreads=nthreads)
    assert np.array_equal(idx, want_idx)
    assert_close_out(out, want_out)
    assert g.ws.device_error() == 0
    return out, idx


TINY = [
    # B, Hq, Hkv, Nmax, lens, budget
    (1, 1, 1, 64, [64], 8),
    (1, 1, 1, 64, [64], 64),
    (1, 1, 1, 64, [64], 100),
    (1, 1, 1, 64, [1], 4),
    (1, 1, 1, 64, [0], 4),
    (2, 4, 2, 50, [50, 13], 16),
    (3, 6, 3, 40, [0, 40, 7], 5),
    (2, 2, 2, 33, [33, 0], 0),
    (1, 8, 1, 300, [300], 17),
    (4, 12, 4, 129, [129, 1, 128, 64], 32),
    (1, 3, 1, 2048, [2047], 2048),
    # 16 blocks per head, one head shorter than the cluster (blocks without tokens)
    (2, 2, 2, 40000, [5, 40000], 16),
    (1, 1, 1, 40000, [39999], 3000),
    # distances too many for shared memory: they go through the workspace
    (1, 8, 1, 200000, [200000], 512),
    # budgets above the kept-list capacity (4096 tokens): the selection falls back to its
    # two in-order scans, in windows of 4096 kept tokens
    (1, 32, 32, 40000, [40000], 8000),
    (1, 64, 32, 20000, [20000], 10000),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,lens,budget", TINY)
def test_tiny(orc, B, Hq, Hkv, N, lens, budget):
    w = synth.WORKLOADS[4].scaled(B=B, Hq=Hq, Hkv=Hkv, Nmax=N, len_range=None, n_needles=2)
    inp = synth.make_inputs(w)
    compare(orc, inp, np.array(lens, np.int32), budget)


def test_all_equal_keys_tie_to_lowest_index(orc):
    w = synth.WORKLOADS[2].scaled(Hq=2, Hkv=2, Nmax=5000)
    inp = synth.make_inputs(w)
    inp["K"][:] = inp["K"][:, :, :1]                 # every token has the same codes
    _, idx = compare(orc, inp, inp["lens"], 300)
    assert (idx[0, :, :] == np.arange(300)).all()


def test_heavy_ties_across_blocks(orc):
    # few distinct key codes over a context split across many blocks
    w = synth.WORKLOADS[2].scaled(Hq=3, Hkv=3, Nmax=40000)
    inp = synth.make_inputs(w)
    r = np.random.default_rng(5)
    pool = inp["K"][:, :, :6].copy()
    pick = r.integers(0, 6, size=w.Nmax)
    inp["K"][:] = pool[:, :, pick]
    compare(orc, inp, inp["lens"], 1000)


def test_single_head_4k_needles(orc):
    w = synth.WORKLOADS[1]
    inp = synth.make_inputs(w)
    _, idx = compare(orc, inp, inp["lens"], 64)
    assert set(synth.needle_positions(w, 0, 0, w.Nmax).tolist()) <= set(idx[0, 0].tolist())


@pytest.mark.parametrize("budget", [128, 256, 1024])
def test_mha32_32k(orc, budget):
    w = synth.WORKLOADS[2]
    inp = synth.make_inputs(w)
    compare(orc, inp, inp["lens"], budget)


def test_mha32_32k_fresh_queries_share_one_workspace(orc):
    w = synth.WORKLOADS[2]
    inp = synth.make_inputs(w)
    g = Gpu(inp, 256)
    codes = orc.encode(inp["K"])
    for step in (1, 2, 10):
        q = synth.query(w, step)
        out, idx = g.step(q, inp["lens"], 256)
        want_out, want_idx, _ = orc.decode_step(q, inp["K"], inp["V"], codes, inp["lens"], 256, nthreads=8)
        assert np.array_equal(idx, want_idx)
        assert_close_out(out, want_out)


def test_gqa_batch8_ragged_full(orc):
    w = synth.WORKLOADS[4]
    inp = synth.make_inputs(w)
    _, idx = compare(orc, inp, inp["lens"], 256)
    for b in range(w.B):
        for g in range(w.Hkv):
            pos = synth.needle_positions(w, b, g, int(inp["lens"][b]))
            for p, h in zip(pos, synth.needle_targets(w, g)):
                assert p in idx[b, h]


def test_repeat_is_bitwise_deterministic(orc):
    w = synth.WORKLOADS[4].scaled(B=2, Nmax=6000, len_range=(3000, 6000))
    inp = synth.make_inputs(w)
    g = Gpu(inp, 256)
    a = g.step(inp["q"], inp["lens"], 256)
    b = g.step(inp["q"], inp["lens"], 256)
    assert np.array_equal(a[0].view(np.uint32), b[0].view(np.uint32))
    assert np.array_equal(a[1], b[1])


def test_sequence_length_beyond_cache_is_clamped_and_flagged(orc):
    w = synth.WORKLOADS[2].scaled(Hq=2, Hkv=2, Nmax=500)
    inp = synth.make_inputs(w)
    g = Gpu(inp, 16)
    out, idx = g.step(inp["q"], [900], 16)
    assert g.ws.device_error() == adamas.DEVERR_SEQLEN
    codes = orc.encode(inp["K"])
    want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, [500], 16)
    assert np.array_equal(idx, want_idx)
    assert_close_out(out, want_out)
    g.ws.reset()
    assert g.ws.device_error() == 0


def test_workspace_too_small_is_rejected():
    w = synth.WORKLOADS[2].scaled(Hq=2, Hkv=2, Nmax=64)
    inp = synth.make_inputs(w)
    g = Gpu(inp, 8)
    g.ws.nbytes = 64
    with pytest.raises(adamas.AdamasError) as e:
        g.step(inp["q"], inp["lens"], 8)
    assert e.value.status == -3


def test_graph_capture_replays(orc):
    w = synth.WORKLOADS[2].scaled(Hq=4, Hkv=4, Nmax=8192)
    inp = synth.make_inputs(w)
    g = Gpu(inp, 128)
    q = dev_bf16(inp["q"])
    lens = dev(inp["lens"])
    out = torch.empty((1, 4, 128), dtype=torch.float32, device="cuda")
    idx = torch.empty((1, 4, 128), dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        adamas.decode_step(q, g.codes, g.K, g.V, lens, 128, g.ws, out, idx)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        adamas.decode_step(q, g.codes, g.K, g.V, lens, 128, g.ws, out, idx)
    out.zero_()
    idx.zero_()
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    codes = orc.encode(inp["K"])
    want_out, want_idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, inp["lens"], 128)
    assert np.array_equal(idx.cpu().numpy(), want_idx)
    assert_close_out(out.cpu().numpy(), want_out)


# ---------------------------------------------------------------- full-size workloads, sampled heads
def _full_on_device(w, layer=0):
    K = torch.empty((w.B, w.Hkv, w.Nmax, 128), dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    for b in range(w.B):
        for h in range(w.Hkv):
            k, v = synth.head_kv(w, b, h, layer)
            K[b, h] = dev_bf16(k)
            V[b, h] = dev_bf16(v)
    return K, V


def _sampled_oracle(orc, w, q, lens, budget, b, kvh):
    k, v = synth.head_kv(w, b, kvh)
    L = int(lens[b])
    kc = orc.encode(k[:L])
    outs, idxs = [], []
    for g in range(w.G):
        h = kvh * w.G + g
        qc = orc.encode(q[b, h])
        D = orc.distance(qc, kc)
        idx = orc.select(D, budget)
        outs.append(orc.attend(q[b, h], k, v, idx))
        idxs.append(idx)
    return np.stack(outs), np.stack(idxs)


@pytest.mark.parametrize("wid,budget,heads", [(3, 1024, [(0, 0), (0, 13), (0, 31)]),
                                              (3, 64, [(0, 7)]),
                                              (3, 128, [(0, 21)]),
                                              (5, 1024, [(0, 5)])])
def test_full_size_sampled_heads(orc, wid, budget, heads):
    w = synth.WORKLOADS[wid]
    K, V = _full_on_device(w)
    codes = torch.empty((w.B, w.Hkv, w.Nmax, 32), dtype=torch.uint8, device="cuda")
    adamas.encode_keys(K, codes)
    q = synth.query(w, 0)
    lens = synth.seq_lens(w)
    ws = adamas.Workspace(w.B, w.Hq, w.Hkv, w.Nmax, budget)
    out, idx = adamas.decode_step(dev_bf16(q), codes, K, V, dev(lens), budget, ws)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    out, idx = out.cpu().numpy(), idx.cpu().numpy()
    for b, kvh in heads:
        want_out, want_idx = _sampled_oracle(orc, w, q, lens, budget, b, kvh)
        hs = slice(kvh * w.G, (kvh + 1) * w.G)
        assert np.array_equal(idx[b, hs], want_idx)
        assert_close_out(out[b, hs], want_out)
        for p, h in zip(synth.needle_positions(w, b, kvh, int(lens[b])), synth.needle_targets(w, kvh)):
            assert p in idx[b, h]
    del K, V, codes
    torch.cuda.empty_cache()
