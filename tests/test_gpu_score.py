"""GPU distances (adamas_score) against the oracle: every L1 code distance must be equal.

Method: ADAMAS long-context sparse attention article (lnwmold.com/news/826806), §2.3."""
import numpy as np
import pytest
import torch

from compressed_sparse_kv_fp32_b200 import adamas, synth
from helpers import dev, dev_bf16, host_u16

pytestmark = pytest.mark.gpu


def run(w, lens=None):
    inp = synth.make_inputs(w)
    lens = inp["lens"] if lens is None else np.asarray(lens, np.int32)
    K = dev_bf16(inp["K"])
    codes = torch.empty(K.shape[:-1] + (32,), dtype=torch.uint8, device="cuda")
    adamas.encode_keys(K, codes)
    dist = adamas.score(dev_bf16(inp["q"]), codes, dev(lens))
    return inp, lens, host_u16(dist)


def oracle_dist(orc, inp, lens):
    codes = orc.encode(inp["K"])
    _, _, D = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, lens, budget=1, want_dist=True)
    return D


@pytest.mark.parametrize("wid,kw", [(1, {}), (2, dict(Hq=4, Hkv=4, Nmax=3000)),
                                    (4, dict(B=3, Nmax=2500, len_range=(1, 2500))),
                                    (5, dict(Nmax=1100, Hq=24, Hkv=8))])
def test_distances_equal(orc, wid, kw):
    w = synth.WORKLOADS[wid].scaled(**kw)
    inp, lens, got = run(w)
    want = oracle_dist(orc, inp, lens)
    for b in range(w.B):
        L = int(lens[b])
        assert np.array_equal(got[b, :, :L].astype(np.int32), want[b, :, :L])
        assert (got[b, :, L:] == 0xFFFF).all()


@pytest.mark.parametrize("G", [1, 2, 3, 5, 6, 7, 8])
def test_every_group_size(orc, G):
    w = synth.WORKLOADS[4].scaled(B=2, Hq=2 * G, Hkv=2, Nmax=777, len_range=(300, 777))
    inp, lens, got = run(w)
    want = oracle_dist(orc, inp, lens)
    for b in range(w.B):
        L = int(lens[b])
        assert np.array_equal(got[b, :, :L].astype(np.int32), want[b, :, :L])
