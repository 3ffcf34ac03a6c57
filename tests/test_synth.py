"""The seeded generator: bf16 rounding against torch's conversion, determinism and
the workload recipe (outliers, needles, lengths)."""
import numpy as np
import torch

from compressed_sparse_kv_fp32_b200 import synth


def test_bf16_round_matches_torch():
    r = np.random.default_rng(0)
    x = np.concatenate([r.standard_normal(100000).astype(np.float32) * 30,
                        np.array([0.0, -0.0, 1e-40, -1e-40, 3.4e38, 1.0 + 2**-8, 1.0 + 3 * 2**-8],
                                 dtype=np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.bf16_round(x), want)
    back = torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.array_equal(synth.bf16_to_f32(want), back)


def test_generation_is_deterministic_and_per_head():
    w = synth.WORKLOADS[2].scaled(Nmax=256, Hq=3, Hkv=3)
    a = synth.make_inputs(w)
    b = synth.make_inputs(w)
    for k in ("K", "V", "q", "lens"):
        assert np.array_equal(a[k], b[k])
    K1, V1 = synth.head_kv(w, 0, 1)
    assert np.array_equal(K1, a["K"][0, 1]) and np.array_equal(V1, a["V"][0, 1])
    assert not np.array_equal(a["K"][0, 0], a["K"][0, 1])


def test_outliers_and_needles():
    w = synth.WORKLOADS[3].scaled(Nmax=4096, Hq=2, Hkv=2)
    K, V = synth.head_kv(w, 0, 1)
    ch = synth.outlier_channels(w, 1)
    Kf, Vf = synth.bf16_to_f32(K), synth.bf16_to_f32(V)
    other = np.setdiff1d(np.arange(128), ch)
    assert Kf[:, ch].std() > 10 * Kf[:, other].std() / 2
    assert Vf[:, ch].std() > 10 * Vf[:, other].std() / 2      # workloads 2-5: K and V
    pos = synth.needle_positions(w, 0, 1, 4096)
    assert len(set(pos.tolist())) == w.n_needles
    assert pos.min() >= 0 and pos.max() < 4096
    qs = synth.bf16_to_f32(synth.bf16_round(synth.needle_query_f32(w, 0, 1)))
    assert np.abs(Kf[pos[0]] - 2 * qs).max() < 1.0


def test_lengths_of_gqa_batch():
    lens = synth.seq_lens(synth.WORKLOADS[4])
    assert lens.shape == (8,) and lens.min() >= 16384 and lens.max() <= 32768
    assert (synth.seq_lens(synth.WORKLOADS[3]) == 131072).all()


def test_queries_alternate_needle_and_fresh():
    w = synth.WORKLOADS[2].scaled(Nmax=64, Hq=2, Hkv=2)
    q0, q1, q10 = synth.query(w, 0), synth.query(w, 1), synth.query(w, 10)
    assert np.array_equal(q0, q10) and not np.array_equal(q0, q1)
