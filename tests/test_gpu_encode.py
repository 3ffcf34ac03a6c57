"""GPU key encoder against the CPU oracle: packed codes must be byte-identical.

Method: ADAMAS long-context sparse attention article (lnwmold.com/news/826806),
§2.1 Hadamard rotation, §2.2 dynamic bucketing, §3.1 packed code cache."""
import numpy as np
import pytest
import torch

from compressed_sparse_kv_fp32_b200 import adamas, synth
from helpers import dev, dev_bf16

pytestmark = pytest.mark.gpu


def gpu_encode(K_u16, pos_begin=None, count=None, codes=None):
    K = dev_bf16(K_u16)
    B, Hkv, N, _ = K.shape
    c = torch.zeros((B, Hkv, N, 32), dtype=torch.uint8, device="cuda") if codes is None else codes
    pb = None if pos_begin is None else dev(np.asarray(pos_begin, dtype=np.int32))
    adamas.encode_keys(K, c, pb, count)
    torch.cuda.synchronize()
    return c.cpu().numpy()


def special_vectors():
    bf = synth.bf16_round
    rows = [np.zeros(128, np.float32), np.ones(128, np.float32), -np.ones(128, np.float32)]
    rows += [np.eye(128, dtype=np.float32)[j] for j in (0, 1, 3, 64, 127)]
    rows.append(np.full(128, 1e-38, np.float32))               # subnormal after rotation
    rows.append(np.where(np.arange(128) % 2 == 0, 1.0, -1.0).astype(np.float32))
    x = np.zeros(128, np.float32)
    x[:2] = [1.0, 1.0]                                          # exact zeros and exact thresholds
    rows.append(x)
    r = np.random.default_rng(3)
    big = r.standard_normal(128).astype(np.float32)
    big[[5, 77]] *= 1000
    rows.append(big)
    rows.append(r.integers(-3, 4, 128).astype(np.float32))      # many exact ties in y
    return bf(np.stack(rows))


def test_special_vectors(orc):
    x = special_vectors()
    K = x[None, None]                                            # [1, 1, n, 128]
    got = gpu_encode(K)[0, 0]
    assert np.array_equal(got, orc.encode(x))


@pytest.mark.parametrize("n", [1, 127, 128, 129, 1000])
def test_ragged_counts(orc, n):
    r = np.random.default_rng(n)
    x = synth.bf16_round(r.standard_normal((2, 3, n, 128)).astype(np.float32) * 5)
    assert np.array_equal(gpu_encode(x), orc.encode(x))


def test_single_head_4k(orc):
    w = synth.WORKLOADS[1]
    K = synth.make_inputs(w)["K"]
    assert np.array_equal(gpu_encode(K), orc.encode(K))


def test_mha32_32k_full(orc):
    w = synth.WORKLOADS[2]
    K = np.stack([synth.head_kv(w, 0, h)[0] for h in range(w.Hkv)])[None]
    assert np.array_equal(gpu_encode(K), orc.encode(K))


def test_append_positions_only(orc):
    # encode [p_b, p_b + count) per sequence; everything else stays untouched
    r = np.random.default_rng(9)
    B, Hkv, N = 3, 2, 300
    x = synth.bf16_round(r.standard_normal((B, Hkv, N, 128)).astype(np.float32))
    start = np.array([0, 17, 299], dtype=np.int32)
    codes = torch.full((B, Hkv, N, 32), 0x5A, dtype=torch.uint8, device="cuda")
    got = gpu_encode(x, start, 5, codes)
    want = np.full((B, Hkv, N, 32), 0x5A, dtype=np.uint8)
    full = orc.encode(x)
    for b in range(B):
        lo, hi = int(start[b]), min(int(start[b]) + 5, N)
        want[b, :, lo:hi] = full[b, :, lo:hi]
    assert np.array_equal(got, want)


def test_append_negative_start_is_skipped(orc):
    r = np.random.default_rng(10)
    x = synth.bf16_round(r.standard_normal((1, 1, 8, 128)).astype(np.float32))
    codes = torch.zeros((1, 1, 8, 32), dtype=torch.uint8, device="cuda")
    got = gpu_encode(x, [-2], 4, codes)
    want = np.zeros((1, 1, 8, 32), np.uint8)
    want[0, 0, :2] = orc.encode(x[0, 0, :2])
    assert np.array_equal(got, want)


# ---- the prefill kernel (more than 8192 vectors per call): tiles of 32 rows per warp
def test_prefill_special_vectors_tiled(orc):
    x = special_vectors()
    r = np.random.default_rng(11)
    filler = synth.bf16_round(r.standard_normal((9000 - x.shape[0], 128)).astype(np.float32) * 3)
    K = np.concatenate([x, filler])[None, None]                  # [1, 1, 9000, 128]
    assert np.array_equal(gpu_encode(K)[0, 0], orc.encode(K[0, 0]))


@pytest.mark.parametrize("n,count,start", [(1000, 1000, [0, 0, 0]),
                                           (1000, 700, [0, 250, 900]),
                                           (777, 777, [5, -40, 700]),
                                           (2049, 1999, [1, 31, 33])])
def test_prefill_ragged_windows(orc, n, count, start):
    # 3 sequences x 5 kv heads, windows [start_b, start_b + count) clipped to [0, n);
    # counts that are not multiples of 32 leave partial tiles at every head's end
    r = np.random.default_rng(n + count)
    B, Hkv = 3, 5
    x = synth.bf16_round(r.standard_normal((B, Hkv, n, 128)).astype(np.float32) * 4)
    codes = torch.full((B, Hkv, n, 32), 0xA5, dtype=torch.uint8, device="cuda")
    got = gpu_encode(x, np.array(start, np.int32), count, codes)
    want = np.full((B, Hkv, n, 32), 0xA5, dtype=np.uint8)
    full = orc.encode(x)
    for b in range(B):
        lo, hi = max(0, start[b]), min(n, start[b] + count)
        if hi > lo:
            want[b, :, lo:hi] = full[b, :, lo:hi]
    assert np.array_equal(got, want)
