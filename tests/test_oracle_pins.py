"""Pins for the CPU oracle, checked against what the method and the mathematics fix.

Each check ties the oracle to something other than itself: closed forms of the
Sylvester-Hadamard rotation, a library Hadamard matrix (scipy) in float64, hand
built boundary values of the bucketing rule, brute force over every byte pair of
the packed L1 distance, Python's sorted() for the token budget, and torch's
scaled_dot_product_attention in float64 for the attention step.

Method: ADAMAS long-context sparse attention article (lnwmold.com/news/826806),
§2.1 (Hadamard rotation), §2.2 (dynamic bucketing), §2.3 (Manhattan distance),
§3.1 (packed code cache), §5.2 (token budget).
"""
import numpy as np
import pytest
import scipy.linalg
import torch

from compressed_sparse_kv_fp32_b200 import synth

C = np.uint32(0x3DB504F3).view(np.float32)          # RN_fp32(1/sqrt(128))
U = 2.0 ** -24                                         # fp32 unit roundoff
H128 = scipy.linalg.hadamard(128).astype(np.float64)   # Sylvester order, library routine


def popc(x):
    return bin(int(x)).count("1")


def unpack(packed):
    """2-bit fields of packed bytes, first code in the top bits (§3.1 shift pattern)."""
    p = np.asarray(packed, dtype=np.uint8)
    f = np.stack([(p >> 6) & 3, (p >> 4) & 3, (p >> 2) & 3, p & 3], axis=-1)
    return f.reshape(p.shape[:-1] + (p.shape[-1] * 4,)).astype(np.int64)


def bf16(x):
    return synth.bf16_round(np.asarray(x, dtype=np.float32))


def random_vectors(n, seed, outliers=True):
    r = np.random.default_rng(seed)
    x = r.standard_normal((n, 128)).astype(np.float32)
    if outliers:
        ch = r.choice(128, 4, replace=False)
        x[:, ch] *= 20
    return bf16(x)


# ----------------------------------------------------------------- rotation
def test_constant_is_rounded_inverse_sqrt128():
    assert np.float32(1 / np.sqrt(np.float64(128))) == C
    assert abs(np.float64(C) - 1 / np.sqrt(128.0)) <= U * (1 / np.sqrt(128.0))


def test_rotation_of_basis_vectors_is_signed_constant(orc):
    # FWHT(e_j)[i] = C * (-1)^popcount(i & j), exactly (closed form of Sylvester H)
    eye = bf16(np.eye(128, dtype=np.float32))
    y = orc.rotate(eye)
    for j in range(128):
        want = np.array([C if popc(i & j) % 2 == 0 else -C for i in range(128)], dtype=np.float32)
        assert np.array_equal(y[j], want), j


def test_rotation_is_orthonormal(orc):
    M = orc.rotate(bf16(np.eye(128, dtype=np.float32))).astype(np.float64)
    assert np.abs(M @ M.T - np.eye(128)).max() < 4 * U
    # same matrix as the library Sylvester matrix, scaled
    assert np.abs(M - H128 / np.sqrt(128.0)).max() <= U


def test_rotation_of_all_bf16_scalars(orc):
    # x = v e_0: every butterfly adds or subtracts an exact zero, so y_i = RN(v * C):
    # pins the bf16 decode on every non-NaN bit pattern
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    keep = np.isfinite(vals) & (bits != 0x8000)          # -0 + 0 = +0 loses the sign
    bits, vals = bits[keep], vals[keep]
    x = np.zeros((bits.size, 128), dtype=np.uint16)
    x[:, 0] = bits
    y = orc.rotate(x)
    want = (vals * C).astype(np.float32)
    assert np.array_equal(y[:, 0].view(np.uint32), want.view(np.uint32))
    assert np.array_equal(y[:, 77].view(np.uint32), want.view(np.uint32))


def test_rotation_matches_library_hadamard(orc):
    x = random_vectors(2000, 1)
    xf = synth.bf16_to_f32(x).astype(np.float64)
    y = orc.rotate(x).astype(np.float64)
    exact = xf @ H128 / np.sqrt(128.0)                  # H symmetric: x @ H == H x
    bound = 9 * U * np.abs(xf).sum(axis=1, keepdims=True) / np.sqrt(128.0) + 1e-30
    assert (np.abs(y - exact) <= bound).all()


def test_rotation_preserves_inner_products(orc):
    # (HQ)(HK)^T = QK^T, §2.1, within the fp32 rounding of the butterfly
    q, k = random_vectors(500, 2), random_vectors(500, 3)
    qf, kf = (synth.bf16_to_f32(v).astype(np.float64) for v in (q, k))
    yq, yk = (orc.rotate(v).astype(np.float64) for v in (q, k))
    lhs = (yq * yk).sum(1)
    rhs = (qf * kf).sum(1)
    bound = 2 * 128 * 7 * U * np.linalg.norm(qf, axis=1) * np.linalg.norm(kf, axis=1)
    assert (np.abs(lhs - rhs) <= bound).all()


def _butterfly_f32(x_bits, widths):
    """NumPy float32 restatement of the rotation: one elementwise add/subtract per
    butterfly stage over the whole batch, stage widths in the given order, then one
    multiply by C (NumPy float32 arithmetic rounds to nearest and never fuses)."""
    y = synth.bf16_to_f32(x_bits).astype(np.float32).copy()
    idx = np.arange(128)
    for h in widths:
        lo = idx[(idx & h) == 0]
        a, b = y[:, lo].copy(), y[:, lo + h].copy()
        y[:, lo] = a + b
        y[:, lo + h] = a - b
    return y * C


def _codes_f32(y):
    """Bucketing and MSB-first packing of float32 rotated rows, restated in NumPy."""
    m = np.abs(y).max(1, keepdims=True)
    c = (3 - (y < -0.5 * m).astype(np.int64) - (y < 0).astype(np.int64)
         - (y < 0.5 * m).astype(np.int64)).reshape(y.shape[0], 32, 4)
    return (c[..., 0] << 6 | c[..., 1] << 4 | c[..., 2] << 2 | c[..., 3]).astype(np.uint8)


def test_rotation_stage_order_is_ascending_bit_for_bit(orc):
    # The fp32 rounding sequence is part of the contract (codes are reproducible bit for
    # bit): widths 1, 2, ..., 64 ascending, no fused multiply-add, one final multiply by C.
    # Bounds alone cannot see the stage order, so an independent float32 restatement must
    # agree on every bit of every rotated value and every code byte, and the reversed
    # order must give other bits on many vectors, which shows that this check can tell
    # the orders apart (codes move only where a value lands on a threshold, so they
    # rarely differ).
    x = np.concatenate([random_vectors(10000, 21), random_vectors(10000, 22, outliers=False)])
    want = _butterfly_f32(x, [1, 2, 4, 8, 16, 32, 64])
    got = orc.rotate(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    assert np.array_equal(orc.encode(x), _codes_f32(want))
    rev = _butterfly_f32(x, [64, 32, 16, 8, 4, 2, 1])
    differ = (rev.view(np.uint32) != got.view(np.uint32)).any(axis=1)
    assert differ.sum() > 100


def test_rotation_spreads_outliers(orc):
    # qualitative claim of §2.1: the rotation flattens outlier channels
    x = random_vectors(1000, 4)
    xf = synth.bf16_to_f32(x)
    y = orc.rotate(x)
    assert np.abs(y).max(1).mean() < 0.5 * np.abs(xf).max(1).mean()


# ----------------------------------------------------------------- bucketing and packing
def test_codes_of_basis_vectors(orc):
    # y = +-C with m = C: +C >= C/2 -> 3, -C < -C/2 -> 0
    codes = unpack(orc.encode(bf16(np.eye(128, dtype=np.float32))))
    for j in range(128):
        want = [3 if popc(i & j) % 2 == 0 else 0 for i in range(128)]
        assert codes[j].tolist() == want


def test_codes_of_all_ones(orc):
    # FWHT(1) = 128 C e_0; y_0 = m -> 3; y_i = 0 is not < 0 and is < m/2 -> 2
    packed = orc.encode(bf16(np.ones((1, 128), dtype=np.float32)))[0]
    assert packed[0] == (3 << 6 | 2 << 4 | 2 << 2 | 2) == 0xEA
    assert (packed[1:] == 0xAA).all()


def test_pack_order_first_code_in_top_bits(orc):
    y = np.zeros((1, 128), dtype=np.float32)
    y[0, :4] = [-3.0, -1.0, 1.0, 3.0]
    y[0, 4] = 4.0                                          # m = 4, thresholds -2, 0, 2
    packed = orc.bucket_pack(y)[0]
    assert packed[0] == 0b00_01_10_11


def test_bucket_threshold_boundaries(orc):
    f = np.float32
    y = np.full((1, 128), 1.0, dtype=np.float32)           # filler -> code 2
    y[0, 0] = 4.0                                          # m = 4 -> 3
    y[0, 1] = -2.0                                         # == -m/2: not below -> 1
    y[0, 2] = np.nextafter(f(-2.0), f(-10.0))              # just below -m/2 -> 0
    y[0, 3] = -0.0                                         # -0 is not < 0 -> 2
    y[0, 4] = 0.0                                          # -> 2
    y[0, 5] = 2.0                                          # == m/2 -> 3
    y[0, 6] = np.nextafter(f(2.0), f(0.0))                 # just below m/2 -> 2
    y[0, 7] = -1e-30                                       # tiny negative -> 1
    y[0, 8] = -4.0                                         # -> 0
    y[0, 9] = np.nextafter(f(0.0), f(1.0))                 # smallest subnormal -> 2
    codes = unpack(orc.bucket_pack(y))[0]
    assert codes[:10].tolist() == [3, 1, 0, 2, 2, 3, 2, 1, 0, 2]
    assert (codes[10:] == 2).all()


def test_bucket_absmax_uses_magnitude(orc):
    y = np.zeros((1, 128), dtype=np.float32)
    y[0, 0] = -8.0                                         # m = 8 from a negative value
    y[0, 1] = 3.0                                          # 3 < 4 -> 2 (would be 3 if m were 3)
    y[0, 2] = -3.9                                         # -3.9 >= -4 -> 1
    codes = unpack(orc.bucket_pack(y))[0]
    assert codes[:3].tolist() == [0, 2, 1]


def test_zero_vector_codes_are_all_three(orc):
    packed = orc.encode(np.zeros((1, 128), dtype=np.uint16))
    assert (packed == 0xFF).all()


def test_codes_match_float64_library_rotation(orc):
    # codes from a float64 rotation with the library Hadamard matrix agree except
    # where a value sits within the fp32 rounding of a threshold
    x = random_vectors(5000, 5)
    xf = synth.bf16_to_f32(x).astype(np.float64)
    y = xf @ H128 / np.sqrt(128.0)
    m = np.abs(y).max(1, keepdims=True)
    want = (y >= -0.5 * m).astype(int) + (y >= 0).astype(int) + (y >= 0.5 * m).astype(int)
    got = unpack(orc.encode(x))
    tol = 16 * U * np.abs(xf).sum(1, keepdims=True) / np.sqrt(128.0)
    near = (np.abs(y + 0.5 * m) < tol) | (np.abs(y) < tol) | (np.abs(y - 0.5 * m) < tol)
    assert ((got == want) | near).all()
    assert (got == want).mean() > 0.9999


# ----------------------------------------------------------------- distance
def test_distance_all_byte_pairs(orc):
    # L1 over the four 2-bit fields of every pair of packed bytes
    fields = unpack(np.arange(256, dtype=np.uint8)[:, None])            # [256, 4]
    want = np.abs(fields[:, None, :] - fields[None, :, :]).sum(-1)      # [256, 256]
    keys = np.zeros((256, 32), dtype=np.uint8)
    keys[:, 5] = np.arange(256)
    for a in range(256):
        q = np.zeros(32, dtype=np.uint8)
        q[5] = a
        assert np.array_equal(orc.distance(q, keys), want[a]), a


def test_distance_between_hadamard_rows(orc):
    # codes of e_j are 3/0 by sign; rows j != k differ in 64 signs -> 64 * 3 = 192
    codes = orc.encode(bf16(np.eye(128, dtype=np.float32)))
    for j in (0, 1, 5, 64, 127):
        D = orc.distance(codes[j], codes)
        assert D[j] == 0
        assert (np.delete(D, j) == 192).all()


def test_distance_metric_properties(orc):
    r = np.random.default_rng(6)
    codes = r.integers(0, 256, size=(200, 32), dtype=np.uint8)
    Dm = np.stack([orc.distance(codes[i], codes) for i in range(200)])
    assert (np.diag(Dm) == 0).all() and np.array_equal(Dm, Dm.T)
    assert Dm.max() <= 384 and Dm.min() >= 0
    i, j, k = r.integers(0, 200, size=(3, 2000))
    assert (Dm[i, k] <= Dm[i, j] + Dm[j, k]).all()


# ----------------------------------------------------------------- select
@pytest.mark.parametrize("n", [0, 1, 7, 33, 64])
def test_select_brute_force_with_ties(orc, n):
    r = np.random.default_rng(100 + n)
    D = r.integers(0, 5, size=n).astype(np.int32)         # heavy ties
    order = sorted(range(n), key=lambda t: (D[t], t))
    for k in sorted({0, 1, n // 2, n, n + 5}):
        got = orc.select(D, k)
        want = (order + [-1] * k)[:k]
        assert got.tolist() == want, (n, k)


def test_select_returns_every_token_when_budget_covers_context(orc):
    D = np.random.default_rng(7).integers(0, 385, size=50).astype(np.int32)
    idx = orc.select(D, 50)
    assert sorted(idx.tolist()) == list(range(50))
    assert (np.diff(D[idx]) >= 0).all()


# ----------------------------------------------------------------- attention
def _dense_sdpa(q, K, V):
    qt = torch.from_numpy(synth.bf16_to_f32(q).astype(np.float64)).view(1, 1, 1, 128)
    kt = torch.from_numpy(synth.bf16_to_f32(K).astype(np.float64)).view(1, 1, -1, 128)
    vt = torch.from_numpy(synth.bf16_to_f32(V).astype(np.float64)).view(1, 1, -1, 128)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).view(128).numpy()


def test_attention_over_all_rows_is_dense_attention(orc):
    K, V = random_vectors(300, 8), random_vectors(300, 9)
    q = random_vectors(1, 10)[0]
    out = orc.attend(q, K, V, np.arange(300, dtype=np.int32))
    assert np.abs(out - _dense_sdpa(q, K, V)).max() < 1e-12


def test_attention_single_row_is_that_value_row(orc):
    K, V = random_vectors(10, 11), random_vectors(10, 12)
    q = random_vectors(1, 13)[0]
    out = orc.attend(q, K, V, np.array([6, -1, -1], dtype=np.int32))
    assert np.array_equal(out, synth.bf16_to_f32(V[6]).astype(np.float64))


def test_attention_ignores_row_order_and_padding(orc):
    K, V = random_vectors(64, 14), random_vectors(64, 15)
    q = random_vectors(1, 16)[0]
    sel = np.array([3, 17, 40, 41, 63], dtype=np.int32)
    a = orc.attend(q, K, V, sel)
    b = orc.attend(q, K, V, np.concatenate([sel[::-1], [-1, -1]]).astype(np.int32))
    assert np.abs(a - b).max() < 1e-13
    assert np.abs(a - _dense_sdpa(q, K[sel], V[sel])).max() < 1e-12


def test_attention_with_no_rows_is_zero(orc):
    K, V = random_vectors(4, 17), random_vectors(4, 18)
    assert (orc.attend(random_vectors(1, 19)[0], K, V, np.full(3, -1, np.int32)) == 0).all()


# ----------------------------------------------------------------- whole decode step
def test_decode_step_full_budget_is_dense_gqa_attention(orc):
    w = synth.WORKLOADS[4].scaled(B=2, Hq=4, Hkv=2, Nmax=64, len_range=(20, 64), n_needles=2)
    inp = synth.make_inputs(w)
    lens = np.array([64, 37], dtype=np.int32)
    codes = orc.encode(inp["K"])
    out, idx, dist = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, lens, budget=80,
                                     nthreads=3, want_dist=True)
    for b in range(2):
        L = int(lens[b])
        for h in range(4):
            g = h // 2
            ref = _dense_sdpa(inp["q"][b, h], inp["K"][b, g, :L], inp["V"][b, g, :L])
            assert np.abs(out[b, h] - ref).max() < 1e-12
            sel = idx[b, h]
            assert sorted(sel[:L].tolist()) == list(range(L)) and (sel[L:] == -1).all()
            qc = orc.encode(inp["q"][b, h])
            D = orc.distance(qc, codes[b, g, :L])
            assert np.array_equal(dist[b, h, :L], D) and (dist[b, h, L:] == -1).all()
            keys = [(D[t], t) for t in sel[:L]]
            assert keys == sorted(keys)


def test_decode_step_threads_do_not_change_results(orc):
    w = synth.WORKLOADS[2].scaled(Hq=6, Hkv=6, Nmax=512)
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    a = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, inp["lens"], 32, nthreads=1)
    b = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, inp["lens"], 32, nthreads=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_decode_step_empty_sequence(orc):
    w = synth.WORKLOADS[2].scaled(Hq=2, Hkv=2, Nmax=16)
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    out, idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], codes,
                                  np.zeros(1, np.int32), budget=4)
    assert (out == 0).all() and (idx == -1).all()


def test_needles_are_selected_single_head_4k(orc):
    # the planted keys K_i = 2 q* + 0.1 N(0,1) must land in the 64-token budget
    w = synth.WORKLOADS[1]
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    _, idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, inp["lens"], 64)
    pos = synth.needle_positions(w, 0, 0, w.Nmax)
    assert set(pos.tolist()) <= set(idx[0, 0].tolist())


def test_needles_are_selected_gqa(orc):
    w = synth.WORKLOADS[4].scaled(B=2, Nmax=2048, len_range=(1024, 2048))
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    _, idx, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, inp["lens"], 256, nthreads=4)
    for b in range(w.B):
        for g in range(w.Hkv):
            pos = synth.needle_positions(w, b, g, int(inp["lens"][b]))
            for p, h in zip(pos, synth.needle_targets(w, g)):
                assert p in idx[b, h], (b, g, p, h)


# ---- group-shared selection for grouped heads (summed distances, one budget per kv head)

def test_group_shared_with_one_head_per_group_is_the_per_head_step(orc):
    w = synth.WORKLOADS[2].scaled(Hq=4, Hkv=4, Nmax=300)
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    lens = np.array([217], dtype=np.int32)
    out_s, idx_s = orc.decode_step_group_shared(inp["q"], inp["K"], inp["V"], codes, lens, 40)
    out_h, idx_h, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, lens, 40)
    assert np.array_equal(idx_s, idx_h)
    assert np.abs(out_s - out_h).max() < 1e-12


def test_group_shared_matches_brute_force(orc):
    # distances summed over the group's heads from unpacked 2-bit fields, ranked by
    # Python's sorted() on (sum, index); attention by torch SDPA over those rows
    w = synth.WORKLOADS[4].scaled(B=2, Hq=6, Hkv=2, Nmax=48, len_range=None, n_needles=2)
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    lens = np.array([48, 29], dtype=np.int32)
    budget = 11
    out, idx = orc.decode_step_group_shared(inp["q"], inp["K"], inp["V"], codes, lens, budget)
    G = 3
    for b in range(2):
        n = int(lens[b])
        for h in range(2):
            kf = unpack(codes[b, h, :n])
            total = np.zeros(n, dtype=np.int64)
            for g in range(G):
                qf = unpack(orc.encode(inp["q"][b, h * G + g]))
                total += np.abs(kf - qf).sum(axis=1)
            want = sorted(range(n), key=lambda t: (total[t], t))[:budget]
            assert idx[b, h, :len(want)].tolist() == want
            assert (idx[b, h, len(want):] == -1).all()
            for g in range(G):
                ref = _dense_sdpa(inp["q"][b, h * G + g], inp["K"][b, h][want], inp["V"][b, h][want])
                assert np.abs(out[b, h * G + g] - ref).max() < 1e-12


def test_group_shared_with_identical_queries_keeps_the_per_head_rows(orc):
    # equal query heads: the summed distance is G times each head's, so the order
    # (and the kept rows) cannot change
    w = synth.WORKLOADS[4].scaled(B=1, Hq=8, Hkv=2, Nmax=400, len_range=None)
    inp = synth.make_inputs(w)
    q = inp["q"].copy()
    q[:, 1:4] = q[:, 0:1]
    q[:, 5:8] = q[:, 4:5]
    codes = orc.encode(inp["K"])
    lens = np.array([400], dtype=np.int32)
    out_s, idx_s = orc.decode_step_group_shared(q, inp["K"], inp["V"], codes, lens, 64)
    out_h, idx_h, _ = orc.decode_step(q, inp["K"], inp["V"], codes, lens, 64)
    for hq in range(8):
        assert np.array_equal(idx_s[0, hq // 4], idx_h[0, hq])
    assert np.abs(out_s - out_h).max() < 1e-12


def test_group_shared_budget_and_empty_sequences(orc):
    w = synth.WORKLOADS[4].scaled(B=2, Hq=4, Hkv=2, Nmax=30, len_range=None)
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    lens = np.array([0, 30], dtype=np.int32)
    out, idx = orc.decode_step_group_shared(inp["q"], inp["K"], inp["V"], codes, lens, 50)
    assert (idx[0] == -1).all() and (out[0] == 0).all()
    for h in range(2):
        assert sorted(idx[1, h, :30].tolist()) == list(range(30)) and (idx[1, h, 30:] == -1).all()
        for g in range(2):  # budget >= len: dense attention over the whole sequence
            ref = _dense_sdpa(inp["q"][1, 2 * h + g], inp["K"][1, h], inp["V"][1, h])
            assert np.abs(out[1, 2 * h + g] - ref).max() < 1e-12


# ---- forced rows (attention sinks and the recent window rank ahead of scored tokens)

def test_forced_rows_none_is_the_plain_step(orc):
    w = synth.WORKLOADS[4].scaled(B=2, Hq=4, Hkv=2, Nmax=200, len_range=(90, 200))
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    out_f, idx_f = orc.decode_step_forced(inp["q"], inp["K"], inp["V"], codes, inp["lens"], 24, 0, 0)
    out_p, idx_p, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, inp["lens"], 24)
    assert np.array_equal(idx_f, idx_p)
    assert np.abs(out_f - out_p).max() < 1e-12


def test_forced_rows_match_brute_force(orc):
    w = synth.WORKLOADS[4].scaled(B=2, Hq=4, Hkv=2, Nmax=40, len_range=None, n_needles=2)
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    lens = np.array([40, 13], dtype=np.int32)
    n_sink, n_recent = 3, 5
    for budget in (4, 10, 20):  # fewer, as many as and more than the forced rows
        out, idx = orc.decode_step_forced(inp["q"], inp["K"], inp["V"], codes, lens, budget, n_sink, n_recent)
        for b in range(2):
            n = int(lens[b])
            for hq in range(4):
                h = hq // 2
                D = np.abs(unpack(codes[b, h, :n]) - unpack(orc.encode(inp["q"][b, hq]))).sum(axis=1)
                rank = [(-1 if (t < n_sink or t >= n - n_recent) else int(D[t]), t) for t in range(n)]
                want = [t for _, t in sorted(rank)][:min(budget, n)]
                assert idx[b, hq, :len(want)].tolist() == want
                assert (idx[b, hq, len(want):] == -1).all()
                ref = _dense_sdpa(inp["q"][b, hq], inp["K"][b, h][want], inp["V"][b, h][want])
                assert np.abs(out[b, hq] - ref).max() < 1e-12


def test_forced_rows_are_always_kept_when_they_fit(orc):
    w = synth.WORKLOADS[2].scaled(Hq=2, Hkv=2, Nmax=1000)
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    lens = np.array([1000], dtype=np.int32)
    _, idx = orc.decode_step_forced(inp["q"], inp["K"], inp["V"], codes, lens, 64, 4, 16)
    forced = list(range(4)) + list(range(984, 1000))
    for hq in range(2):
        assert idx[0, hq, :20].tolist() == forced
        assert len(set(idx[0, hq].tolist())) == 64


# ---- paged cache (a block table maps each sequence's logical pages to physical pages)

def test_paged_step_equals_the_contiguous_step(orc):
    # scatter a contiguous cache into shuffled physical pages; reading through the
    # table must give the contiguous step back exactly
    w = synth.WORKLOADS[4].scaled(B=3, Hq=4, Hkv=2, Nmax=96, len_range=None, n_needles=2)
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    lens = np.array([96, 37, 1], dtype=np.int32)
    P, max_pages = 16, 6
    rng = np.random.default_rng(5)
    n_pages = 3 * max_pages + 4
    perm = rng.permutation(n_pages)[:3 * max_pages].reshape(3, max_pages).astype(np.int32)
    Kp = rng.integers(0, 2 ** 16, size=(n_pages, 2, P, 128), dtype=np.uint16)  # garbage where unused
    Vp = rng.integers(0, 2 ** 16, size=(n_pages, 2, P, 128), dtype=np.uint16) & np.uint16(0x3FFF)
    Kp &= np.uint16(0x3FFF)
    Cp = rng.integers(0, 256, size=(n_pages, 2, P, 32), dtype=np.uint8)
    for b in range(3):
        for lp in range(max_pages):
            page = perm[b, lp]
            Kp[page] = inp["K"][b, :, lp * P:(lp + 1) * P]
            Vp[page] = inp["V"][b, :, lp * P:(lp + 1) * P]
            Cp[page] = codes[b, :, lp * P:(lp + 1) * P]
    out_p, idx_p = orc.decode_step_paged(inp["q"], Kp, Vp, Cp, perm, lens, 20)
    out_c, idx_c, _ = orc.decode_step(inp["q"], inp["K"], inp["V"], codes, lens, 20)
    assert np.array_equal(idx_p, idx_c)
    assert np.array_equal(out_p, out_c)


def test_paged_step_rejects_a_bad_table(orc):
    w = synth.WORKLOADS[2].scaled(Hq=2, Hkv=2, Nmax=32)
    inp = synth.make_inputs(w)
    Kp = np.zeros((2, 2, 16, 128), np.uint16)
    Cp = np.zeros((2, 2, 16, 32), np.uint8)
    with pytest.raises(ValueError):
        orc.decode_step_paged(inp["q"], Kp, Kp, Cp, np.array([[0, 5]], np.int32), np.array([32], np.int32), 4)


# ---- forced rows and group-shared selection together

def test_general_step_reduces_to_the_specific_steps(orc):
    w = synth.WORKLOADS[4].scaled(B=2, Hq=6, Hkv=2, Nmax=60, len_range=None, n_needles=2)
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    lens = np.array([60, 23], dtype=np.int32)
    args = (inp["q"], inp["K"], inp["V"], codes, lens)
    o, i = orc.decode_step_general(*args, 12, 2, 5, group_shared=False)
    o2, i2 = orc.decode_step_forced(*args, 12, 2, 5)
    assert np.array_equal(i, i2) and np.abs(o - o2).max() < 1e-12
    o, i = orc.decode_step_general(*args, 12, group_shared=True)
    o2, i2 = orc.decode_step_group_shared(*args, 12)
    assert np.array_equal(i, i2) and np.abs(o - o2).max() < 1e-12
    o, i = orc.decode_step_general(*args, 12)
    o2, i2, _ = orc.decode_step(*args, 12)
    assert np.array_equal(i, i2) and np.abs(o - o2).max() < 1e-12


def test_general_step_forced_and_shared_match_brute_force(orc):
    # summed unpacked-field L1 over the group, forced rows ranked at -1, Python sorted()
    w = synth.WORKLOADS[4].scaled(B=2, Hq=4, Hkv=2, Nmax=36, len_range=None, n_needles=2)
    inp = synth.make_inputs(w)
    codes = orc.encode(inp["K"])
    lens = np.array([36, 11], dtype=np.int32)
    n_sink, n_recent = 2, 3
    for budget in (3, 5, 9):
        out, idx = orc.decode_step_general(inp["q"], inp["K"], inp["V"], codes, lens, budget, n_sink, n_recent,
                                           group_shared=True)
        for b in range(2):
            n = int(lens[b])
            for h in range(2):
                kf = unpack(codes[b, h, :n])
                tot = sum(np.abs(kf - unpack(orc.encode(inp["q"][b, 2 * h + g]))).sum(axis=1) for g in range(2))
                rank = [(-1 if (t < n_sink or t >= n - n_recent) else int(tot[t]), t) for t in range(n)]
                want = [t for _, t in sorted(rank)][:min(budget, n)]
                assert idx[b, h, :len(want)].tolist() == want
                assert (idx[b, h, len(want):] == -1).all()
                for g in range(2):
                    ref = _dense_sdpa(inp["q"][b, 2 * h + g], inp["K"][b, h][want], inp["V"][b, h][want])
                    assert np.abs(out[b, 2 * h + g] - ref).max() < 1e-12
