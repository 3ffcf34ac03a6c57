"""GPU decode step with its options (adamas_decode_step_ex) against the CPU oracle.

Forced rows (attention sinks and the recent window rank ahead of every scored
token), group-shared selection for grouped heads (distances summed over the
group's query heads, one budget per kv head), a paged cache read through a block
table, and the appended K/V rows written by the launch itself.  Indices must be
identical to the oracle's; outputs within max-abs 1e-2 / relative-RMS 1e-3.

Method: ADAMAS long-context sparse attention article (lnwmold.com/news/826806),
§2.3 (L1 scoring), §5.2 (token budget), §3.2 and §6 (tokens that keep full
attention), §3.1 (the cache grows by one row per token)."""
import numpy as np
import pytest
import torch

from compressed_sparse_kv_fp32_b200 import adamas, synth
from helpers import assert_close_out, dev, dev_bf16, host_u16

pytestmark = pytest.mark.gpu


def _setup(w, lens=None):
    inp = synth.make_inputs(w)
    if lens is not None:
        inp["lens"] = np.asarray(lens, np.int32)
    K, V = dev_bf16(inp["K"]), dev_bf16(inp["V"])
    codes = torch.empty(K.shape[:-1] + (32,), dtype=torch.uint8, device="cuda")
    adamas.encode_keys(K, codes)
    return inp, K, V, codes


def _run(inp, K, V, codes, budget, **kw):
    B, Hq, _ = inp["q"].shape
    Hkv = K.shape[1]
    Nmax = K.shape[2] if "block_table" not in kw else kw["block_table"].shape[1] * K.shape[2]
    ws = adamas.Workspace(B, Hq, Hkv, Nmax, budget)
    out, idx = adamas.decode(dev_bf16(inp["q"]), codes, K, V, dev(inp["lens"]), budget, ws, **kw)
    torch.cuda.synchronize()
    return out.cpu().numpy(), idx.cpu().numpy(), ws.device_error()


# ---------------------------------------------------------------- forced rows
@pytest.mark.parametrize("B,Hq,Hkv,N,lens,n_sink,n_recent,budgets", [
    (2, 4, 2, 40, [40, 13], 3, 5, (4, 8, 20)),           # fewer, as many as and more than the forced rows
    (1, 2, 2, 40000, [40000], 4, 64, (16, 68, 256)),      # 16 blocks per head: forced rows in the first and last
    (3, 12, 3, 3000, [3000, 70, 0], 0, 100, (64,)),       # recent window only; a short and an empty sequence
    (1, 8, 1, 200000, [200000], 16, 16, (512,)),          # distances in the workspace
])
def test_forced_rows(orc, B, Hq, Hkv, N, lens, n_sink, n_recent, budgets):
    w = synth.WORKLOADS[4].scaled(B=B, Hq=Hq, Hkv=Hkv, Nmax=N, len_range=None, n_needles=2)
    inp, K, V, codes = _setup(w, lens)
    ocodes = orc.encode(inp["K"])
    for budget in budgets:
        out, idx, err = _run(inp, K, V, codes, budget, n_sink=n_sink, n_recent=n_recent)
        want_out, want_idx = orc.decode_step_forced(inp["q"], inp["K"], inp["V"], ocodes, inp["lens"], budget,
                                                    n_sink, n_recent)
        assert err == 0
        assert np.array_equal(idx, want_idx), budget
        assert_close_out(out, want_out)


# ---------------------------------------------------------------- group-shared selection
@pytest.mark.parametrize("B,Hq,Hkv,N,lens,budget", [
    (2, 6, 2, 48, [48, 29], 11),
    (2, 4, 4, 300, [300, 217], 40),                       # one query head per group: the per-head step
    (3, 32, 8, 5000, [5000, 1200, 3333], 256),            # the GQA batch shape, smaller
    (1, 8, 1, 200000, [200000], 512),                     # G = 8, distances in the workspace
    (2, 24, 8, 20000, [20000, 9000], 1024),               # G = 3
])
def test_group_shared(orc, B, Hq, Hkv, N, lens, budget):
    w = synth.WORKLOADS[4].scaled(B=B, Hq=Hq, Hkv=Hkv, Nmax=N, len_range=None, n_needles=2)
    inp, K, V, codes = _setup(w, lens)
    out, idx, err = _run(inp, K, V, codes, budget, policy=adamas.SELECT_GROUP_SHARED)
    want_out, want_idx = orc.decode_step_group_shared(inp["q"], inp["K"], inp["V"], orc.encode(inp["K"]),
                                                      inp["lens"], budget)
    assert err == 0
    assert np.array_equal(idx, want_idx)
    assert_close_out(out, want_out)


def test_group_shared_heavy_ties(orc):
    w = synth.WORKLOADS[4].scaled(B=1, Hq=8, Hkv=2, Nmax=30000, len_range=None, n_needles=2)
    inp = synth.make_inputs(w)
    r = np.random.default_rng(7)
    pool = inp["K"][:, :, :5].copy()
    inp["K"][:] = pool[:, :, r.integers(0, 5, size=w.Nmax)]
    K, V = dev_bf16(inp["K"]), dev_bf16(inp["V"])
    codes = torch.empty(K.shape[:-1] + (32,), dtype=torch.uint8, device="cuda")
    adamas.encode_keys(K, codes)
    out, idx, err = _run(inp, K, V, codes, 3000, policy=adamas.SELECT_GROUP_SHARED)
    want_out, want_idx = orc.decode_step_group_shared(inp["q"], inp["K"], inp["V"], orc.encode(inp["K"]),
                                                      inp["lens"], 3000)
    assert err == 0
    assert np.array_equal(idx, want_idx)
    assert_close_out(out, want_out)


def test_group_shared_budget_above_its_limit_is_rejected():
    w = synth.WORKLOADS[4].scaled(B=1, Hq=4, Hkv=1, Nmax=8000, len_range=None)
    inp, K, V, codes = _setup(w)
    with pytest.raises(adamas.AdamasError) as e:
        _run(inp, K, V, codes, 5000, policy=adamas.SELECT_GROUP_SHARED)
    assert e.value.status == -2


# ---------------------------------------------------------------- paged cache
def _paginate(inp, orc, P, extra_pages, seed):
    """Scatter a contiguous cache into shuffled physical pages [n_pages, Hkv, P, ...]; the
    page codes are the oracle's codes of the page keys (zero keys where unused)."""
    B, Hkv, N, _ = inp["K"].shape
    max_pages = (N + P - 1) // P
    n_pages = B * max_pages + extra_pages
    rng = np.random.default_rng(seed)
    table = rng.permutation(n_pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    Kp = np.zeros((n_pages, Hkv, P, 128), np.uint16)
    Vp = np.zeros_like(Kp)
    pad = max_pages * P - N
    Kc = np.pad(inp["K"], ((0, 0), (0, 0), (0, pad), (0, 0)))
    Vc = np.pad(inp["V"], ((0, 0), (0, 0), (0, pad), (0, 0)))
    for b in range(B):
        for lp in range(max_pages):
            Kp[table[b, lp]] = Kc[b, :, lp * P:(lp + 1) * P]
            Vp[table[b, lp]] = Vc[b, :, lp * P:(lp + 1) * P]
    return Kp, Vp, orc.encode(Kp), table


@pytest.mark.parametrize("B,Hq,Hkv,N,lens,P,budget", [
    (3, 4, 2, 96, [96, 37, 1], 16, 20),
    (2, 8, 2, 40000, [40000, 27000], 16, 256),            # 16 blocks per head: stages span 64 pages
    (1, 4, 4, 9000, [8999], 64, 1024),
    (2, 2, 1, 5000, [5000, 3000], 1, 64),                 # one token per page
])
def test_paged_cache(orc, B, Hq, Hkv, N, lens, P, budget):
    w = synth.WORKLOADS[4].scaled(B=B, Hq=Hq, Hkv=Hkv, Nmax=N, len_range=None, n_needles=2)
    inp = synth.make_inputs(w)
    inp["lens"] = np.asarray(lens, np.int32)
    Kp, Vp, Cp, table = _paginate(inp, orc, P, extra_pages=3, seed=N)
    Kd, Vd = dev_bf16(Kp), dev_bf16(Vp)
    codes = torch.zeros(Cp.shape, dtype=torch.uint8, device="cuda")
    adamas.encode_keys(Kd, codes)                          # pages as B = n_pages sequences of P tokens
    assert np.array_equal(codes.cpu().numpy(), Cp)
    out, idx, err = _run(inp, Kd, Vd, codes, budget, block_table=dev(table))
    want_out, want_idx = orc.decode_step_paged(inp["q"], Kp, Vp, Cp, table, inp["lens"], budget)
    assert err == 0
    assert np.array_equal(idx, want_idx)
    assert_close_out(out, want_out)


def test_paged_bad_table_entry_is_flagged(orc):
    w = synth.WORKLOADS[4].scaled(B=1, Hq=2, Hkv=1, Nmax=64, len_range=None)
    inp = synth.make_inputs(w)
    Kp, Vp, Cp, table = _paginate(inp, orc, 16, extra_pages=0, seed=1)
    table[0, 2] = 99                                       # outside [0, n_pages)
    Kd, Vd = dev_bf16(Kp), dev_bf16(Vp)
    codes = torch.zeros(Cp.shape, dtype=torch.uint8, device="cuda")
    adamas.encode_keys(Kd, codes)
    _, _, err = _run(inp, Kd, Vd, codes, 8, block_table=dev(table))
    assert err & adamas.DEVERR_TABLE


# ---------------------------------------------------------------- appended rows written by the launch
@pytest.mark.parametrize("B,Hq,Hkv,N,lens,apos,budget", [
    (2, 4, 2, 50, [50, 13], [49, 12], 16),
    (2, 8, 2, 40000, [40000, 30000], [20001, 29999], 256),
    (1, 8, 1, 200000, [200000], [199999], 512),
])
def test_append_rows_written_by_the_launch(B, Hq, Hkv, N, lens, apos, budget):
    w = synth.WORKLOADS[4].scaled(B=B, Hq=Hq, Hkv=Hkv, Nmax=N, len_range=None, n_needles=2)
    inp = synth.make_inputs(w)
    K, V = dev_bf16(inp["K"]), dev_bf16(inp["V"])
    codes = torch.empty(K.shape[:-1] + (32,), dtype=torch.uint8, device="cuda")
    adamas.encode_keys(K, codes)
    r = np.random.default_rng(N)
    k_new = dev_bf16(synth.bf16_round(r.standard_normal((B, Hkv, 128)).astype(np.float32) * 2))
    v_new = dev_bf16(synth.bf16_round(r.standard_normal((B, Hkv, 128)).astype(np.float32)))
    q, seq, ap = dev_bf16(inp["q"]), dev(np.asarray(lens, np.int32)), dev(np.asarray(apos, np.int32))
    ws = adamas.Workspace(B, Hq, Hkv, N, budget)
    # reference: rows written first, then the fused append + decode launch
    K2, V2, c2 = K.clone(), V.clone(), codes.clone()
    for b in range(B):
        K2[b, :, apos[b]] = k_new[b]
        V2[b, :, apos[b]] = v_new[b]
    ref_out, ref_idx = adamas.decode_step_append(q, c2, K2, V2, seq, ap, budget, ws)
    torch.cuda.synchronize()
    out, idx = adamas.decode(q, codes, K, V, seq, budget, ws, append_pos=ap, k_new=k_new, v_new=v_new)
    torch.cuda.synchronize()
    assert ws.device_error() == 0
    assert torch.equal(K, K2) and torch.equal(V, V2) and torch.equal(codes, c2)
    assert torch.equal(idx, ref_idx)
    # the same kept rows; the reference may run the sliced step (long context, one kv
    # head), whose merge of slice states sums in another fp32 order: the outputs agree
    # within the float tolerance of every parity test
    assert_close_out(out.cpu().numpy(), ref_out.cpu().numpy())


# ---------------------------------------------------------------- every option at once
def test_paged_forced_shared_append_together(orc):
    B, Hq, Hkv, N, P, budget, n_sink, n_recent = 2, 8, 2, 9000, 32, 300, 4, 32
    lens, apos = [9000, 5000], [8999, 4999]
    w = synth.WORKLOADS[4].scaled(B=B, Hq=Hq, Hkv=Hkv, Nmax=N, len_range=None, n_needles=2)
    inp = synth.make_inputs(w)
    inp["lens"] = np.asarray(lens, np.int32)
    r = np.random.default_rng(3)
    k_new = synth.bf16_round(r.standard_normal((B, Hkv, 128)).astype(np.float32))
    v_new = synth.bf16_round(r.standard_normal((B, Hkv, 128)).astype(np.float32))
    # the oracle sees the cache with the new rows already in place
    Kw, Vw = inp["K"].copy(), inp["V"].copy()
    for b in range(B):
        Kw[b, :, apos[b]] = k_new[b]
        Vw[b, :, apos[b]] = v_new[b]
    ocodes = orc.encode(Kw)
    Kp, Vp, Cp, table = _paginate(inp, orc, P, extra_pages=2, seed=5)
    Kd, Vd = dev_bf16(Kp), dev_bf16(Vp)
    codes = torch.zeros(Cp.shape, dtype=torch.uint8, device="cuda")
    adamas.encode_keys(Kd, codes)
    out, idx, err = _run(inp, Kd, Vd, codes, budget, block_table=dev(table), append_pos=dev(np.asarray(apos, np.int32)),
                         k_new=dev_bf16(k_new), v_new=dev_bf16(v_new), n_sink=n_sink, n_recent=n_recent,
                         policy=adamas.SELECT_GROUP_SHARED)
    want_out, want_idx = orc.decode_step_general(inp["q"], Kw, Vw, ocodes, inp["lens"], budget, n_sink, n_recent,
                                                 group_shared=True)
    assert err == 0
    assert np.array_equal(idx, want_idx)
    assert_close_out(out, want_out)
    # the new rows and their codes are in their pages
    Kh, Ch = host_u16(Kd), codes.cpu().numpy()
    for b in range(B):
        page, slot = table[b, apos[b] // P], apos[b] % P
        assert np.array_equal(Kh[page, :, slot], k_new[b])
        assert np.array_equal(Ch[page, :, slot], orc.encode(k_new[b]))
