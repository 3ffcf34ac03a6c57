"""Throughput of the ADAMAS sparse decode path on B200.

One step = one attention layer's decode for the whole batch of a workload: one
launch that encodes the appended token's key into the code cache, encodes the
query, scores every cached token of every kv head by the L1 distance of the
codes, selects the budget of best tokens and runs exact attention over their
K/V rows.  The default workload is the 128K-context one (batch 1, 32 heads,
head dim 128, context 131072, budget 1024, per-head selection); four layer
buffers rotate so that the working set is far larger than L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--budget K] [--policy per_head|group_shared]
                    [--slices S] [--page-size P]

Prints one JSON line.  --impl reference times the CPU oracle on a bounded sample
of the same workload.  Under torchrun every rank runs its own independent copy of
the workload (weak scaling, no collective on the data path); the time is the max
over ranks.

--page-size P keeps every layer's cache in pages of P tokens, [n_pages][Hkv][P][...],
placed in a shuffled order and read through a block table (the step with options).

--slices S times the sequence-sharded step instead: every sequence split into S
contiguous slices.  Under torchrun S must equal the number of ranks (one slice per
GPU, histograms and softmax states exchanged over NCCL); on one GPU the S slices
are emulated one after the other (their kernels run in turn, the exchanges are
local stacks), so the time is the sum of the S slices' work.
"""
from __future__ import annotations

import argparse
import ctypes
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from compressed_sparse_kv_fp32_b200 import accounting, synth  # noqa: E402

METRIC = "decode steps/s and achieved HBM GB/s (% of B200 peak) at 128K ctx, budget 1024"
UNIT = "decode steps/s"
DEFAULT_WORKLOAD = "mha32_128k"
DEFAULT_BUDGET = {"single_head_4k": 64, "mha32_32k": 1024, "mha32_128k": 1024, "gqa8x4_b8_32k": 256,
                  "gqa8x3_1m": 1024}
LAYERS = 4
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="adamas", choices=["adamas", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=500)
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="rotating layer buffers (fewer only for profiling captures)")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(DEFAULT_BUDGET))
    ap.add_argument("--budget", type=int, default=None)
    ap.add_argument("--policy", default="per_head", choices=["per_head", "group_shared"])
    ap.add_argument("--slices", type=int, default=0, help="time the sequence-sharded step over S slices")
    ap.add_argument("--page-size", type=int, default=0,
                    help="read the cache through a block table of pages of this many tokens (shuffled pages)")
    a = ap.parse_args()
    if a.budget is None:
        a.budget = DEFAULT_BUDGET[a.workload]
    return a


def workload_of(name):
    return next(w for w in synth.WORKLOADS.values() if w.name == name)


def metric_of(args, w):
    if args.workload == DEFAULT_WORKLOAD and args.budget == 1024 and args.policy == "per_head" and not args.page_size:
        return METRIC
    return (f"decode steps/s and achieved HBM GB/s (% of B200 peak): {w.name}, context {w.Nmax}, "
            f"budget {args.budget}, {args.policy.replace('_', '-')} selection"
            + (f", paged cache ({args.page_size}-token pages)" if args.page_size else ""))


def source_hash() -> str:
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "compressed_sparse_kv_fp32_b200", "csrc", "*"))):
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        v = float(json.load(open(path))["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this source."""
    path = os.path.join(ROOT, "profiles", f"{kernel}.json")
    try:
        p = json.load(open(path))
    except Exception:
        return None
    if p.get("source_hash") != source_hash():
        return None
    return p.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm = [float(r[0]) for r in self.rows if len(r) >= 8 and r[0].replace(".", "").isdigit()]
        if not sm:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows if len(r) >= 8 for i in range(4)
                          if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(self.rows[-1][1]),
                "samples": len(sm), "reasons": reasons}


# ---------------------------------------------------------------- CPU oracle (baseline / reference arm)
def oracle_sample(w, budget: int, policy: str, max_heads: int, min_seconds: float):
    """Time the oracle's decode step on a sample of the workload's (sequence, kv head)
    pairs at their full length; the value is scaled to whole steps."""
    from oracle import oracle

    lens = synth.seq_lens(w)
    pairs = [(b, h) for b in range(w.B) for h in range(w.Hkv)][:max_heads]
    cores = os.cpu_count() or 1
    by_b = {}
    for b, h in pairs:
        by_b.setdefault(b, []).append(h)
    sub = []
    for b, hs in by_b.items():
        n = int(lens[b])
        K = np.stack([synth.head_kv(w, b, h, rows=n)[0] for h in hs])[None]
        V = np.stack([synth.head_kv(w, b, h, rows=n)[1] for h in hs])[None]
        qh = [h * w.G + g for h in hs for g in range(w.G)]
        q = synth.query(w, 1)[b:b + 1, qh]
        sub.append((q, K, V, oracle.encode(K), np.array([n], np.int32), len(hs)))
    reps, t0 = 0, time.perf_counter()
    while True:
        for q, K, V, codes, ln, nh in sub:
            if policy == "group_shared":
                oracle.decode_step_group_shared(q, K, V, codes, ln, budget)
            else:
                oracle.decode_step(q, K, V, codes, ln, budget, nthreads=min(cores, nh * w.G))
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    steps = reps * len(pairs) / (w.B * w.Hkv)
    used = 1 if policy == "group_shared" else min(cores, max(nh for *_, nh in sub) * w.G)
    return {"value": steps / el, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"{reps} oracle decode steps over {len(pairs)} of {w.B * w.Hkv} (sequence, kv head) pairs "
                      f"at full length ({w.name}, budget {budget}, {policy.replace('_', '-')} selection: query "
                      f"encode + L1 over every token + sort + float64 attention); value scaled to whole steps"}


def config_block(w, args, n_layers=LAYERS):
    lens = synth.seq_lens(w)
    shape = (f"batch {w.B}, {w.Hq} query heads over {w.Hkv} kv heads, head_dim {w.d}, context {w.Nmax}"
             + ("" if w.len_range is None else f" (lengths {int(lens.min())}..{int(lens.max())})"))
    return {"workload": f"{w.name}: {shape}, budget {args.budget}, {args.policy.replace('_', '-')} selection, "
                        f"1 appended token per sequence per step",
            "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "context": w.Nmax, "budget": args.budget, "head_dim": w.d,
            "policy": args.policy,
            "l2": f"{n_layers} rotating layer buffers (K, V, codes), working set "
                  f"{n_layers * (2 * w.B * w.Hkv * w.Nmax * 256 + w.B * w.Hkv * w.Nmax * 32) / 2**30:.1f} GiB > L2",
            "parallelism": "independent replica per GPU"}


def run_reference(args, rank, world):
    if rank != 0:  # rank 0 alone times the oracle and prints; the others do no work
        return
    w = workload_of(args.workload)
    cb = oracle_sample(w, args.budget, args.policy, max_heads=min(8, os.cpu_count() or 1), min_seconds=15.0)
    line = {"impl": "reference", "metric": metric_of(args, w), "value": cb["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / cb["value"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8/f64",
            "data": "synthetic", "config": config_block(w, args), "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings over the process group (identity on one rank)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_value(world: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job throughput: every rank runs `steps` steps of its own replica."""
    return world * steps / (elapsed_ms / 1e3)


# ---------------------------------------------------------------- GPU arm
def run_gpu(args, rank, world):
    import torch
    import torch.distributed as dist

    from compressed_sparse_kv_fp32_b200 import adamas

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lib = adamas.load()
    w = workload_of(args.workload)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.Nmax, w.d
    budget = args.budget
    shared = args.policy == "group_shared"
    lens_np = synth.seq_lens(w)

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)

    # one layer generated on the host head by head, copied into every layer buffer
    n_layers = max(1, args.layers)
    Ks = [torch.empty((B, Hkv, N, d), dtype=torch.bfloat16, device=dev) for _ in range(n_layers)]
    Vs = [torch.empty_like(Ks[0]) for _ in range(n_layers)]
    new_k = np.empty((B, Hkv, d), np.uint16)
    new_v = np.empty_like(new_k)
    for b in range(B):
        for h in range(Hkv):
            k, v = synth.head_kv(w, b, h)
            kd, vd = to_dev(k), to_dev(v)
            for l in range(n_layers):
                Ks[l][b, h].copy_(kd)
                Vs[l][b, h].copy_(vd)
            new_k[b, h], new_v[b, h] = k[lens_np[b] - 1], v[lens_np[b] - 1]
    P = args.page_size
    table = None
    if P > 0:  # pages of P tokens in a shuffled physical order, read through a block table
        max_pages = (N + P - 1) // P
        n_pages = B * max_pages
        perm = torch.from_numpy(np.random.default_rng(7).permutation(n_pages)).to(dev)
        table = perm.to(torch.int32).view(B, max_pages).contiguous()
        for l in range(n_layers):
            for X in (Ks, Vs):
                pad = torch.zeros((B, Hkv, max_pages * P, d), dtype=torch.bfloat16, device=dev)
                pad[:, :, :N] = X[l]
                logical = pad.view(B, Hkv, max_pages, P, d).permute(0, 2, 1, 3, 4).reshape(n_pages, Hkv, P, d)
                phys = torch.empty((n_pages, Hkv, P, d), dtype=torch.bfloat16, device=dev)
                phys[perm] = logical
                X[l] = phys
                del pad, logical
        N = max_pages * P
    layers = []
    for l in range(n_layers):
        codes = torch.empty(tuple(Ks[l].shape[:3]) + (32,), dtype=torch.uint8, device=dev)
        adamas.encode_keys(Ks[l], codes)
        q = to_dev(synth.query(w, l + 1))
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
        idx = torch.empty((B, Hkv if shared else Hq, budget), dtype=torch.int32, device=dev)
        ws = adamas.Workspace(B, Hq, Hkv, N, budget, device=dev)
        layers.append(dict(K=Ks[l], V=Vs[l], codes=codes, q=q, out=out, idx=idx, ws=ws))
    lens = torch.from_numpy(lens_np).to(dev)
    pos = (lens - 1).to(torch.int32)   # the appended token: the newest of every sequence
    torch.cuda.synchronize()

    # ---- prefill encoder: the whole cache of one layer, the layers in turn (inputs > L2)
    enc_reps = 2 * n_layers
    for i in range(n_layers):
        adamas.encode_keys(layers[i]["K"], layers[i]["codes"])
    torch.cuda.synchronize()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record()
    for i in range(enc_reps):
        L = layers[i % n_layers]
        adamas.encode_keys(L["K"], L["codes"])
    g1.record()
    torch.cuda.synchronize()
    enc_us = g0.elapsed_time(g1) / enc_reps * 1e3
    (enc_us,) = max_over_ranks([enc_us], dev)

    # one launch per step through the C ABI, arguments prepared once per layer
    stream = torch.cuda.current_stream().cuda_stream
    argss = []
    for L in layers:
        argss.append(adamas.DecodeArgs(
            L["q"].data_ptr(), L["codes"].data_ptr(), L["K"].data_ptr(), L["V"].data_ptr(), lens.data_ptr(),
            B, Hq, Hkv, N, d, budget, L["out"].data_ptr(), L["idx"].data_ptr(), L["ws"].buffer.data_ptr(),
            L["ws"].nbytes, pos.data_ptr(), None, None,
            None if table is None else table.data_ptr(), 0 if table is None else table.numel(),
            P if table is not None else 0, table.shape[1] if table is not None else 0, 0, 0,
            adamas.SELECT_GROUP_SHARED if shared else adamas.SELECT_PER_HEAD))
    refs = [ctypes.byref(a) for a in argss]
    f_step = lib.adamas_decode_step_ex

    def step(i):
        if f_step(refs[i % n_layers], stream) != 0:
            raise RuntimeError("decode step failed")

    gpu_id = "0"
    try:
        p = torch.cuda.get_device_properties(dev)
        gpu_id = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
    except Exception:
        gpu_id = str(local)
    sampler = ClockSampler(gpu_id)
    sampler.start()

    for i in range(max(3, args.warmup)):
        step(i)
    t_end = time.perf_counter() + (1.0 if n_layers == LAYERS else 0.0)  # ~1 s busy so clocks settle
    i = 0
    while time.perf_counter() < t_end:
        step(i)
        i += 1
        if i % 256 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    K_steps = args.steps
    # one launch per step and nothing else on the stream between launches (an event
    # between two launches would keep the next one from starting while the previous
    # one drains), so the launch duration is the timed region over the steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(K_steps):
        step(i)
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()

    elapsed_ms = t0.elapsed_time(t1)
    dec_ms = elapsed_ms / K_steps
    for L in layers:
        if L["ws"].device_error() != 0:
            raise RuntimeError("device error word set during the bench")

    elapsed_ms, dec_ms = max_over_ranks([elapsed_ms, dec_ms], dev)

    # ---- end to end through the Python API: pinned host inputs in, results out, every
    # step: one copy in (q and the new token's K and V rows), one launch (which writes
    # the rows into the cache, encodes the key and decodes), one copy out (out and idx)
    e2e_steps = min(args.e2e_steps, K_steps)
    nq, nkv = B * Hq * d, B * Hkv * d
    in_pin = torch.empty(nq + 2 * nkv, dtype=torch.bfloat16).pin_memory()
    in_pin[:nq].copy_(torch.from_numpy(synth.query(w, 3).reshape(-1).view(np.int16)).view(torch.bfloat16))
    in_pin[nq:nq + nkv].copy_(torch.from_numpy(new_k.reshape(-1).view(np.int16)).view(torch.bfloat16))
    in_pin[nq + nkv:].copy_(torch.from_numpy(new_v.reshape(-1).view(np.int16)).view(torch.bfloat16))
    in_dev = torch.empty_like(in_pin, device=dev)
    q_dev = in_dev[:nq].view(B, Hq, d)
    krow_dev = in_dev[nq:nq + nkv].view(B, Hkv, d)
    vrow_dev = in_dev[nq + nkv:].view(B, Hkv, d)
    rows = Hkv if shared else Hq
    n_out, n_idx = B * Hq * d, B * rows * budget   # fp32 and int32 words
    res_dev = torch.empty(n_out + n_idx, dtype=torch.int32, device=dev)
    res_pin = torch.empty_like(res_dev, device="cpu").pin_memory()
    out_dev = res_dev[:n_out].view(torch.float32).view(B, Hq, d)
    idx_dev = res_dev[n_out:].view(B, rows, budget)
    h2d = in_pin.numel() * 2
    d2h = res_pin.numel() * 4
    policy = adamas.SELECT_GROUP_SHARED if shared else adamas.SELECT_PER_HEAD

    # the C ABI call a serving loop makes (arguments prepared once per layer, as a
    # loop would keep them), reading its inputs from and writing its results to the
    # device buffers that the copies fill and drain
    e2e_args = [adamas.DecodeArgs(
        q_dev.data_ptr(), L["codes"].data_ptr(), L["K"].data_ptr(), L["V"].data_ptr(), lens.data_ptr(),
        B, Hq, Hkv, N, d, budget, out_dev.data_ptr(), idx_dev.data_ptr(), L["ws"].buffer.data_ptr(), L["ws"].nbytes,
        pos.data_ptr(), krow_dev.data_ptr(), vrow_dev.data_ptr(),
        None if table is None else table.data_ptr(), 0 if table is None else table.numel(),
        P if table is not None else 0, table.shape[1] if table is not None else 0, 0, 0, policy) for L in layers]
    e2e_refs = [ctypes.byref(a) for a in e2e_args]
    cur = torch.cuda.current_stream()

    def e2e_step(i):
        in_dev.copy_(in_pin, non_blocking=True)
        if f_step(e2e_refs[i % n_layers], stream) != 0:
            raise RuntimeError("decode step failed")
        res_pin.copy_(res_dev, non_blocking=True)
        cur.synchronize()

    for i in range(3 if e2e_steps > 0 else 0):
        e2e_step(i)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) if e2e_steps > 0 else float("nan")
    (e2e_ms,) = max_over_ranks([e2e_ms], dev)

    if rank != 0:
        return
    ms_per_step = elapsed_ms / K_steps
    value = job_value(world, K_steps, elapsed_ms)
    keff = [min(budget, int(n)) for n in lens_np]
    unique = sum(Hkv * k for k in keff) if shared else None
    step_bytes = accounting.decode_step_bytes(lens_np, Hq, Hkv, budget, d, unique_rows=unique)
    enc_bytes = B * Hkv * accounting.encode_bytes_per_vector(d)
    peak, peak_kind = measured_peak()
    launch_bytes = step_bytes["total"] + enc_bytes   # the launch also encodes the appended keys
    achieved_dec = launch_bytes / (dec_ms / 1e3) / 1e9
    achieved_step = launch_bytes / (ms_per_step / 1e3) / 1e9
    headline = args.workload == DEFAULT_WORKLOAD and budget == 1024 and not shared and not P
    traffic = profiled_traffic("decode_step_kernel_mha32_128k") if headline else None
    enc_all = B * Hkv * N * accounting.encode_bytes_per_vector(d)
    line = {
        "metric": metric_of(args, w), "value": value, "unit": UNIT, "n_gpus": world, "steps": K_steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8/fp32", "data": "synthetic",
        "config": dict(config_block(w, args, n_layers),
                       **({"page_size": P, "cache": f"{B * ((w.Nmax + P - 1) // P)} pages of {P} tokens in shuffled "
                           "order, read through a block table"} if P > 0 else {})),
        "achieved_hbm_gbs": achieved_step, "pct_of_peak_hbm": 100.0 * achieved_step / peak,
        "peak_hbm_gbs": peak, "peak_kind": peak_kind,
        "roofline": {"bound": "hbm", "kernel": "decode_step_kernel" if not (shared or P) else "decode_step_ext_kernel",
                     "achieved": achieved_dec, "peak": peak,
                     "unit": "GB/s", "frac": achieved_dec / peak, "traffic": traffic,
                     "algorithmic_bytes_per_launch": launch_bytes, "avg_launch_us": dec_ms * 1e3,
                     "bytes": {"codes": step_bytes["codes"], "kv_rows": step_bytes["kv_rows"], "q": step_bytes["q"],
                               "appended_keys": enc_bytes},
                     "peak_source": f"MEASURED_PEAKS.json hbm_gbs ({peak_kind})"},
        "e2e": ({"value": job_value(world, e2e_steps, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                 "d2h_bytes_per_step": d2h,
                 "per_step": "1 copy in, 1 launch through the C ABI (rows written, key encoded, decode), "
                             "1 copy out, 1 synchronise"}
                if e2e_steps > 0 else None),
        "gpu_launches": K_steps,
        "clocks": clocks,
        "encode": {"kernel": "encode_keys_kernel", "what": f"prefill of {B * Hkv * N} key vectors ({N} tokens x "
                   f"{B * Hkv} kv heads), timed outside the decode steps",
                   "avg_launch_us": enc_us, "algorithmic_bytes_per_launch": enc_all,
                   "achieved_gbs": enc_all / (enc_us / 1e6) / 1e9, "peak": peak, "unit": "GB/s",
                   "frac": enc_all / (enc_us / 1e6) / 1e9 / peak},
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample(w, budget, args.policy, max_heads=min(8, os.cpu_count() or 1),
                                             min_seconds=12.0)
    print(json.dumps(line), flush=True)


def run_sharded(args, rank, world):
    """The sequence-sharded step (see the module docstring for --slices)."""
    import torch

    from compressed_sparse_kv_fp32_b200 import adamas, sharded

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = workload_of(args.workload)
    B, Hq, Hkv, d, budget = w.B, w.Hq, w.Hkv, w.d, args.budget
    S = args.slices
    if world > 1 and S != world:
        raise SystemExit("--slices must equal the number of ranks under torchrun")
    mine = [rank] if world > 1 else list(range(S))
    lens_np = synth.seq_lens(w)
    bounds = [[sharded.slice_bounds(int(n), S, r) for n in lens_np] for r in range(S)]

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)

    slices = {}
    for r in mine:
        ln = np.array([e - a for a, e in bounds[r]], np.int32)
        nmax = max(1, int(ln.max()))
        K = torch.zeros((B, Hkv, nmax, d), dtype=torch.bfloat16, device=dev)
        V = torch.zeros_like(K)
        for b in range(B):
            a, e = bounds[r][b]
            for h in range(Hkv):
                k, v = synth.head_kv(w, b, h)
                K[b, h, :e - a] = to_dev(k[a:e])
                V[b, h, :e - a] = to_dev(v[a:e])
        codes = torch.empty((B, Hkv, nmax, 32), dtype=torch.uint8, device=dev)
        adamas.encode_keys(K, codes)
        slices[r] = dict(K=K, V=V, codes=codes, lens=torch.from_numpy(ln).to(dev),
                         ops=sharded.CudaShardOps(B, Hq, Hkv, nmax, budget, device=dev))
    q = to_dev(synth.query(w, 1))
    torch.cuda.synchronize()

    if world > 1:
        ex = sharded.TorchExchange()
        sl = slices[rank]

        def step():
            return sharded.decode_step_sharded(q, sl["codes"], sl["K"], sl["V"], sl["lens"], budget, sl["ops"], ex)
    else:
        def step():
            hist_all = torch.stack([slices[r]["ops"].score(q, slices[r]["codes"], slices[r]["lens"], budget)
                                    for r in mine], 0)
            st = [slices[r]["ops"].attend(q, slices[r]["K"], slices[r]["V"], slices[r]["lens"], budget, hist_all, r)
                  for r in mine]
            idx = st[0][1]
            for _, i in st[1:]:
                idx = torch.maximum(idx, i)
            return slices[mine[0]]["ops"].merge(torch.stack([p for p, _ in st], 0)), idx

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    (elapsed_ms,) = max_over_ranks([t0.elapsed_time(t1)], dev)
    # per slice: its two kernels alone (score, then attend with the gathered
    # histograms), the time one GPU of a real sharded step spends in kernels
    per_slice = None
    if world == 1:
        hist_all = torch.stack([slices[r]["ops"].score(q, slices[r]["codes"], slices[r]["lens"], budget)
                                for r in mine], 0)
        per_slice = []
        for r in mine:
            sl = slices[r]
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            reps = max(1, args.steps // 4)
            ev[0].record()
            for _ in range(reps):
                sl["ops"].score(q, sl["codes"], sl["lens"], budget)
                sl["ops"].attend(q, sl["K"], sl["V"], sl["lens"], budget, hist_all, r)
            ev[1].record()
            torch.cuda.synchronize()
            per_slice.append(ev[0].elapsed_time(ev[1]) / reps * 1e3)
    for r in mine:
        if slices[r]["ops"].workspace.device_error() != 0:
            raise RuntimeError("device error word set during the sharded bench")
    if rank != 0:
        return
    ms = elapsed_ms / args.steps
    step_bytes = accounting.decode_step_bytes(lens_np, Hq, Hkv, budget, d)
    # the sharded step also writes and reads back every distance (2 B per token and query head)
    spill = 2 * 2 * int(lens_np.sum()) * Hq
    line = {
        "metric": f"sharded decode steps/s, {w.name}, budget {budget}, {S} slices"
                  + (" emulated on one GPU" if world == 1 else " on as many GPUs"),
        "value": 1e3 / ms, "unit": "decode steps/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "u8/fp32", "data": "synthetic",
        "config": dict(config_block(w, args), slices=S,
                       workload=f"{w.name}: batch {B}, {Hq} query heads over {Hkv} kv heads, context {w.Nmax}, "
                                f"budget {budget}, sequences split into {S} contiguous slices, no append",
                       l2=f"one buffer per slice, codes of all slices {B * Hkv * w.Nmax * 32 / 2**30:.2f} GiB",
                       parallelism=f"sequence-sharded over {S} slices"),
        "algorithmic_bytes_per_step": step_bytes["total"] + spill,
        "achieved_gbs": (step_bytes["total"] + spill) / (ms / 1e3) / 1e9,
        "per_slice_kernel_us": per_slice,
        "exchange_bytes_per_rank": {"histograms": B * Hq * adamas.HIST_STRIDE * 4,
                                    "states": B * Hq * adamas.PARTIAL_FLOATS * 4, "idx": B * Hq * budget * 4},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        (run_sharded if args.slices > 0 else run_gpu)(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
