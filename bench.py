#!/usr/bin/env python
"""Benchmark of the HySparse2 hybrid-block hot path on B200.

One step = one hybrid block on the decode workload (8 sequences x 1 new query
at 32,768 tokens of bf16 MQA cache, 32 query heads, head_dim 128): the
full-attention layer with top-1024 + recent-128 selection, then three
sparse-attention layers that reuse its KV cache and indices, each with its
own queries.  The metric is hybrid-block decode tokens/s (queries through the
whole block per second).  The same line also carries the KV Bridging GEMM
("bridge") and the E4M3 configurations ("configs": 4 x 256K decode and the
4096-query chunk over a 1M-token cache), each timed on its own.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hs2|reference]

N > 1 runs one process per GPU under torch.distributed.run: every rank runs
its own replica of the workload (weak scaling; the decode path shards by
sequence with no exchange), times are the max over ranks.  --impl reference
times the CPU oracle on the same workload (rank 0 only).
"""

import argparse
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

from hs2_synth import WORKLOADS, make_attention_inputs  # noqa: E402

WORKLOAD = "decode_bf16_32k"
L2_FLUSH_BYTES = 512 << 20
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["hs2", "reference"], default="hs2")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-bridge", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--only", choices=["append", "blocks", "configs", "decode_fp8_256k",
                                       "chunk_fp8_1m"], default=None,
                    help="run one section alone on one GPU and print its JSON (for profiling)")
    ap.add_argument("--profile-case", choices=list(PROFILE_CASES), default=None,
                    help="two untimed calls of one small case, for an ncu capture of its kernels")
    return ap.parse_args()


# Small cases of the library's calls for ncu captures: inputs larger than L2
# where DRAM figures matter, a few GB on the device at most.
PROFILE_CASES = {
    "decode_bf16": "hs2_full_attn_select on the 8 x 32K bf16 decode workload",
    "decode_fp8": "hs2_full_attn_select on the 4 x 256K E4M3 decode workload",
    "chunk_small": "hs2_full_attn_select on a 512-query chunk over 128K E4M3 tokens",
    "sparse_chunk": "hs2_sparse_attn on a 1024-query chunk over 256K E4M3 tokens",
    "sparse_decode": "hs2_sparse_attn on the 8 x 32K bf16 decode workload",
    "bridge_131k": "hs2_bridge_kv of 131072 tokens into 6 layers' bf16 caches",
    "bridge_append": "hs2_bridge_kv of 64 tokens into 6 layers' E4M3 caches",
}


def run_profile_case(name):
    """Two calls of one PROFILE_CASES case, L2 flushed before each; exits non-zero
    when the device status reports an error."""
    import torch
    import long_context_hs2_b200 as hs2
    g = torch.Generator(device="cuda").manual_seed(1)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def l2_flush():
        flush.zero_()
        flush.view(torch.int64).amax()

    def e4m3(n, D):
        x = torch.randn(n, D, device="cuda", generator=g)
        sc = x.abs().amax(1).clamp_min(1e-30) / 448.0 * (1 + torch.rand(n, device="cuda", generator=g) / 2)
        return (x / sc[:, None]).to(torch.float8_e4m3fn).view(torch.uint8), sc.float()

    def attn(wname, **kw):
        wl = WORKLOADS[wname].resized(**kw) if kw else WORKLOADS[wname]
        B, T, L, H, D = wl.B, wl.T, wl.L, wl.H, wl.D
        q = torch.randn(B, T, H, D, device="cuda", generator=g).to(torch.bfloat16)
        if wl.kv_dtype == "fp8":
            k, ks = e4m3(B * L, D)
            v, vs = e4m3(B * L, D)
            kv, dt = hs2.kv_cache(k, v, ks, vs), hs2.HS2_KV_FP8_E4M3
        else:
            k = torch.randn(B * L, D, device="cuda", generator=g).to(torch.bfloat16)
            v = torch.randn(B * L, D, device="cuda", generator=g).to(torch.bfloat16)
            kv, dt = hs2.kv_cache(k, v), hs2.HS2_KV_BF16
        slots = wl.topk + wl.window
        nb = hs2.hs2_full_attn_select_workspace(B, T, L, H, D, wl.topk, wl.window, dt)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        O = torch.empty(B, T, H, D, device="cuda")
        idx = torch.empty(B, T, slots, dtype=torch.int32, device="cuda")
        ns = torch.empty(B, T, dtype=torch.int32, device="cuda")
        full = lambda: hs2.hs2_full_attn_select(q, kv, B, T, L, H, D, wl.scale, wl.topk,
                                                wl.window, dt, O, None, idx, ns, ws, nb)
        sparse = lambda: hs2.hs2_sparse_attn(q, kv, B, T, L, H, D, wl.scale, idx, ns, slots, dt, O)
        return full, sparse

    if name == "decode_bf16":
        calls = [attn("decode_bf16_32k")[0]] * 2
    elif name == "decode_fp8":
        calls = [attn("decode_fp8_256k")[0]] * 2
    elif name == "chunk_small":
        calls = [attn("chunk_fp8_1m", T=512, L=131072)[0]] * 2
    elif name == "sparse_chunk":
        full, sparse = attn("chunk_fp8_1m", T=1024, L=262144)
        calls = [full, sparse, sparse]
    elif name == "sparse_decode":
        full, sparse = attn("decode_bf16_32k")
        calls = [full, sparse, sparse]
    elif name == "bridge_131k":
        T, hidden, nl, D = 131072, 4096, 6, 128
        wt = (torch.randn(nl * 2 * D, hidden, device="cuda", generator=g) / 64).to(torch.bfloat16)
        x = (torch.randn(T, hidden, device="cuda", generator=g) / 64).to(torch.bfloat16)
        bufs = [(torch.empty(T, D, dtype=torch.bfloat16, device="cuda"),
                 torch.empty(T, D, dtype=torch.bfloat16, device="cuda"), None, None)
                for _ in range(nl)]
        caches = [hs2.kv_cache(*b_) for b_ in bufs]
        calls = [lambda: hs2.hs2_bridge_kv(x, T, hidden, wt, nl, D, hs2.HS2_KV_BF16, caches, 0)] * 2
    else:  # bridge_append
        T, hidden, nl, D, rows = 64, 4096, 6, 128, 2048
        wt = (torch.randn(nl * 2 * D, hidden, device="cuda", generator=g) / 64).to(torch.bfloat16)
        x = (torch.randn(T, hidden, device="cuda", generator=g) / 64).to(torch.bfloat16)
        bufs = [(torch.empty(rows, D, dtype=torch.uint8, device="cuda"),
                 torch.empty(rows, D, dtype=torch.uint8, device="cuda"),
                 torch.empty(rows, device="cuda"), torch.empty(rows, device="cuda"))
                for _ in range(nl)]
        caches = [hs2.kv_cache(*b_) for b_ in bufs]
        calls = [lambda: hs2.hs2_bridge_kv(x, T, hidden, wt, nl, D, hs2.HS2_KV_FP8_E4M3, caches,
                                           1000)] * 2
    for c in calls:
        l2_flush()
        c()
        torch.cuda.synchronize()
    st = hs2.hs2_last_device_status()
    print(json.dumps({"profile_case": name, "what": PROFILE_CASES[name], "status": st}), flush=True)
    if st != 0:
        raise SystemExit(1)


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (burst)"
    except Exception:
        return 1590.0, "fallback"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# Multi-GPU runs are replicas: the decode path shards by sequence with no
# exchange, so rank r runs its own sequences (the workload with its seed moved
# by r) and the only collectives are barriers and the max-over-ranks timing.
def rank_workload(rank: int):
    base = WORKLOADS[WORKLOAD]
    return base.resized(seed=base.seed + 1000 * rank)


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest of every rank's `value` (a no-op for one rank)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (ms * 1e-3)


# ------------------------------------------------------------- oracle arm --
def oracle_rows_per_s(inp, rows, n_sparse):
    """Oracle time for the block on `rows` query rows (full + select + sparse layers)."""
    import oracle
    wl = inp.wl
    t0 = time.perf_counter()
    r = oracle.full_attn_select(inp.q, inp.k, inp.v, inp.k_scale, inp.v_scale, scale=wl.scale,
                                topk=wl.topk, window=wl.window, rows=rows)
    idx = np.full((wl.B * wl.T, wl.topk + wl.window), -1, dtype=np.int32)
    ns = np.zeros(wl.B * wl.T, dtype=np.int32)
    idx[rows] = r["idx"]
    ns[rows] = r["n_sel"]
    for layer in range(n_sparse):
        oracle.sparse_attn(inp.q_sparse[layer], inp.k, inp.v, inp.k_scale, inp.v_scale, idx, ns,
                           scale=wl.scale, rows=rows)
    dt = time.perf_counter() - t0
    return len(rows) / dt, dt, oracle.threads()


def bench_config(wl, world):
    """The `config` object of both arms' JSON lines (the same keys and values)."""
    return {"workload": WORKLOAD, "B": wl.B, "T": wl.T, "L": wl.L, "H": wl.H, "D": wl.D,
            "kv": wl.kv_dtype, "topk": wl.topk, "window": wl.window,
            "sparse_layers": wl.n_sparse, "parallelism": "replicas (dp%d)" % world,
            "l2": "flushed before each step (512 MB write, then read back)"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    wl = WORKLOADS[WORKLOAD]
    inp = make_attention_inputs(wl)
    rows = np.arange(1)          # one sequence's query per step: a bounded sample
    for _ in range(args.warmup):
        oracle_rows_per_s(inp, rows, wl.n_sparse)
    times = []
    cores = 1
    for s in range(args.steps):
        rows = np.array([s % (wl.B * wl.T)])
        _, dt, cores = oracle_rows_per_s(inp, rows, wl.n_sparse)
        times.append(dt)
    ms = 1000.0 * statistics.median(times)
    value = 1000.0 / ms
    line = {
        "impl": "reference", "metric": "hybrid-block decode tokens/s", "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": bench_config(wl, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": "1 of the 8 sequences per step (full attention + selection "
                                   "+ 3 sparse layers), plain C++ fp64 oracle"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ KV Bridging --
def bench_bridge(torch, hs2, args, stream):
    """Times hs2_bridge_kv on the bridge workload (131072 tokens x 4096 -> 6 layers of
    K|V, D=128), bf16 and E4M3 outputs, as a tensor-bound roofline beside the decode
    metric.  Timing inputs are drawn on the device with torch's generator in the
    workload's distributions (X ~ N(0,1)/64, Wt ~ N(0, 1/4096)); parity of this shape
    against the oracle is covered by the test suite."""
    from hs2_synth import WORKLOADS as W
    wl = W["bridge_131k"]
    T, hidden, nl, D = wl.T, wl.hidden, wl.n_layers, wl.D
    g = torch.Generator(device="cuda").manual_seed(wl.seed)
    x = (torch.randn(T, hidden, device="cuda", generator=g) / 64).to(torch.bfloat16)
    wt = (torch.randn(nl * 2 * D, hidden, device="cuda", generator=g) / 64).to(torch.bfloat16)
    out = {}
    flops = 2.0 * T * hidden * nl * 2 * D
    peak = measured_tensor_peak()
    for name, dt in (("bf16", hs2.HS2_KV_BF16), ("fp8", hs2.HS2_KV_FP8_E4M3)):
        if dt == hs2.HS2_KV_BF16:
            bufs = [(torch.empty(T, D, dtype=torch.bfloat16, device="cuda"),
                     torch.empty(T, D, dtype=torch.bfloat16, device="cuda"), None, None)
                    for _ in range(nl)]
        else:
            bufs = [(torch.empty(T, D, dtype=torch.uint8, device="cuda"),
                     torch.empty(T, D, dtype=torch.uint8, device="cuda"),
                     torch.empty(T, device="cuda"), torch.empty(T, device="cuda"))
                    for _ in range(nl)]
        caches = [hs2.kv_cache(*b) for b in bufs]
        for _ in range(3):
            hs2.hs2_bridge_kv(x, T, hidden, wt, nl, D, dt, caches, 0, stream)
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(10)]
        for a, b in evs:
            a.record(stream)
            hs2.hs2_bridge_kv(x, T, hidden, wt, nl, D, dt, caches, 0, stream)
            b.record(stream)
        torch.cuda.synchronize()
        st = hs2.hs2_last_device_status()
        if st != 0:
            raise RuntimeError("bridge device status: " + hs2.hs2_status_string(st))
        ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
        tf = flops / (ms * 1e-3) / 1e12
        out[name] = {"ms": ms, "tflops": tf, "frac": tf / peak[0], "peak": peak[0],
                     "peak_source": peak[1]}
        del bufs, caches
    out["workload"] = "bridge_131k: X [131072 x 4096] bf16, Wt [1536 x 4096] bf16, 6 layers, D=128"
    out["bound"] = "tensor"
    out["unit"] = "TFLOP/s"
    return out


def bench_bridge_append(torch, hs2, stream, flush_fn, peak_gbs):
    """Times the decode-time append of hs2_bridge_kv: T in {1, 64} new tokens
    bridged into the six target layers (hidden 4096, D = 128) at a row offset of
    existing caches, L2 flushed before every call.  The call reads the weights
    once (HBM-bound): algorithmic bytes = Wt + X + the written rows."""
    from hs2_synth import WORKLOADS as W
    wl = W["bridge_131k"]
    hidden, nl, D = wl.hidden, wl.n_layers, wl.D
    g = torch.Generator(device="cuda").manual_seed(wl.seed)
    wt = (torch.randn(nl * 2 * D, hidden, device="cuda", generator=g) / 64).to(torch.bfloat16)
    rows = 4096
    out = {}
    for T in (1, 64):
        x = (torch.randn(T, hidden, device="cuda", generator=g) / 64).to(torch.bfloat16)
        for name, dt in (("bf16", hs2.HS2_KV_BF16), ("fp8", hs2.HS2_KV_FP8_E4M3)):
            if dt == hs2.HS2_KV_BF16:
                bufs = [(torch.empty(rows, D, dtype=torch.bfloat16, device="cuda"),
                         torch.empty(rows, D, dtype=torch.bfloat16, device="cuda"), None, None)
                        for _ in range(nl)]
                row_bytes = 2 * D * 2
            else:
                bufs = [(torch.empty(rows, D, dtype=torch.uint8, device="cuda"),
                         torch.empty(rows, D, dtype=torch.uint8, device="cuda"),
                         torch.empty(rows, device="cuda"), torch.empty(rows, device="cuda"))
                        for _ in range(nl)]
                row_bytes = 2 * (D + 4)
            caches = [hs2.kv_cache(*b) for b in bufs]
            for _ in range(3):
                hs2.hs2_bridge_kv(x, T, hidden, wt, nl, D, dt, caches, 1000, stream)
            torch.cuda.synchronize()
            ts = []
            for _ in range(20):
                flush_fn()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                hs2.hs2_bridge_kv(x, T, hidden, wt, nl, D, dt, caches, 1000, stream)
                b.record(stream)
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b))
            st = hs2.hs2_last_device_status()
            if st != 0:
                raise RuntimeError("bridge append device status: " + hs2.hs2_status_string(st))
            ms = float(np.median(ts))
            nbytes = wt.numel() * 2 + x.numel() * 2 + T * nl * row_bytes
            out["T%d_%s" % (T, name)] = {"us": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9,
                                         "frac_hbm": nbytes / (ms * 1e-3) / 1e9 / peak_gbs,
                                         "algorithmic_bytes": nbytes}
            del bufs, caches
    out["workload"] = "T new tokens x hidden 4096 -> 6 layers of K|V (D=128) at a row offset"
    out["bound"] = "hbm"
    return out


def bench_block_selection(torch, hs2, inp, kv, q, stream, flush_fn):
    """A/B of the selection granularity on the decode workload's own inputs (the
    full-attention call alone, L2 flushed before each): token-level selection
    against the 64-token block-level selection of the earlier HySparse, with the
    same 1024-position budget; needle recall = share of the planted needles
    whose position is selected for the query they were planted for."""
    wl = inp.wl
    B, T, L, H, D = wl.B, wl.T, wl.L, wl.H, wl.D
    slots = wl.topk + wl.window
    dt = hs2.HS2_KV_BF16
    nb = hs2.hs2_full_attn_select_workspace(B, T, L, H, D, wl.topk, wl.window, dt)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    O = torch.empty(B, T, H, D, device="cuda")
    idx = torch.empty(B, T, slots, dtype=torch.int32, device="cuda")
    ns = torch.empty(B, T, dtype=torch.int32, device="cuda")
    out = {}
    for label, block in (("token", 0), ("block64", 64)):
        def call():
            if block:
                hs2.hs2_full_attn_select_blocks(q, kv, B, T, L, H, D, wl.scale, wl.topk,
                                                wl.window, block, dt, O, None, idx, ns, ws, nb,
                                                stream)
            else:
                hs2.hs2_full_attn_select(q, kv, B, T, L, H, D, wl.scale, wl.topk, wl.window, dt,
                                         O, None, idx, ns, ws, nb, stream)
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        ts = []
        for _ in range(10):
            flush_fn()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        st = hs2.hs2_last_device_status()
        if st != 0:
            raise RuntimeError("block selection device status: " + hs2.hs2_status_string(st))
        gi = idx.cpu().numpy().reshape(B * T, slots)
        gn = ns.cpu().numpy().reshape(-1)
        hit = [int(j) in set(gi[b * T + t, :gn[b * T + t]].tolist()) for b, j, t in inp.needles]
        out[label] = {"full_ms": float(np.median(ts)), "needle_recall": float(np.mean(hit))}
    out["needles"] = int(len(inp.needles))
    out["budget"] = "%d positions + %d window" % (wl.topk, wl.window)
    return out


# ------------------------------------------------------- other configurations --
def bench_other_configs(torch, hs2, stream, flush_fn, peak_gbs, peak_tflops,
                        names=("decode_fp8_256k", "chunk_fp8_1m")):
    """Times the full-attention call and one sparse layer on the E4M3 configurations
    (4 x 256K decode; the 4096-query chunk over a 1M-token cache), beside the decode
    metric.  Inputs are drawn on the device in the workloads' distributions (Q, K, V
    ~ N(0,1); E4M3 codes with the per-token scale max|x|/448); L2 is flushed before
    every timed call; parity of these shapes is covered by the test suite."""
    out = {}
    for name, reps in (("decode_fp8_256k", 10), ("chunk_fp8_1m", 3)):
        if name not in names:
            continue
        wl = WORKLOADS[name]
        B, T, L, H, D = wl.B, wl.T, wl.L, wl.H, wl.D
        g = torch.Generator(device="cuda").manual_seed(wl.seed)
        q = torch.randn(B, T, H, D, device="cuda", generator=g).to(torch.bfloat16)

        def e4m3(n_rows):
            x = torch.randn(n_rows, D, device="cuda", generator=g)
            sc = x.abs().amax(dim=1).clamp_min(1e-30) / 448.0
            return (x / sc[:, None]).to(torch.float8_e4m3fn).view(torch.uint8), sc

        k, ks = e4m3(B * L)
        v, vs = e4m3(B * L)
        kv = hs2.kv_cache(k, v, ks, vs)
        dt = hs2.HS2_KV_FP8_E4M3
        slots = wl.topk + wl.window
        nb = hs2.hs2_full_attn_select_workspace(B, T, L, H, D, wl.topk, wl.window, dt)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        O = torch.empty(B, T, H, D, device="cuda")
        idx = torch.empty(B, T, slots, dtype=torch.int32, device="cuda")
        ns = torch.empty(B, T, dtype=torch.int32, device="cuda")

        def full():
            hs2.hs2_full_attn_select(q, kv, B, T, L, H, D, wl.scale, wl.topk, wl.window, dt, O,
                                     None, idx, ns, ws, nb, stream)

        def sparse():
            hs2.hs2_sparse_attn(q, kv, B, T, L, H, D, wl.scale, idx, ns, slots, dt, O, stream)

        res = {}
        for label, fn in (("full", full), ("sparse", sparse)):
            for _ in range(2):
                fn()
            torch.cuda.synchronize()
            ts = []
            for _ in range(reps):
                flush_fn()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b))
            res[label] = float(np.median(ts))
        st = hs2.hs2_last_device_status()
        if st != 0:
            raise RuntimeError(name + " device status: " + hs2.hs2_status_string(st))
        kv_bytes = 2 * B * L * (D + 4)
        sp_bytes = B * T * slots * 2 * (D + 4) + B * T * H * D * 6
        entry = {"workload": name, "full_ms": res["full"], "sparse_layer_ms": res["sparse"],
                 "sparse_gbs": sp_bytes / (res["sparse"] * 1e-3) / 1e9,
                 "sparse_frac_hbm": sp_bytes / (res["sparse"] * 1e-3) / 1e9 / peak_gbs}
        if T == 1:
            full_bytes = kv_bytes + B * T * H * D * 6 + B * T * slots * 4
            entry.update({"full_gbs": full_bytes / (res["full"] * 1e-3) / 1e9,
                          "full_frac_hbm": full_bytes / (res["full"] * 1e-3) / 1e9 / peak_gbs})
        else:
            # the method's work: QK^T and PV over the causal (query, key, head)
            # triples (a recomputation of QK^T for the scores is not counted)
            triples = sum((L - T + t + 1) for t in range(T)) * H
            flops = triples * 4 * D
            exps = triples
            entry.update({"full_tflops": flops / (res["full"] * 1e-3) / 1e12,
                          "full_frac_tensor": flops / (res["full"] * 1e-3) / 1e12 / peak_tflops,
                          "full_exp_per_s": exps / (res["full"] * 1e-3)})
        out[name] = entry
        del k, v, ks, vs, ws, O, q
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ GPU arm --
PARTIAL_PROFILE = os.path.join(ROOT, "profiles", "attn_tc_fused_decode_bf16_32k.md")
# the fused kernel's sources and the host code that plans its launch (splits,
# keys per split, fused selection, retained logits)
KERNEL_SOURCES = ("attn_tc.cuh", "tc_common.cuh", "hs2_common.cuh", "full_attn.cuh", "select.cuh",
                  "hs2_api.cu")


def kernel_source_hash():
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "long_context_hs2_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(path):
    """DRAM bytes per launch of the dominant kernel from its committed ncu
    summary, or None when there is none or the kernel sources changed since."""
    try:
        fields = {}
        with open(path) as f:
            for line in f:
                if ":" in line and line.startswith("- "):
                    k, v = line[2:].split(":", 1)
                    fields[k.strip()] = v.strip().strip("`")
        if fields.get("kernel_source_sha") != kernel_source_hash():
            return None
        return float(fields["dram_bytes_per_launch"])
    except Exception:
        return None


def run_hs2(args, world, rank, local):
    import torch
    import torch.distributed as dist
    import long_context_hs2_b200 as hs2

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    hs2.load_library()
    wl = rank_workload(rank)       # each rank: its own sequences
    inp = make_attention_inputs(wl)
    B, T, L, H, D = wl.B, wl.T, wl.L, wl.H, wl.D
    slots = wl.topk + wl.window
    dt = hs2.HS2_KV_BF16

    def up(a, dtype):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(dtype)

    k = up(inp.k, torch.bfloat16)
    v = up(inp.v, torch.bfloat16)
    kv = hs2.kv_cache(k, v)
    qs = [up(q, torch.bfloat16) for q in [inp.q] + inp.q_sparse]
    ws_bytes = hs2.hs2_full_attn_select_workspace(B, T, L, H, D, wl.topk, wl.window, dt)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    # the step's inputs (all layers' queries) and results (outputs, indices,
    # counts) each live in one device buffer, so that the end-to-end steps move
    # them with one host-to-device and one device-to-host copy
    n_q = B * T * H * D
    q_all = torch.empty(len(qs) * n_q, dtype=torch.bfloat16, device="cuda")
    d_q = [q_all[i * n_q:(i + 1) * n_q].view(B, T, H, D) for i in range(len(qs))]
    n_out = len(qs) * n_q + B * T * slots + B * T
    out_all = torch.empty(n_out, dtype=torch.float32, device="cuda")
    outs = [out_all[i * n_q:(i + 1) * n_q].view(B, T, H, D) for i in range(len(qs))]
    o_idx = len(qs) * n_q
    idx = out_all[o_idx:o_idx + B * T * slots].view(torch.int32).view(B, T, slots)
    nsel = out_all[o_idx + B * T * slots:].view(torch.int32).view(B, T)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def l2_flush():
        # write a buffer larger than L2, then read it back so that no dirty
        # lines of the flush are left to be written back inside the next step
        flush.zero_()
        flush.view(torch.int64).amax()

    def step(q_list):
        hs2.hs2_full_attn_select(q_list[0], kv, B, T, L, H, D, wl.scale, wl.topk, wl.window, dt,
                                 outs[0], None, idx, nsel, ws, ws_bytes, stream)
        for s in range(wl.n_sparse):
            hs2.hs2_sparse_attn(q_list[1 + s], kv, B, T, L, H, D, wl.scale, idx, nsel, slots, dt,
                                outs[1 + s], stream)

    def block(q_list):
        # captured into graphs: the library launches on the current (capturing) stream
        hs2.hs2_full_attn_select(q_list[0], kv, B, T, L, H, D, wl.scale, wl.topk, wl.window, dt,
                                 outs[0], None, idx, nsel, ws, ws_bytes)
        for s in range(wl.n_sparse):
            hs2.hs2_sparse_attn(q_list[1 + s], kv, B, T, L, H, D, wl.scale, idx, nsel, slots, dt,
                                outs[1 + s])

    for _ in range(args.warmup):
        l2_flush()
        step(qs)
    torch.cuda.synchronize()
    st = hs2.hs2_last_device_status()
    if st != 0:
        raise RuntimeError("device status after warm-up: " + hs2.hs2_status_string(st))

    # Every step replays one CUDA graph holding the whole block (the full
    # layer's counter memset and fused kernel, then the sparse layers, the first
    # launched programmatically behind the fused kernel), as a decode loop would.
    # The fused kernel's own duration comes from a second timed pass of the same
    # steps whose graphs also hold a pair of stage events around that kernel:
    # the two event nodes serialise the graph (about 8 us per step on B200), so
    # the headline steps carry none.
    for dq, q in zip(d_q, qs):
        dq.copy_(q)
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        block(d_q)
    stage_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
    for a, b in stage_ev:  # torch marks them recorded; reversed, so a pair the
        b.record(stream)   # graphs never re-record shows a negative time below
        a.record(stream)
    g_stage = []
    for i in range(args.steps):
        g = torch.cuda.CUDAGraph()
        hs2.hs2_set_stage_events(*stage_ev[i])
        with torch.cuda.graph(g):
            block(d_q)
        hs2.hs2_set_stage_events()
        g_stage.append(g)
    for i in range(max(args.warmup, args.steps)):
        l2_flush()
        g_step.replay()
        l2_flush()
        g_stage[i % args.steps].replay()
    torch.cuda.synchronize()

    # ---- device-timed steps (inputs resident in HBM; L2 flushed before each),
    # then the instrumented pass
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    ev_st = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    clocks = ClockSampler(local if world == 1 else int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        l2_flush()
        a, c = ev[i]
        a.record(stream)
        g_step.replay()
        c.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    for i in range(args.steps):
        l2_flush()
        a, c = ev_st[i]
        a.record(stream)
        g_stage[i].replay()
        c.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(c) for a, c in ev]
    inst_ms = [a.elapsed_time(c) for a, c in ev_st]
    partial_ms = [a.elapsed_time(b) for a, b in stage_ev]
    if min(partial_ms) <= 0:
        raise RuntimeError("stage events were not recorded by the instrumented graphs")
    # step start -> end of the fused kernel; end of the fused kernel -> step end
    full_ms = [a.elapsed_time(b) for (a, _), (_, b) in zip(ev_st, stage_ev)]
    sparse_ms = [b.elapsed_time(c) / wl.n_sparse for (_, b), (_, c) in zip(stage_ev, ev_st)]
    st = hs2.hs2_last_device_status()
    if st != 0:
        raise RuntimeError("device status after timing: " + hs2.hs2_status_string(st))

    # ---- end to end: pinned host queries in, outputs back, every step
    h_q = torch.empty(q_all.shape, dtype=q_all.dtype, pin_memory=True)
    h_q.copy_(q_all.cpu())
    h_out = torch.empty(out_all.shape, dtype=out_all.dtype, pin_memory=True)
    h2d = q_all.numel() * q_all.element_size()
    d2h = out_all.numel() * out_all.element_size()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        l2_flush()
        a, c = e2e_ev[i]
        a.record(stream)
        q_all.copy_(h_q, non_blocking=True)
        g_step.replay()
        h_out.copy_(out_all, non_blocking=True)
        c.record(stream)
    torch.cuda.synchronize()
    e2e_ms = [a.elapsed_time(c) for a, c in e2e_ev]
    phases = fused_phases(torch, hs2, l2_flush, lambda: step(qs), 2 * B * L * D * 2 + B * T * H * D * 2)

    def agg(xs):
        return max_over_ranks(float(np.median(xs)), world, "cuda")

    ms = agg(step_ms)
    full = agg(full_ms)
    sparse = agg(sparse_ms)
    partial = agg(partial_ms)
    inst = agg(inst_ms)
    e2e = agg(e2e_ms)
    peak, peak_kind = measured_peaks()
    # algorithmic bytes of the dominant kernel (the fused attention pass: one pass over
    # K and V, plus the queries) and of one sparse layer (the selected K/V rows,
    # queries, outputs, indices)
    partial_bytes = 2 * B * L * D * 2 + B * T * H * D * 2
    sparse_bytes = B * T * slots * 2 * D * 2 + B * T * H * D * 2 + B * T * H * D * 4 + B * T * slots * 4
    achieved = partial_bytes / (partial * 1e-3) / 1e9
    traffic = profiled_traffic(PARTIAL_PROFILE)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rps, dts, cores = oracle_rows_per_s(inp, np.arange(B * T), wl.n_sparse)
        cpu = {"value": rps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": "one full step: %d sequences x 1 query, full attention + selection + "
                         "%d sparse layers (%.1f s)" % (B, wl.n_sparse, dts)}
    bridge = bench_bridge(torch, hs2, args, stream) if (rank == 0 and not args.no_bridge) else None
    append = (bench_bridge_append(torch, hs2, stream, l2_flush, peak)
              if (rank == 0 and not args.no_bridge) else None)
    blocks = (bench_block_selection(torch, hs2, inp, kv, qs[0], stream, l2_flush)
              if rank == 0 and not args.no_configs else None)
    others = None
    if rank == 0 and not args.no_configs:
        others = bench_other_configs(torch, hs2, stream, l2_flush, peak,
                                     measured_tensor_peak()[0])
    del g_step, g_stage
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": "hybrid-block decode tokens/s",
        "value": job_throughput(B * T, world, ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": bench_config(WORKLOADS[WORKLOAD], world),
        "e2e": {"value": job_throughput(B * T, world, e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        # per step: the fused full-attention kernel (partials, score and
        # selection in one launch for this shape) and one per sparse layer
        "gpu_launches": (1 + wl.n_sparse) * args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "attn_tc_fused_kernel<32,1,bf16> (partials over K/V, score pass, "
                               "selection; algorithmic bytes: K and V once, and the queries)",
                     "algorithmic_bytes": partial_bytes, "ms": partial,
                     "peak_source": peak_kind,
                     "timing": "CUDA events around the kernel inside each step graph, in a "
                               "second timed pass of the same steps"},
        # from the instrumented pass: fused kernel end -> step end, per sparse layer;
        # step start -> fused kernel end; and that pass's whole step
        "sparse_layer": {"ms": sparse, "achieved_gbs": sparse_bytes / (sparse * 1e-3) / 1e9,
                         "frac": sparse_bytes / (sparse * 1e-3) / 1e9 / peak},
        "full_ms": full,
        "instrumented_ms_per_step": inst,
        "fused_phases": phases,
        "clocks": clk,
        "cpu_baseline": cpu,
        "bridge": bridge,
        "bridge_append": append,
        "block_selection": blocks,
        "configs": others,
    }
    print(json.dumps(line), flush=True)


def fused_phases(torch, hs2, l2_flush, call, stream_bytes, reps=5):
    """Where the fused kernel's time goes, from the global-timer stamps its CTAs
    write when enabled (outside every timed region; L2 flushed before each
    call).  Times in us from the first CTA's start, medians over `reps` calls:
    when the last CTA finished its partial pass (every K/V tile streamed),
    passed each group barrier, finished the score pass and finished; and the
    partial pass's achieved bandwidth: K and V once plus the queries over
    first start -> last partial done."""
    n = 1024
    buf = torch.zeros(n * hs2.HS2_PHASES, dtype=torch.int64, device="cuda")
    rows = []
    try:
        hs2.hs2_set_phase_stamps(buf, n)
        for _ in range(reps):
            buf.zero_()
            l2_flush()
            call()
            torch.cuda.synchronize()
            st = buf.view(n, hs2.HS2_PHASES).cpu().numpy()
            st = st[st[:, 0] > 0]
            t0 = st[:, 0].min()
            rows.append([(st[:, k].max() - t0) / 1e3 if (st[:, k] > 0).all() else float("nan")
                         for k in range(7)])
    finally:
        hs2.hs2_set_phase_stamps(None)
    med = np.nanmedian(np.array(rows), axis=0)
    names = ["start_spread", "partial_done", "barrier1", "score_done", "barrier2", "barrier3", "end"]
    out = {k: (float(v) if np.isfinite(v) else None) for k, v in zip(names, med)}
    out["unit"] = "us from the first CTA's start (latest CTA per phase)"
    if out["partial_done"]:
        peak, _ = measured_peaks()
        out["stream_gbs"] = stream_bytes / (out["partial_done"] * 1e-6) / 1e9
        out["stream_frac"] = out["stream_gbs"] / peak
    return out


def run_section(args):
    """One section of the GPU arm alone (no headline step): for profiling."""
    import torch
    import long_context_hs2_b200 as hs2
    torch.cuda.set_device(0)
    hs2.load_library()
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def l2_flush():
        flush.zero_()
        flush.view(torch.int64).amax()

    peak, _ = measured_peaks()
    if args.only == "append":
        out = bench_bridge_append(torch, hs2, stream, l2_flush, peak)
    elif args.only == "blocks":
        inp = make_attention_inputs(WORKLOADS[WORKLOAD])
        up = (lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
              .view(torch.bfloat16))
        kv = hs2.kv_cache(up(inp.k), up(inp.v))
        out = bench_block_selection(torch, hs2, inp, kv, up(inp.q), stream, l2_flush)
    else:
        names = ("decode_fp8_256k", "chunk_fp8_1m") if args.only == "configs" else (args.only,)
        out = bench_other_configs(torch, hs2, stream, l2_flush, peak, measured_tensor_peak()[0],
                                  names)
    print(json.dumps({"section": args.only, args.only: out}), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup()
    if args.profile_case:
        run_profile_case(args.profile_case)
    elif args.only:
        run_section(args)
    elif args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_hs2(args, world, rank, local)


if __name__ == "__main__":
    main()
