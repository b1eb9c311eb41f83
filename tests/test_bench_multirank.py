"""bench.py's multi-rank host logic, on CPU with two gloo ranks.

A multi-GPU bench run is a set of replicas: each rank decodes its own
sequences (the workload's seed moved by the rank), the step time is the
maximum over ranks, and the job's throughput counts every rank's tokens.
The reference (oracle) arm runs on rank 0 alone.  These tests run that host
logic as two processes joined by torch.distributed over gloo.
"""

import argparse
import contextlib
import importlib.util
import io
import json
import multiprocessing as mp
import os
import socket

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("hs2_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    bench = _load_bench()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w, r, _ = bench.dist_setup()
        wl = bench.rank_workload(r)
        ms = bench.max_over_ranks(1.0 + r, w, "cpu")       # rank r's step: 1 + r ms
        thr = bench.job_throughput(wl.B * wl.T, w, ms)
        from hs2_synth import make_attention_inputs
        small = wl.resized(B=1, L=256, n_needles=2, n_sparse=1)
        digest = int(make_attention_inputs(small).k.astype("int64").sum())
        args = argparse.Namespace(gpus=w, steps=1, warmup=0)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(args, w, r)
        dist.barrier()
        out.put((r, w, wl.seed, ms, thr, digest, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_timing_and_reference_arm():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, seed0, ms0, thr0, dig0, txt0), (r1, w1, seed1, ms1, thr1, dig1, txt1) = res
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    # every rank sees the slowest rank's step time; throughput counts both ranks
    assert ms0 == ms1 == 2.0
    assert thr0 == thr1 == 8 * 2 / 2e-3
    # each rank decodes its own sequences
    assert seed1 == seed0 + 1000 and dig0 != dig1
    # the reference arm prints one JSON line on rank 0 only
    assert txt1 == ""
    line = json.loads(txt0.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["metric"] == "hybrid-block decode tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_profiled_traffic_follows_the_kernel_sources(tmp_path):
    # an ncu summary gives `traffic` only while the source hash it records
    # matches the kernel sources; otherwise (or with no summary) it is null
    bench = _load_bench()
    body = "# summary\n\n- kernel_source_sha: `%s`\n- dram_bytes_per_launch: 138362624\n"
    current = tmp_path / "current.md"
    current.write_text(body % bench.kernel_source_hash())
    assert bench.profiled_traffic(str(current)) == 138362624.0
    stale = tmp_path / "stale.md"
    stale.write_text(body % "0000000000000000")
    assert bench.profiled_traffic(str(stale)) is None
    assert bench.profiled_traffic(str(tmp_path / "missing.md")) is None
