"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the timing
reduction takes the max over ranks, and under torchrun the reference arm runs
on rank 0 alone and prints exactly one JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world),
                       "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_setup(world)
    try:
        bench.barrier(w)
        got = bench.max_over_ranks(1.5 + rank * 2.25, w)
        q.put((r, got))
    finally:
        bench.finish(w)


def test_max_over_ranks_with_gloo_world_size_two():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 3.75), (1, 3.75)]


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny", "--steps", "2",
           "--warmup", "3", "--cpu-seconds", "0.5"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_threshold_and_scale_options_reach_the_workload_and_the_json_line():
    """--alpha replaces the workload's threshold (inf: pure vector-wise), is
    written as a JSON-safe value, and the scale flags map onto the library's
    modes."""
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    from mixed_precision_int8_b200 import workloads
    wl = workloads.get_workload("tiny")
    same = bench.with_alpha(wl, argparse.Namespace(alpha=None))
    assert same.alpha == wl.alpha
    off = bench.with_alpha(wl, argparse.Namespace(alpha=float("inf")))
    assert off.alpha == float("inf") and off.s == wl.s and off.h == wl.h
    assert json.loads(json.dumps({"alpha": bench.alpha_json(off.alpha)})) == {"alpha": "inf"}
    assert bench.alpha_json(6.0) == 6.0
    assert bench.SCALE_MODES == {"row": 0, "column": 0, "tensor": 1}
