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
           "--impl", "reference", "--gpus", "2", "--workload", "tiny", "--steps", "2",
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
    assert d["config"]["parallelism"] == "replicas x2"
    # the time per step is that of the sample actually run each step
    assert d["ms_per_step"] * d["steps"] / 1e3 < 600


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


def test_gpus_flag_and_launcher_must_agree():
    """--gpus N without torchrun launches N ranks; under a launcher whose
    WORLD_SIZE differs from N the run stops with an error instead of timing
    the wrong number of replicas."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.check_world(1, {}) == "run"
    assert bench.check_world(4, {}) == "launch"
    assert bench.check_world(2, {"WORLD_SIZE": "2"}) == "run"
    msg = bench.check_world(8, {"WORLD_SIZE": "1"})
    assert msg not in ("run", "launch") and "WORLD_SIZE=1" in msg
    cmd = bench.launch_command(2, ["--gpus", "2", "--steps", "3"])
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node" in cmd and cmd[cmd.index("--nproc-per-node") + 1] == "2"
    assert "127.0.0.1" in cmd and cmd[-3:] == ["--gpus", "2", "--steps", "3"][-3:]


def test_both_arms_describe_the_workload_with_the_same_config():
    """The reference arm's config has exactly our arm's keys and values, so
    the two lines describe one workload; the L2 policy depends on the
    workload's input size only."""
    sys.path.insert(0, ROOT)
    import bench
    from mixed_precision_int8_b200 import workloads
    args = bench.parse_args(["--workload", "opt175b_ffn_up_prefill"])
    for name in workloads.WORKLOAD_ORDER:
        wl = workloads.get_workload(name)
        c1 = bench.workload_config(wl, 1, args)
        assert set(c1) == {"workload", "s", "h", "o", "alpha", "outlier_cols",
                           "parallelism", "scales", "l2"}
        assert c1 == bench.workload_config(wl, 1, args)
    big = workloads.get_workload("opt175b_ffn_up_prefill")
    small = workloads.get_workload("opt6.7b_attn_prefill")
    assert not bench.needs_flush(big) and "no flush" in bench.l2_policy(big)
    assert bench.needs_flush(small) and "flushed" in bench.l2_policy(small)
    assert not bench.needs_flush(workloads.get_workload("opt175b_decode"))
    assert args.workload == "opt175b_ffn_up_prefill"
    assert bench.parse_args([]).workload == "opt175b_ffn_up_prefill"
