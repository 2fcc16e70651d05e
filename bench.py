#!/usr/bin/env python
"""Benchmark of the B200 LLM.int8() linear layer (one JSON line on stdout).

A step is one llmint8_matmul call: the whole hot path (outlier detection, row
quantisation, outlier tiles, int8 tcgen05 GEMM with the fused dequantisation /
outlier product / fp16 store) on one batch of seeded synthetic input already
resident in HBM. The metric is effective TOPS = 2*s*h*o / step time, with the
fraction of the layer's roofline max(2*s*h*o / P_int8, compulsory bytes / HBM)
beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--per-shape A,B,..|none] [--impl ours|reference]

The headline workload (default: the OPT-175B-like FFN up-projection, the
largest single-GPU shape) gives the line's top-level keys; the other
OPT-shaped workloads follow in ``per_shape`` with the same fields.

Timing: W untimed warm-up steps; then exactly K steps between a barrier +
synchronize on both sides, each step timed with CUDA events on the launching
stream. Where a workload's inputs (X and the int8 weight) fit twice in the
126 MB L2, a 512 MB buffer is written before every timed step (outside the
step's events); larger inputs stream from HBM by themselves and nothing is
flushed. The line's ``config.l2`` says which. SM clocks and throttle reasons
are sampled with NVML as fast as it answers during the K timed steps; a
second, longer window of the same steps (``clocks_soak``) repeats them for at
least half a second. Multi-GPU (torchrun, or --gpus N, which launches it):
independent replicas on every rank (the layer has no exchange step), time =
max over ranks, value = total work of all ranks / that time. With
--parallel columns each rank instead owns a block of W's output columns
(strong scaling: the layer's work is split, value = the whole layer's work /
the slowest rank's time; the blocks need no exchange).

--impl reference times the CPU oracle (plain C, OpenMP) on the host cores,
on a bounded row sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from mixed_precision_int8_b200 import workloads  # noqa: E402

METRIC = "LLM.int8() matmul effective TOPS"
UNIT = "TOPS"
DEFAULT_WORKLOAD = "opt175b_ffn_up_prefill"
# name@alpha: the workload with another outlier threshold (4.5: about 63
# outlier columns on the 6.7B shape; 0: every column, the fp16 extreme)
DEFAULT_PER_SHAPE = ("opt6.7b_attn_prefill", "opt13b_ffn_up_prefill",
                     "opt175b_decode", "opt6.7b_attn_prefill@4.5",
                     "opt6.7b_attn_prefill@0")
L2_BYTES = 126 << 20
FLUSH_BYTES = 512 << 20
# per-shape entries time at least this many steps (short bursts, like the
# headline's K steps, so no entry runs long enough to meet the power cap)
PER_SHAPE_MIN_STEPS = 50
SOAK_MIN_S = 0.5
# scale granularity flags -> LLMINT8_SCALE_VECTORWISE (0) / TENSORWISE (1)
SCALE_MODES = {"row": 0, "column": 0, "tensor": 1}
KERNEL_SOURCES = ["mixed_precision_int8_b200/csrc/gemm_sm100.cuh",
                  "mixed_precision_int8_b200/csrc/gemm_pair_sm100.cuh",
                  "mixed_precision_int8_b200/csrc/decode_sm100.cuh",
                  "mixed_precision_int8_b200/csrc/quant_kernels.cuh",
                  "mixed_precision_int8_b200/csrc/outlier_rows.cuh",
                  "mixed_precision_int8_b200/csrc/ptx_sm100.cuh",
                  "mixed_precision_int8_b200/csrc/llmint8_api.cu"]


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernels are
    unchanged since it was taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("kernel_source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def l2_policy(wl) -> str:
    """How the cache is kept out of the measurement for this workload."""
    inputs = 2 * wl.s * wl.h + wl.h * wl.o
    if inputs > 2 * L2_BYTES:
        return (f"inputs larger than L2 (X + int8 W = {inputs / 1e6:.0f} MB > "
                f"2 x 126 MB): no flush")
    return "flushed (512 MB write) before every timed step"


def needs_flush(wl) -> bool:
    return 2 * wl.s * wl.h + wl.h * wl.o <= 2 * L2_BYTES


def parallelism(world: int, args) -> str:
    if world <= 1:
        return "single"
    return f"{'column blocks' if args.parallel == 'columns' else 'replicas'} x{world}"


def workload_config(wl, world: int, args) -> dict:
    """The line's `config`: the same keys and values in both arms."""
    return {"workload": wl.name, "s": wl.s, "h": wl.h, "o": wl.o,
            "alpha": alpha_json(wl.alpha), "outlier_cols": wl.n_outlier_cols,
            "parallelism": parallelism(world, args),
            "scales": {"x": args.x_scale, "w": args.w_scale},
            "l2": l2_policy(wl)}


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons with NVML in a thread, as fast
    as NVML answers (a short sleep between reads)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown",
               0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap",
               0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting"}

    def __init__(self, index: int, period_s: float = 0.0002):
        self.samples = []
        self.ok = False
        self.period = period_s
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(
                self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()
            self._t = None

    def summary(self, t0: float, t1: float):
        if not self.ok or not self.samples:
            return None
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        use = inside if inside else self.samples
        mhz = statistics.median(s[1] for s in use)
        bits = 0
        for s in use:
            bits |= s[2]
        reasons = sorted(n for b, n in self.REASONS.items()
                         if bits & b and n != "gpu_idle")
        return {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(inside), "window_s": round(t1 - t0, 4),
                "window": "timed region" if inside else "whole run"}


# ------------------------------------------------------------ CPU oracle

def fp16_matmul_ms(X, W, dev, flush, K, Wm, world):
    """The same product in plain fp16 through cuBLAS (fp32 accumulation),
    timed like the step: the reference the pages quote their speedups
    against (Appendix D, Table 5)."""
    import torch
    torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = False
    Xd = torch.from_numpy(X).to(dev)
    Wd = torch.from_numpy(W).to(dev)
    out = torch.empty((X.shape[0], W.shape[1]), dtype=torch.float16, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(Wm):
        if flush is not None:
            flush.fill_(1)
        torch.matmul(Xd, Wd, out=out)
    ts = []
    torch.cuda.synchronize()
    for k in range(K):
        if flush is not None:
            flush.fill_(k & 0xFF)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        torch.matmul(Xd, Wd, out=out)
        b.record(stream)
        ts.append((a, b))
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ts) / K
    del Xd, Wd, out
    torch.cuda.empty_cache()
    return max_over_ranks(ms, world, dev)


def with_alpha(wl, args, alpha=None):
    """The workload with `alpha` (else --alpha) in place of its threshold."""
    a = alpha if alpha is not None else args.alpha
    return wl if a is None else dataclasses.replace(wl, alpha=a)


def split_spec(spec: str):
    """'name' or 'name@alpha' -> (name, alpha or None)."""
    name, _, a = spec.partition("@")
    return name, (float(a) if a else None)


def alpha_json(a: float):
    return a if a != float("inf") else "inf"


def oracle_rows_for(wl, X, Wq, aw, budget_s: float, x_tensor: bool = False):
    """Number of rows of a sample that the oracle runs in about budget_s
    (grown by 4x until a run takes a quarter of the budget; the outlier set
    is always computed over all rows, a fixed cost)."""
    import oracle
    order = np.random.default_rng(123).permutation(wl.s)

    def timed(n):
        rows = np.sort(order[:n])
        t = time.perf_counter()
        oracle.matmul(X, Wq, aw, wl.alpha, rows=rows, x_tensor=x_tensor)
        return time.perf_counter() - t

    n = min(wl.s, 4)
    el = timed(n)
    while el < budget_s / 4 and n < wl.s:
        n = min(wl.s, n * 4)
        el = timed(n)
    return int(max(1, min(wl.s, n * budget_s / max(el, 1e-6)))), order


def cpu_oracle_run(wl, X, Wq, aw, budget_s: float, x_tensor: bool = False):
    """Time the oracle once on a row sample sized to about budget_s."""
    import oracle
    n, order = oracle_rows_for(wl, X, Wq, aw, budget_s, x_tensor)
    rows = np.sort(order[:n])
    t = time.perf_counter()
    oracle.matmul(X, Wq, aw, wl.alpha, rows=rows, x_tensor=x_tensor)
    el = time.perf_counter() - t
    tops = 2.0 * n * wl.h * wl.o / el / 1e12
    return {"value": tops, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{n} of {wl.s} rows x all {wl.o} columns of "
                      f"{wl.name} (outlier set over all rows), {el:.1f} s"}


# ---------------------------------------------------------------- ranks

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if _cuda_ok() else "gloo"
        dist.init_process_group(backend=backend,
                                timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def _cuda_ok():
    import torch
    return torch.cuda.is_available()


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def finish(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_command(n: int, argv) -> list:
    """torchrun command that runs this script on n local ranks."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            "--nproc-per-node", str(n), "--master-addr", "127.0.0.1",
            "--master-port", str(_free_port()), os.path.abspath(__file__)] + list(argv)


def check_world(n_gpus: int, env) -> str:
    """'run' (this process is one of the n ranks), 'launch' (start n ranks
    with torchrun) or an error message when --gpus and the launcher disagree."""
    world = env.get("WORLD_SIZE")
    if world is None:
        return "run" if n_gpus == 1 else "launch"
    if int(world) != n_gpus:
        return (f"--gpus {n_gpus} but WORLD_SIZE={world}: launch one rank per "
                f"GPU with torchrun --nproc-per-node {n_gpus}")
    return "run"


# ------------------------------------------------------------- our path

def layer_roofline_ms(wl, peaks) -> float:
    """Roofline time of the whole layer: the slower of the int8 tensor peak
    and the compulsory bytes at the measured HBM bandwidth."""
    p_int8 = 2.0 * peaks["bf16_tflops"] * 1e12
    return max(wl.int8_ops / p_int8, wl.compulsory_bytes / (peaks["hbm_gbs"] * 1e9)) * 1e3


def bench_workload(name, args, world, rank, local, K, Wm, headline: bool):
    """Time one workload; returns the per-shape entry (the headline's keys
    are the line's top-level keys)."""
    import torch
    from mixed_precision_int8_b200 import binding
    from mixed_precision_int8_b200.column_parallel import shard_columns

    dev = torch.device("cuda", local)
    name, alpha_override = split_spec(name)
    wl, X, cols, W = workloads.make_inputs(name)
    wl = with_alpha(wl, args, alpha_override)
    s, h, o_layer = wl.s, wl.h, wl.o
    columns = args.parallel == "columns" and world > 1
    col0, o = shard_columns(o_layer, world, rank) if columns else (0, o_layer)
    if o == 0:
        raise SystemExit(f"rank {rank} has no columns of {o_layer} at world {world}")
    Xd = torch.from_numpy(X).to(dev)
    Wd = torch.from_numpy(W).to(dev)
    x_mode = SCALE_MODES[args.x_scale]
    pw = binding.llmint8_prepare_weight_cols(Wd, col0, o, w_scale=SCALE_MODES[args.w_scale])
    torch.cuda.synchronize()
    del Wd
    out = torch.empty((s, o), dtype=torch.float16, device=dev)
    ws = binding.Workspace(s, h, o, device=dev, max_outliers=args.max_outliers)
    flush = (torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
             if needs_flush(wl) else None)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        binding.llmint8_matmul(Xd, pw, wl.alpha, out=out, workspace=ws,
                               events=ev, x_scale=x_mode)

    for _ in range(Wm):
        if flush is not None:
            flush.fill_(1)
        step()
    torch.cuda.synchronize()
    launches_per_step = binding.llmint8_matmul.last_launches
    n_outliers, _, _ = binding.llmint8_read_outlier_tiles(ws, tiles=False)  # |O|

    def timed_steps(n, with_kernel_events: bool):
        """n steps timed with CUDA events on the launching stream: where the
        workload needs an L2 flush, each step between its own events with
        the flush outside them; otherwise the n steps back to back between
        one pair. With with_kernel_events the library also records events
        around its GEMM/decode kernel, which turns off that launch's overlap
        with the kernel before it, so the step time is taken without them."""
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        stops = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        g0 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        g1 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        barrier(world)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        if flush is None and not with_kernel_events:
            # nothing to keep out of the timing: the n steps run back to
            # back, as consecutive layers do, between one pair of events
            starts[0].record(stream)
            for _ in range(n):
                step(None)
            stops[0].record(stream)
        else:
            for k in range(n):
                if flush is not None:
                    flush.fill_(k & 0xFF)
                starts[k].record(stream)
                step((g0[k], g1[k]) if with_kernel_events else None)
                stops[k].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        t1 = time.perf_counter()
        if flush is None and not with_kernel_events:
            step_ms = [starts[0].elapsed_time(stops[0]) / n] * n
        else:
            step_ms = [a.elapsed_time(b) for a, b in zip(starts, stops)]
        kern_ms = ([binding.event_elapsed_ms(a, b) for a, b in zip(g0, g1)]
                   if with_kernel_events else None)
        return step_ms, kern_ms, t0, t1

    # headline: exactly K steps; per-shape entries: at least
    # PER_SHAPE_MIN_STEPS
    n_steps = K if headline else max(K, PER_SHAPE_MIN_STEPS)
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    step_ms, _, t_wall0, t_wall1 = timed_steps(n_steps, False)
    clock_sum = clocks.summary(t_wall0, t_wall1) if clocks else None
    ms_per_step = max_over_ranks(sum(step_ms) / n_steps, world, dev)
    # the dominant kernel's own time, right after (same conditions)
    _, gemm_ms, g_t0, g_t1 = timed_steps(n_steps, True)
    gemm_ms_avg = sum(gemm_ms) / n_steps
    kernel_clocks = clocks.summary(g_t0, g_t1) if clocks else None
    # then a longer window of the same steps (at least SOAK_MIN_S): how the
    # layer holds up under sustained load, reported beside the K-step numbers
    soak_ms, soak_t0, soak_t1 = [], None, None
    if headline and not args.no_soak:
        # the same number of repetitions on every rank (each has barriers)
        reps = int(max_over_ranks(
            float(int(SOAK_MIN_S / max(1e-4, t_wall1 - t_wall0)) + 1), world, dev))
        soak_t0 = time.perf_counter()
        for _ in range(reps):
            ms, _, _, soak_t1 = timed_steps(n_steps, False)
            soak_ms += ms
    if clocks:
        clocks.stop()
    status_bits = binding.llmint8_read_device_status(ws)

    # end to end through the host-buffer entry point
    e2e_ms = None
    if not args.no_e2e:
        Xh = torch.from_numpy(X).pin_memory()
        outh = torch.empty((s, o), dtype=torch.float16).pin_memory()
        wsh = binding.Workspace(s, h, o, device=dev, host=True,
                                max_outliers=args.max_outliers)
        for _ in range(max(1, Wm)):
            binding.llmint8_matmul_host(Xh, pw, wl.alpha, outh, wsh, x_scale=x_mode)
        e_ms = []
        barrier(world)
        torch.cuda.synchronize()
        for k in range(n_steps):
            if flush is not None:
                flush.fill_(k & 0xFF)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            binding.llmint8_matmul_host(Xh, pw, wl.alpha, outh, wsh, x_scale=x_mode)
            b.record(stream)
            b.synchronize()
            e_ms.append(a.elapsed_time(b))
        barrier(world)
        e2e_ms = max_over_ranks(sum(e_ms) / n_steps, world, dev)
        del wsh, Xh, outh
    fp16_ms = None if args.no_fp16_ref else fp16_matmul_ms(
        X, np.ascontiguousarray(W[:, col0:col0 + o]), dev, flush, n_steps, Wm, world)

    ops = 2.0 * s * h * o  # this rank's
    # whole-job work: every replica's layer, or the one layer split in blocks
    job_ops = 2.0 * s * h * o_layer * (1 if columns else world)
    value = job_ops / (ms_per_step * 1e-3) / 1e12
    e2e_value = None if e2e_ms is None else job_ops / (e2e_ms * 1e-3) / 1e12
    peaks = measured_peaks()
    decode = s <= binding.llmint8_decode_max_rows()
    if decode:
        kernel = "k_decode_i8"
        # int8 weight + int8 rows + fp16 output + scales
        algo_bytes = h * o + s * h + 2 * s * o + 4 * (s + o)
        achieved = algo_bytes / (gemm_ms_avg * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                "kernel": kernel, "algorithmic_bytes": algo_bytes,
                "peak_source": f"hbm_gbs ({peaks['source']})"}
    else:
        kernel = ("k_gemm_i8_pair"
                  if binding.llmint8_prefill_kernel(s, h, o) == binding.PATH_PREFILL_PAIR
                  else "k_gemm_i8_fused")
        peak = 2.0 * peaks["bf16_tflops"]
        achieved = ops / (gemm_ms_avg * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "kernel": kernel,
                "peak_source": "bf16_tflops x 2 (nominal int8/bf16 dense "
                               f"ratio 4.5/2.25), {peaks['source']}"}
    # the committed DRAM counters are for the workload's own threshold
    roof["traffic"] = recorded_traffic(wl.name, kernel) if alpha_override is None else None
    roof["kernel_ms"] = gemm_ms_avg
    roof["kernel_timing"] = ("CUDA events recorded by the library around "
                             "this kernel, averaged over a second pass of the "
                             "same steps right after the timed one")
    roof["kernel_clocks"] = kernel_clocks
    entry = {
        "workload": wl.name if alpha_override is None else f"{wl.name}@alpha={alpha_override:g}",
        "outliers": n_outliers, "value": value, "unit": UNIT,
        "scaling": "strong" if columns else "weak",
        "ms_per_step": ms_per_step, "steps": n_steps,
        # the roofline of this rank's share of the layer
        "step_roofline_frac": layer_roofline_ms(dataclasses.replace(wl, o=o), peaks) / ms_per_step,
        "config": workload_config(wl, world, args),
        "e2e": None if e2e_value is None else {
            "value": e2e_value, "unit": UNIT,
            "h2d_bytes_per_step": 2 * s * h,
            "d2h_bytes_per_step": 2 * s * o},
        "gpu_launches": launches_per_step * n_steps,
        "roofline": roof,
        "device_status": status_bits,
        "fp16_matmul": None if fp16_ms is None else {
            "ms_per_step": fp16_ms, "speedup": fp16_ms / ms_per_step,
            "what": "torch.matmul of the fp16 X and W (cuBLAS, fp32 accumulation), "
                    "timed like the step: the pages' Table 5 baseline"},
        "clocks": clock_sum,
    }
    if headline and soak_t1 is not None:
        soak = clocks.summary(soak_t0, soak_t1) if clocks else {}
        soak = dict(soak or {})
        soak["ms_per_step"] = sum(soak_ms) / len(soak_ms)
        soak["value"] = job_ops / (soak["ms_per_step"] * 1e-3) / 1e12
        soak["steps"] = len(soak_ms)
        soak["what"] = ("the same steps back to back for at least "
                        f"{SOAK_MIN_S} s after the timed ones (sustained load; "
                        "the power cap may lower the clock)")
        entry["clocks_soak"] = soak
    if headline and rank == 0 and world == 1 and not args.no_cpu_baseline:
        Wq = pw.wq.cpu().numpy()
        aw = pw.aw.cpu().numpy()
        entry["cpu_baseline"] = cpu_oracle_run(wl, X, Wq, aw, args.cpu_seconds,
                                               x_tensor=args.x_scale == "tensor")
    del pw, ws, out, Xd, flush
    torch.cuda.empty_cache()
    return entry


def run_ours(args, world, rank, local):
    import torch
    from mixed_precision_int8_b200 import binding, build

    torch.cuda.set_device(local)
    build.build()
    binding.load_library()
    K, Wm = args.steps, args.warmup
    head = bench_workload(args.workload, args, world, rank, local, K, Wm, True)
    shapes = [] if args.per_shape == "none" else [
        n for n in (args.per_shape.split(",") if args.per_shape else DEFAULT_PER_SHAPE)
        if n and n != args.workload]
    per_shape = [bench_workload(n, args, world, rank, local, K, Wm, False) for n in shapes]
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": Wm, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": head["scaling"], "vs_baseline": None,
        "dtype": "i8", "data": "synthetic (seeded, OPT-shaped outliers)",
        "config": head["config"], "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"], "roofline": head["roofline"],
        "step_roofline_frac": head["step_roofline_frac"],
        "device_status": head["device_status"],
        "fp16_matmul": head["fp16_matmul"], "clocks": head["clocks"],
    }
    for k in ("clocks_soak", "cpu_baseline"):
        if k in head:
            line[k] = head[k]
    line["per_shape"] = per_shape
    return line


# ------------------------------------------------------ reference (oracle)

def run_reference(args, world):
    """The CPU oracle on the host cores: each step one row sample of the
    workload (the same sample every step), sized once during warm-up so that
    warm-up plus K steps take about --cpu-seconds."""
    import oracle
    wl, X, cols, W = workloads.make_inputs(args.workload)
    wl = with_alpha(wl, args)
    Wq, aw = oracle.prepare_weight(W, tensor=args.w_scale == "tensor")
    x_tensor = args.x_scale == "tensor"
    per_step = max(0.2, args.cpu_seconds / max(1, args.steps + args.warmup))
    n, order = oracle_rows_for(wl, X, Wq, aw, per_step, x_tensor)
    rows = np.sort(order[:n])

    def one():
        t = time.perf_counter()
        oracle.matmul(X, Wq, aw, wl.alpha, rows=rows, x_tensor=x_tensor)
        return time.perf_counter() - t

    for _ in range(args.warmup):
        one()
    secs = [one() for _ in range(args.steps)]
    ms = 1e3 * sum(secs) / len(secs)
    value = 2.0 * n * wl.h * wl.o / (ms * 1e-3) / 1e12
    sample = (f"{n} of {wl.s} rows x all {wl.o} columns of {wl.name} per step "
              f"(outlier set over all rows); {args.steps} steps in {sum(secs):.1f} s")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8 codes, fp64 accumulation",
        "data": "synthetic (seeded, OPT-shaped outliers)",
        "config": workload_config(wl, world, args),
        "cpu_baseline": {"value": value, "unit": UNIT,
                         "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=list(workloads.WORKLOADS))
    ap.add_argument("--per-shape", default=None,
                    help="comma-separated workloads timed after the headline "
                         "(default: the other OPT shapes; 'none' for none)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp16-ref", action="store_true",
                    help="skip timing the plain fp16 cuBLAS product for context")
    ap.add_argument("--no-soak", action="store_true",
                    help="skip the sustained-load window (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end timing (profiling runs)")
    ap.add_argument("--max-outliers", type=int, default=0,
                    help="outlier columns the workspace holds (0: h, any alpha)")
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "columns"],
                    help="N > 1: independent replicas (weak scaling) or one layer "
                         "split into blocks of output columns (strong scaling)")
    ap.add_argument("--alpha", type=float, default=None,
                    help="outlier threshold instead of the workload's (inf: no "
                         "decomposition, pure vector-wise int8)")
    ap.add_argument("--x-scale", default="row", choices=["row", "tensor"],
                    help="absmax per row of X (the method) or one per tensor")
    ap.add_argument("--w-scale", default="column", choices=["column", "tensor"],
                    help="absmax per column of W (the method) or one per tensor")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.per_shape not in (None, "none"):
        bad = [n for n in args.per_shape.split(",")
               if n and split_spec(n)[0] not in workloads.WORKLOADS]
        if bad:
            ap.error(f"unknown workloads in --per-shape: {bad}")
    return args


def main():
    args = parse_args()
    plan = check_world(args.gpus, os.environ)
    if plan == "launch":
        sys.exit(subprocess.call(launch_command(args.gpus, sys.argv[1:])))
    if plan != "run":
        print(plan, file=sys.stderr)
        sys.exit(2)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        # rank 0 alone times the CPU oracle; other ranks exit without work
        if int(os.environ.get("RANK", "0")) != 0:
            return
        print(json.dumps(run_reference(args, world)), flush=True)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        line = run_ours(args, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        finish(world)


if __name__ == "__main__":
    main()
