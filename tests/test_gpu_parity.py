"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact: outlier flags / list / count, row scales, int8 row codes, weight
scales and codes, the fp16 outlier tiles and the int32 accumulators.
Within |gpu - oracle| <= 2e-3 (1 + |oracle|): the fp16 output.

Small cases run the oracle on every output; the five OPT-shaped workloads
run it on seeded row x column samples (each output element of the method
depends only on its row of X, the global outlier set and its weight column).
"""
import functools
import math

import numpy as np
import pytest
import torch

import oracle
from mixed_precision_int8_b200 import binding, build, workloads
from tests.parity_utils import (assert_close_fp16, gpu_matmul, gpu_prepare,
                                oracle_prepared, oracle_prepared_by_blocks,
                                sample_cols, sample_rows,
                                to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    binding.load_library()
    yield


# (s, h, o, outlier columns, alpha) — ragged tails in every dimension
SMALL = [
    (16, 256, 256, (7, 200), 6.0),
    (1, 128, 256, (3,), 6.0),
    (3, 144, 48, (0, 143), 6.0),
    (8, 512, 784, (5, 6, 7), 6.0),
    (17, 256, 272, (100,), 6.0),
    (129, 272, 784, (1, 2, 270), 6.0),
    (300, 1024, 528, tuple(range(0, 1024, 64)), 6.0),      # |O| = 16
    (200, 1040, 256, tuple(range(3, 1040, 61)), 6.0),      # |O| = 17
    (64, 256, 512, (9, 99), math.inf),                    # decomposition off
    (40, 128, 256, (), 0.0),                               # every column out
    (256, 4096, 256, (11, 4000), 6.0),
    (9, 1040, 256, tuple(range(3, 1040, 61)), 6.0),        # decode, |O| = 17
    (12, 256, 272, (), 0.0),                               # decode, |O| = h
]


def _small_inputs(case, seed=0):
    s, h, o, cols, alpha = case
    rng = np.random.default_rng(1000 + seed + s + h + o)
    X = workloads.random_x(rng, s, h, outlier_cols=cols, lo=6.0, hi=60.0)
    W = workloads.random_w(rng, h, o, sigma=0.02)
    return X, W, alpha


def _check_quantize_rows(X, alpha):
    Xq, ax, flags, idx, n = binding.llmint8_quantize_rows(to_dev(X), alpha)
    torch.cuda.synchronize()
    f_ref, idx_ref, n_ref = oracle.detect_outliers(X, alpha)
    assert int(n.item()) == n_ref
    assert np.array_equal(flags.cpu().numpy(), f_ref)
    assert np.array_equal(idx.cpu().numpy()[:n_ref], idx_ref)
    Xq_ref, ax_ref = oracle.quantize_rows(X, f_ref)
    assert np.array_equal(ax.cpu().numpy(), ax_ref)
    assert np.array_equal(Xq.cpu().numpy(), Xq_ref)
    return f_ref, idx_ref


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}a{c[4]}")
def test_quantize_rows_bit_exact_small(case):
    X, _, alpha = _small_inputs(case)
    _check_quantize_rows(X, alpha)


def test_quantize_rows_special_rows():
    rng = np.random.default_rng(5)
    X = workloads.random_x(rng, 12, 256, outlier_cols=(4,), row_frac=1.0)
    X[3] = 0                      # all-zero row: ax = 0, codes 0
    X[5] = 0
    X[5, 4] = 20.0                # only the outlier entry nonzero
    X[7, 9] = np.float16(6.0)     # exactly alpha: column 9 becomes outlier
    X[8, 10] = np.float16(5.9960938)
    X[9, :] = np.float16(-3.0)    # constant row: all codes -127
    X[9, 4] = 8.0
    X[10, 11] = np.float16(127.0 / 16.0)   # tie cases of the rounding rule
    X[10, 12:20] = (np.arange(8) * 2 + 1).astype(np.float16) / np.float16(32)
    f, idx = _check_quantize_rows(X, 6.0)
    assert 9 in idx.tolist() and 10 not in idx.tolist()


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}")
def test_prepare_weight_bit_exact_small(case):
    _, W, _ = _small_inputs(case)
    W[:, 1] = 0  # a zero column
    pw, _ = gpu_prepare(W)
    torch.cuda.synchronize()
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    assert np.array_equal(pw.aw.cpu().numpy(), aw_ref)
    assert np.array_equal(pw.wq.cpu().numpy(), Wq_ref)


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}a{c[4]}")
def test_matmul_small_cases(case):
    X, W, alpha = _small_inputs(case)
    s = X.shape[0]
    pw, _ = gpu_prepare(W)
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    ref, ci_ref = oracle.matmul(X, Wq_ref, aw_ref, alpha, want_ci=True)
    paths = [1, 2] if s <= 16 else [1]
    for path in paths:
        out, ci, ws = gpu_matmul(X, pw, alpha, path=path, want_ci=True)
        assert np.array_equal(ci, ci_ref), f"int32 accumulators, path {path}"
        assert_close_fp16(out, ref, f"out path {path}")
    # fp16 outlier tiles of the last call, bit-exact
    f_ref, idx_ref, n_ref = oracle.detect_outliers(X, alpha)
    n, XO, WO = binding.llmint8_read_outlier_tiles(ws)
    assert n == n_ref
    assert np.array_equal(XO.numpy().view(np.uint16),
                          np.ascontiguousarray(X[:, idx_ref]).view(np.uint16))
    WO_ref = oracle.outlier_weights(Wq_ref, aw_ref, idx_ref)
    assert np.array_equal(WO.numpy().view(np.uint16), WO_ref.view(np.uint16))


PLAIN_CASES = [c for c in SMALL if c[0] > 16] + [
    (300, 1040, 15376, tuple(range(3, 1040, 61)), 6.0),   # more tiles than SMs
]


@pytest.mark.parametrize("keep_fp16", [False, True], ids=["w_from_int8", "w_fp16"])
@pytest.mark.parametrize("case", PLAIN_CASES, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}a{c[4]}")
def test_every_place_of_the_outlier_row_build_matches_the_oracle(case, keep_fp16):
    """The fp16 outlier rows of W built by the GEMM's CTAs in shares (the
    default), by the activation fix-up before the GEMM, and by every GEMM
    CTA on its own (what a CTA falls back to when its peers are not
    resident): each against the oracle, and bit for bit against each other."""
    X, W, alpha = _small_inputs(case, seed=17)
    pw, _ = gpu_prepare(W, keep_fp16=keep_fp16)
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    ref, ci_ref = oracle.matmul(X, Wq_ref, aw_ref, alpha, want_ci=True,
                                W16=W if keep_fp16 else None)
    f_ref, idx_ref, n_ref = oracle.detect_outliers(X, alpha)
    WO_ref = (np.ascontiguousarray(W[idx_ref, :]) if keep_fp16
              else oracle.outlier_weights(Wq_ref, aw_ref, idx_ref))
    outs = []
    for mode in (binding.WO_SHARED, binding.WO_BEFORE_GEMM, binding.WO_EACH_CTA):
        out, ci, ws = gpu_matmul(X, pw, alpha, path=1, want_ci=True, wo_build=mode)
        assert np.array_equal(ci, ci_ref), f"int32 accumulators, wo_build={mode}"
        assert_close_fp16(out, ref, f"out wo_build={mode}")
        n, _, WO = binding.llmint8_read_outlier_tiles(ws)
        assert n == n_ref
        assert np.array_equal(WO.numpy().view(np.uint16), WO_ref.view(np.uint16)), mode
        outs.append(out)
    for o in outs[1:]:
        assert np.array_equal(outs[0].view(np.uint16), o.view(np.uint16))


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}a{c[4]}")
def test_matmul_small_cases_with_fp16_outlier_rows(case):
    """The caller's fp16 W supplies the outlier rows of W: output against the
    oracle in the same mode, and the WO tiles equal W's rows bit for bit."""
    X, W, alpha = _small_inputs(case, seed=5)
    s = X.shape[0]
    pw, Wd = gpu_prepare(W, keep_fp16=True)
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    ref, ci_ref = oracle.matmul(X, Wq_ref, aw_ref, alpha, want_ci=True, W16=W)
    for path in ([1, 2] if s <= 16 else [1]):
        out, ci, ws = gpu_matmul(X, pw, alpha, path=path, want_ci=True)
        assert np.array_equal(ci, ci_ref), f"int32 accumulators, path {path}"
        assert_close_fp16(out, ref, f"out path {path}")
        f_ref, idx_ref, n_ref = oracle.detect_outliers(X, alpha)
        n, _, WO = binding.llmint8_read_outlier_tiles(ws)
        assert n == n_ref
        assert np.array_equal(WO.numpy().view(np.uint16),
                              np.ascontiguousarray(W[idx_ref, :]).view(np.uint16)), path


@pytest.mark.parametrize("name", ["opt6.7b_attn_prefill", "opt175b_decode"])
def test_workload_matmul_with_fp16_outlier_rows(name):
    wl, X, cols, W = workloads.make_inputs(name)
    pw, Wd = gpu_prepare(W, keep_fp16=True)
    rows = sample_rows(wl.s, 48)
    c = sample_cols(wl.o, 512)
    Wq_ref, aw_ref = oracle_prepared(W, c)
    ref = oracle.matmul(X, Wq_ref, aw_ref, wl.alpha, rows=rows,
                        W16=np.ascontiguousarray(W[:, c]))
    out, _, _ = gpu_matmul(X, pw, wl.alpha)
    assert_close_fp16(out[np.ix_(rows, c)], ref)
    del Wd, pw
    torch.cuda.empty_cache()


# More output tiles than SMs, with a ragged last wave, checked element by
# element: ragged k (h = 1040) and o (60 full tiles + 16 columns), |O| = 17
# (outlier rows beyond the shared-memory ones), an 8-row case forced onto
# the prefill kernel, and two full waves plus two tiles.
MANY_TILES = [
    (300, 1040, 15376, tuple(range(3, 1040, 61)), 6.0),
    (8, 512, 40960, (5, 300), 6.0),
    (129, 4096, 38144, (11, 4000), 6.0),
]


@pytest.mark.parametrize("case", MANY_TILES, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}")
def test_matmul_many_tiles_bit_exact_int32(case):
    X, W, alpha = _small_inputs(case, seed=21)
    pw, _ = gpu_prepare(W)
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    ref, ci_ref = oracle.matmul(X, Wq_ref, aw_ref, alpha, want_ci=True)
    for rep in range(2):  # the second call reuses the workspace
        out, ci, _ = gpu_matmul(X, pw, alpha, path=1, want_ci=True)
        assert np.array_equal(ci, ci_ref), f"int32 accumulators, call {rep}"
        assert_close_fp16(out, ref, f"out, call {rep}")


# Tensor-wise baselines ("Quantization Primitives"; Table 1 "Int8 absmax"):
# one absmax for all of X and/or all of W, on the same kernels.
TENSOR_CASES = [SMALL[i] for i in (0, 2, 4, 5, 6, 9, 11, 12)]
VW, TW = binding.SCALE_VECTORWISE, binding.SCALE_TENSORWISE


@pytest.mark.parametrize("case", TENSOR_CASES, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}a{c[4]}")
def test_quantize_rows_tensorwise_bit_exact(case):
    X, _, alpha = _small_inputs(case, seed=11)
    if X.shape[0] > 2:
        X[1] = 0  # an all-zero row takes the tensor constant too
    Xq, ax, flags, idx, n = binding.llmint8_quantize_rows(to_dev(X), alpha, x_scale=TW)
    torch.cuda.synchronize()
    f_ref, _, n_ref = oracle.detect_outliers(X, alpha)
    assert int(n.item()) == n_ref
    assert np.array_equal(flags.cpu().numpy(), f_ref)
    Xq_ref, ax_ref = oracle.quantize_rows(X, f_ref, tensor=True)
    assert np.array_equal(ax.cpu().numpy(), ax_ref)
    assert np.array_equal(Xq.cpu().numpy(), Xq_ref)


@pytest.mark.parametrize("case", TENSOR_CASES, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}")
def test_prepare_weight_tensorwise_bit_exact(case):
    _, W, _ = _small_inputs(case, seed=12)
    W[:, 1] = 0
    pw = binding.llmint8_prepare_weight(to_dev(W), w_scale=TW)
    torch.cuda.synchronize()
    Wq_ref, aw_ref = oracle.prepare_weight(W, tensor=True)
    assert np.array_equal(pw.aw.cpu().numpy(), aw_ref)
    assert np.array_equal(pw.wq.cpu().numpy(), Wq_ref)


@pytest.mark.parametrize("modes", [(TW, VW), (VW, TW), (TW, TW)], ids=["xT", "wT", "xTwT"])
@pytest.mark.parametrize("case", TENSOR_CASES, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}a{c[4]}")
def test_matmul_tensorwise_small(case, modes):
    x_mode, w_mode = modes
    X, W, alpha = _small_inputs(case, seed=13)
    s = X.shape[0]
    pw = binding.llmint8_prepare_weight(to_dev(W), w_scale=w_mode)
    Wq_ref, aw_ref = oracle.prepare_weight(W, tensor=(w_mode == TW))
    ref, ci_ref = oracle.matmul(X, Wq_ref, aw_ref, alpha, want_ci=True,
                                x_tensor=(x_mode == TW))
    for path in ([1, 2] if s <= 16 else [1]):
        ws = binding.Workspace(s, pw.h, pw.o)
        ci = torch.full((s, pw.o), -7, dtype=torch.int32, device="cuda")
        out = binding.llmint8_matmul(to_dev(X), pw, alpha, workspace=ws, ci=ci,
                                     path=path, x_scale=x_mode)
        torch.cuda.synchronize()
        assert binding.llmint8_read_device_status(ws) == 0
        assert np.array_equal(ci.cpu().numpy(), ci_ref), f"int32 accumulators, path {path}"
        assert_close_fp16(out.cpu().numpy(), ref, f"out path {path}")


@pytest.mark.parametrize("name", ["opt6.7b_attn_prefill", "opt175b_decode"])
def test_workload_matmul_tensorwise(name):
    """Both tensors tensor-wise at full size, on sampled rows and columns.
    The oracle's weight constant is taken over the sampled columns plus the
    column that holds W's largest magnitude, so it is W's own constant."""
    wl, X, cols, W = workloads.make_inputs(name)
    Wd = to_dev(W)
    pw = binding.llmint8_prepare_weight(Wd, w_scale=TW)
    del Wd
    rows = sample_rows(wl.s, 48)
    c = sample_cols(wl.o, 512)
    jmax = int(np.abs(W.astype(np.float32)).max(axis=0).argmax())
    cw = np.append(c, jmax)
    Wq_ref, aw_ref = oracle.prepare_weight(np.ascontiguousarray(W[:, cw]), tensor=True)
    ref, ci_ref = oracle.matmul(X, Wq_ref[:-1], aw_ref[:-1], wl.alpha, rows=rows,
                                want_ci=True, x_tensor=True)
    ws = binding.Workspace(wl.s, pw.h, pw.o)
    ci = torch.empty((wl.s, pw.o), dtype=torch.int32, device="cuda")
    out = binding.llmint8_matmul(to_dev(X), pw, wl.alpha, workspace=ws, ci=ci, x_scale=TW)
    torch.cuda.synchronize()
    assert binding.llmint8_read_device_status(ws) == 0
    assert np.array_equal(pw.aw[c].cpu().numpy(), aw_ref[:-1])
    assert np.array_equal(pw.wq[c].cpu().numpy(), Wq_ref[:-1])
    assert np.array_equal(ci.cpu().numpy()[np.ix_(rows, c)], ci_ref)
    assert_close_fp16(out.cpu().numpy()[np.ix_(rows, c)], ref)
    del pw, ci, out, ws
    torch.cuda.empty_cache()


# rows too long for a shared-memory stage of the one-read pass (2h bytes plus
# its bitmask above the per-CTA budget): the column-pass + row-pass kernels
LONG_H = 108544


def test_long_rows_quantize_bit_exact_and_empty_input():
    rng = np.random.default_rng(31)
    X = workloads.random_x(rng, 40, LONG_H, outlier_cols=(5, 70000, LONG_H - 1))
    _check_quantize_rows(X, 6.0)
    # s = 0: nothing to quantise, an empty outlier set
    Xq, ax, flags, idx, n = binding.llmint8_quantize_rows(
        torch.empty((0, LONG_H), dtype=torch.float16, device="cuda"), 6.0)
    torch.cuda.synchronize()
    assert int(n.item()) == 0 and int(flags.sum().item()) == 0


@pytest.mark.parametrize("s", [40, 8])
def test_long_rows_matmul(s):
    rng = np.random.default_rng(32 + s)
    X = workloads.random_x(rng, s, LONG_H, outlier_cols=(3, 54321))
    W = workloads.random_w(rng, LONG_H, 256, sigma=0.01)
    pw, _ = gpu_prepare(W)
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    rows = sample_rows(s, 12)
    ref, ci_ref = oracle.matmul(X, Wq_ref, aw_ref, 6.0, rows=rows, want_ci=True)
    out, ci, _ = gpu_matmul(X, pw, 6.0, want_ci=True)
    assert np.array_equal(ci[rows], ci_ref)
    assert_close_fp16(out[rows], ref)


def test_matmul_zero_rows_and_zero_weight_columns():
    rng = np.random.default_rng(9)
    X = workloads.random_x(rng, 20, 256, outlier_cols=(4, 77), row_frac=1.0)
    X[2] = 0
    X[6] = 0
    X[6, 4] = -9.5
    W = workloads.random_w(rng, 256, 256)
    W[:, 3] = 0
    W[:, 200] = 0
    pw, _ = gpu_prepare(W)
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    ref, ci_ref = oracle.matmul(X, Wq_ref, aw_ref, 6.0, want_ci=True)
    out, ci, _ = gpu_matmul(X, pw, 6.0, want_ci=True)
    assert np.array_equal(ci, ci_ref)
    assert_close_fp16(out, ref)
    assert np.all(out[2] == 0) and np.all(out[:, 3] == 0)


def test_repeated_calls_are_deterministic_and_status_stays_clear():
    X, W, alpha = _small_inputs(SMALL[5])
    pw, _ = gpu_prepare(W)
    Xd = to_dev(X)
    ws = binding.Workspace(X.shape[0], pw.h, pw.o)
    outs = [binding.llmint8_matmul(Xd, pw, alpha, workspace=ws).cpu().numpy()
            for _ in range(3)]
    assert all(np.array_equal(outs[0].view(np.uint16), o.view(np.uint16))
               for o in outs[1:])
    assert binding.llmint8_read_device_status(ws) == 0


def test_workspace_state_carries_nothing_between_calls():
    """One workspace, calls with different outlier sets, row counts and
    paths in turn: each call's outlier set, codes and output are its own."""
    rng = np.random.default_rng(77)
    h, o = 1024, 256
    W = workloads.random_w(rng, h, o)
    pw, _ = gpu_prepare(W)
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    ws = binding.Workspace(300, h, o)
    xs = [workloads.random_x(rng, 300, h, outlier_cols=(5, 600)),
          workloads.random_x(rng, 300, h, outlier_cols=(77,)),
          workloads.random_x(rng, 8, h, outlier_cols=(900,)),   # decode path
          workloads.random_x(rng, 300, h),                       # no outliers
          workloads.random_x(rng, 131, h, outlier_cols=(5, 1000))]
    for X in xs + xs[:2]:
        out = binding.llmint8_matmul(to_dev(X), pw, 6.0, workspace=ws)
        n, XO, _ = binding.llmint8_read_outlier_tiles(ws, s=X.shape[0])
        f_ref, idx_ref, n_ref = oracle.detect_outliers(X, 6.0)
        assert n == n_ref
        assert np.array_equal(XO.numpy().view(np.uint16),
                              np.ascontiguousarray(X[:, idx_ref]).view(np.uint16))
        ref = oracle.matmul(X, Wq_ref, aw_ref, 6.0)
        assert_close_fp16(out.cpu().numpy(), ref)
    assert binding.llmint8_read_device_status(ws) == 0


def test_bounded_waits_run_out_report_and_leave_the_context_usable():
    """The wait self-test's mbarrier phase and flag are never satisfied: both
    waits give up after their limit, the status word says so, and the next
    call on the same workspace and stream runs normally."""
    X, W, alpha = _small_inputs(SMALL[0])
    pw, _ = gpu_prepare(W)
    ws = binding.Workspace(X.shape[0], pw.h, pw.o)
    binding.llmint8_wait_selftest(ws, limit_ns=2_000_000)
    bits = binding.llmint8_read_device_status(ws)
    assert bits == 0x20  # LLMINT8_DEV_TIMEOUT_SELFTEST, nothing else
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    out = binding.llmint8_matmul(to_dev(X), pw, alpha, workspace=ws)
    assert_close_fp16(out.cpu().numpy(), oracle.matmul(X, Wq_ref, aw_ref, alpha))
    assert binding.llmint8_read_device_status(ws) == 0


def test_host_buffer_entry_point_matches_device_path():
    X, W, alpha = _small_inputs(SMALL[4])
    s, h = X.shape
    pw, _ = gpu_prepare(W)
    dev_out, _, _ = gpu_matmul(X, pw, alpha)
    Xh = torch.from_numpy(X).pin_memory()
    outh = torch.empty((s, pw.o), dtype=torch.float16).pin_memory()
    ws = binding.Workspace(s, h, pw.o, host=True)
    binding.llmint8_matmul_host(Xh, pw, alpha, outh, ws)
    assert np.array_equal(outh.numpy().view(np.uint16), dev_out.view(np.uint16))


def test_invalid_arguments_with_real_buffers_enqueue_nothing():
    X, W, alpha = _small_inputs(SMALL[0])
    pw, _ = gpu_prepare(W)
    Xd = to_dev(X)
    ws = binding.Workspace(16, 256, 256)
    out = torch.zeros((16, 256), dtype=torch.float16, device="cuda")
    with pytest.raises(binding.Llmint8Error) as e:
        binding.llmint8_matmul(Xd, pw, -1.0, out=out, workspace=ws)
    assert e.value.code == -7
    small = binding.Workspace(16, 256, 256)
    small.nbytes -= 1
    with pytest.raises(binding.Llmint8Error) as e:
        binding.llmint8_matmul(Xd, pw, 6.0, out=out, workspace=small)
    assert e.value.code == -4
    with pytest.raises(ValueError):
        binding.llmint8_matmul(Xd[:, :240].contiguous(), pw, 6.0,
                               out=out, workspace=ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0


# ------------------------------------------------ the five OPT-shaped loads

@functools.lru_cache(maxsize=1)
def _workload(name):
    wl, X, cols, W = workloads.make_inputs(name)
    pw, Wd = gpu_prepare(W)
    del Wd
    torch.cuda.synchronize()
    return wl, X, cols, W, pw


@pytest.mark.parametrize("name", workloads.WORKLOAD_ORDER)
def test_workload_quantize_rows_bit_exact(name):
    wl, X, cols, W, pw = _workload(name)
    f_ref, idx_ref = _check_quantize_rows(X, wl.alpha)
    assert set(cols.tolist()) <= set(idx_ref.tolist())


@pytest.mark.parametrize("name", workloads.WORKLOAD_ORDER)
def test_workload_prepare_weight_bit_exact(name):
    wl, X, cols, W, pw = _workload(name)
    c = sample_cols(wl.o, 512) if wl.o > 4096 else None
    Wq_ref, aw_ref = oracle_prepared(W, c)
    wq = pw.wq.cpu().numpy()
    aw = pw.aw.cpu().numpy()
    if c is not None:
        wq, aw = wq[c], aw[c]
    assert np.array_equal(aw, aw_ref)
    assert np.array_equal(wq, Wq_ref)


@pytest.mark.parametrize("name", workloads.WORKLOAD_ORDER)
def test_workload_matmul(name):
    """Every output of the small workloads (s * o <= 2048 * 4096: the tiny
    case, the 6.7B attention projection and the 175B decode batch), and 256
    rows x every column of the two large FFN shapes."""
    wl, X, cols, W, pw = _workload(name)
    full = wl.s * wl.o <= 2048 * 4096
    rows = np.arange(wl.s) if full else sample_rows(wl.s, 256)
    c = np.arange(wl.o)
    Wq_ref, aw_ref = oracle_prepared_by_blocks(W)
    ref, ci_ref = oracle.matmul(X, Wq_ref, aw_ref, wl.alpha, rows=rows,
                                want_ci=True)
    paths = [0, 1] if wl.s <= 16 else [0]
    for path in paths:
        out, ci, ws = gpu_matmul(X, pw, wl.alpha, path=path, want_ci=True)
        assert np.array_equal(ci[np.ix_(rows, c)], ci_ref), f"Ci path {path}"
        assert_close_fp16(out[np.ix_(rows, c)], ref, f"out path {path}")
        # properties that hold for every output: finite, and rows with no
        # outlier entry and zero codes are exactly zero
        assert np.isfinite(out.astype(np.float32)).all()


# More than 16 outlier columns: the outlier tiles take the wide (K-major,
# zero-padded) layout and the prefill GEMM sums the fp16 outlier product on
# the tensor cores (kind::f16 into a second TMEM accumulator); the decode
# kernel reads the same layout on CUDA cores.
WIDE_CASES = [
    (300, 1024, 1024, tuple(range(5, 1024, 16)), 6.0),   # |O| = 64: one fp16 k-block
    (129, 1040, 784, tuple(range(3, 1040, 13)), 6.0),    # |O| = 80: a partial k-block
    (256, 512, 2048, (), 0.0),                           # every column out: |O| = 512
    (8, 1024, 512, tuple(range(5, 1024, 16)), 6.0),      # |O| = 64, decode and prefill
    # |O| = 97, filling over half of its span (the builders' dense schedule):
    # an aligned stretch (whole 8- and 16-column groups), a consecutive but
    # unaligned run, scattered columns and a partial group
    (200, 1024, 512, tuple(range(16, 80)) + tuple(range(83, 102)) + tuple(range(104, 200, 7)),
     6.0),
]


@pytest.mark.parametrize("keep_fp16", [False, True], ids=["w_from_int8", "w_fp16"])
@pytest.mark.parametrize("case", WIDE_CASES, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}a{c[4]}")
def test_wide_outlier_sets_on_the_tensor_cores(case, keep_fp16):
    X, W, alpha = _small_inputs(case, seed=23)
    s = X.shape[0]
    pw, _ = gpu_prepare(W, keep_fp16=keep_fp16)
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    ref, ci_ref = oracle.matmul(X, Wq_ref, aw_ref, alpha, want_ci=True,
                                W16=W if keep_fp16 else None)
    f_ref, idx_ref, n_ref = oracle.detect_outliers(X, alpha)
    assert n_ref > 16
    WO_ref = (np.ascontiguousarray(W[idx_ref, :]) if keep_fp16
              else oracle.outlier_weights(Wq_ref, aw_ref, idx_ref))
    XO_ref = np.ascontiguousarray(X[:, idx_ref])
    runs = [(1, m) for m in (binding.WO_SHARED, binding.WO_BEFORE_GEMM, binding.WO_EACH_CTA)]
    if s <= 16:
        runs.append((2, binding.WO_SHARED))
    for path, mode in runs:
        out, ci, ws = gpu_matmul(X, pw, alpha, path=path, want_ci=True, wo_build=mode)
        assert np.array_equal(ci, ci_ref), f"int32 accumulators, path {path} mode {mode}"
        assert_close_fp16(out, ref, f"out path {path} mode {mode}")
        n, XO, WO = binding.llmint8_read_outlier_tiles(ws)
        assert n == n_ref
        assert np.array_equal(XO.numpy().view(np.uint16), XO_ref.view(np.uint16))
        assert np.array_equal(WO.numpy().view(np.uint16), WO_ref.view(np.uint16))


def test_every_column_an_outlier_at_the_6p7b_shape():
    """alpha = 0 on the OPT-6.7B attention shape: |O| = h = 4096, so the
    layer is the fp16 product X.W^O on the tensor cores (64 fp16 k-blocks
    per tile) plus an all-zero int8 part; 64 sampled rows x every column."""
    wl, X, cols, W = workloads.make_inputs("opt6.7b_attn_prefill")
    pw, _ = gpu_prepare(W)
    rows = sample_rows(wl.s, 64)
    Wq_ref, aw_ref = oracle_prepared_by_blocks(W)
    ref, ci_ref = oracle.matmul(X, Wq_ref, aw_ref, 0.0, rows=rows, want_ci=True)
    assert not ci_ref.any()
    out, ci, ws = gpu_matmul(X, pw, 0.0, want_ci=True)
    assert not ci.any()
    assert_close_fp16(out[rows], ref)
    assert np.isfinite(out.astype(np.float32)).all()
    del pw, ws
    torch.cuda.empty_cache()
