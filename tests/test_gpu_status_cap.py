"""GPU tests of two workspace options of llmint8_matmul_ex.

Outlier cap (opts.max_outliers): a workspace sized for at most `cap` outlier
columns. A call whose |O| fits gives the method's output; one whose |O|
exceeds the cap writes no outlier tile, sets LLMINT8_DEV_OUTLIER_CAP and
returns the int8 part alone, which equals the method's output on X with its
outlier columns zeroed (those columns then have zero codes, the same row
scales and nothing to add). Both kernels, bit for bit on the int32
accumulators and within the fp16 tolerance on the output.

Host status word (opts.status_host): the call's last kernel copies the
workspace's status bits to a pinned host word, and the next call on it
returns LLMINT8_ERR_DEVICE_STATUS before enqueuing anything, with no
synchronisation. The bits come from the bounded-wait self-test, whose waits
nothing satisfies; no GPU is faulted.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from mixed_precision_int8_b200 import binding, build, workloads
from tests.parity_utils import assert_close_fp16, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    binding.load_library()
    yield


def _problem(s, h, o, cols, seed):
    rng = np.random.default_rng(seed)
    X = workloads.random_x(rng, s, h, outlier_cols=cols, lo=6.0, hi=60.0)
    W = workloads.random_w(rng, h, o)
    return X, W


CAP_CASES = [
    (300, 1024, 784, (3, 500, 777, 1000, 1001)),   # prefill, |O| = 5
    (9, 512, 272, (0, 17, 300, 301, 511)),          # decode, |O| = 5
    (200, 1040, 256, tuple(range(3, 1040, 61))),    # prefill, |O| = 17
]


@pytest.mark.parametrize("case", CAP_CASES, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}o{len(c[3])}")
def test_outlier_cap_fits_and_exceeded(case):
    s, h, o, cols = case
    X, W = _problem(s, h, o, cols, seed=s + h)
    n = len(cols)
    pw = binding.llmint8_prepare_weight(to_dev(W))
    Wq, aw = oracle.prepare_weight(W)
    ref, ci_ref = oracle.matmul(X, Wq, aw, 6.0, want_ci=True)
    X0 = X.copy()
    X0[:, list(cols)] = 0
    ref0 = oracle.matmul(X0, Wq, aw, 6.0)
    f_ref, idx_ref, n_ref = oracle.detect_outliers(X, 6.0)
    assert n_ref == n
    for path in ([1, 2] if s <= 16 else [1]):
        for cap, fits in ((n, True), (n + 3, True), (n - 1, False), (1, False)):
            ws = binding.Workspace(s, h, o, max_outliers=cap)
            assert ws.nbytes < binding.llmint8_workspace_size(s, h, o)
            ci = torch.full((s, o), -7, dtype=torch.int32, device="cuda")
            out = binding.llmint8_matmul(to_dev(X), pw, 6.0, workspace=ws, ci=ci, path=path)
            torch.cuda.synchronize()
            bits = binding.llmint8_read_device_status(ws)
            assert np.array_equal(ci.cpu().numpy(), ci_ref), (path, cap)
            k, XO, WO = binding.llmint8_read_outlier_tiles(ws, s=s)
            assert k == n
            if fits:
                assert bits == 0, (path, cap)
                assert_close_fp16(out.cpu().numpy(), ref, f"path {path} cap {cap}")
                assert np.array_equal(XO.numpy().view(np.uint16),
                                      np.ascontiguousarray(X[:, idx_ref]).view(np.uint16))
                WO_ref = oracle.outlier_weights(Wq, aw, idx_ref)
                assert np.array_equal(WO.numpy().view(np.uint16), WO_ref.view(np.uint16))
            else:
                assert bits == binding.DEV_OUTLIER_CAP, (path, cap, bits)
                assert XO is None and WO is None
                assert_close_fp16(out.cpu().numpy(), ref0, f"int8 part, path {path} cap {cap}")


def test_outlier_cap_on_the_6p7b_workload():
    """The OPT-6.7B-shaped layer in a workspace for 64 outlier columns: the
    same output as with the worst-case workspace, a fraction of its size."""
    wl, X, cols, W = workloads.make_inputs("opt6.7b_attn_prefill")
    pw = binding.llmint8_prepare_weight(to_dev(W))
    Xd = to_dev(X)
    full = binding.Workspace(wl.s, wl.h, wl.o)
    capped = binding.Workspace(wl.s, wl.h, wl.o, max_outliers=64)
    assert capped.nbytes * 2 < full.nbytes
    a = binding.llmint8_matmul(Xd, pw, wl.alpha, workspace=full)
    b = binding.llmint8_matmul(Xd, pw, wl.alpha, workspace=capped)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert binding.llmint8_read_device_status(capped) == 0


@pytest.mark.parametrize("path", [1, 2], ids=["prefill", "decode"])
def test_host_status_word_makes_the_next_call_report(path):
    rng = np.random.default_rng(40 + path)
    s = 64 if path == 1 else 8
    X = workloads.random_x(rng, s, 256, outlier_cols=(9,))
    W = workloads.random_w(rng, 256, 256)
    pw = binding.llmint8_prepare_weight(to_dev(W))
    Wq, aw = oracle.prepare_weight(W)
    ref = oracle.matmul(X, Wq, aw, 6.0)
    Xd = to_dev(X)
    ws = binding.Workspace(s, 256, 256)
    word = binding.HostStatusWord()
    # a clean call leaves the word clear
    out = binding.llmint8_matmul(Xd, pw, 6.0, workspace=ws, path=path, status_host=word)
    torch.cuda.synchronize()
    assert word.value == 0
    assert_close_fp16(out.cpu().numpy(), ref)
    # an anomaly recorded on the workspace (the self-test's waits run out) is
    # copied to the word by the next call's last kernel ...
    binding.llmint8_wait_selftest(ws, limit_ns=2_000_000)
    binding.llmint8_matmul(Xd, pw, 6.0, workspace=ws, path=path, status_host=word)
    torch.cuda.synchronize()
    assert word.value == binding.DEV_TIMEOUT_SELFTEST
    # ... and the call after that reports it without enqueuing anything
    marker = torch.full((s, 256), 3.0, dtype=torch.float16, device="cuda")
    with pytest.raises(binding.Llmint8Error) as e:
        binding.llmint8_matmul(Xd, pw, 6.0, out=marker, workspace=ws, path=path,
                               status_host=word)
    assert e.value.code == -6
    torch.cuda.synchronize()
    assert bool((marker == 3.0).all())
    # recovery: clear the word and the workspace's status, re-initialise
    assert binding.llmint8_read_device_status(ws) == binding.DEV_TIMEOUT_SELFTEST
    word.clear()
    assert binding.load_library().llmint8_workspace_init(
        ctypes.c_void_p(ws.buf.data_ptr()), ws.nbytes,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    out = binding.llmint8_matmul(Xd, pw, 6.0, workspace=ws, path=path, status_host=word)
    torch.cuda.synchronize()
    assert word.value == 0
    assert_close_fp16(out.cpu().numpy(), ref)


def test_host_status_word_must_be_device_addressable():
    rng = np.random.default_rng(50)
    X = workloads.random_x(rng, 32, 256)
    W = workloads.random_w(rng, 256, 256)
    pw = binding.llmint8_prepare_weight(to_dev(W))
    ws = binding.Workspace(32, 256, 256)
    pageable = torch.zeros((1,), dtype=torch.int32)
    opts = binding.llmint8_matmul_opts()
    opts.status_host = pageable.data_ptr()
    out = torch.zeros((32, 256), dtype=torch.float16, device="cuda")
    rc = binding.load_library().llmint8_matmul_ex(
        ctypes.c_void_p(to_dev(X).data_ptr()), 32, ctypes.byref(pw.c), 6.0,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(ws.buf.data_ptr()), ws.nbytes,
        ctypes.byref(opts), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -7
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
