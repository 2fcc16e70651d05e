"""GPU test of llmint8_matmul_noalloc, the entry point for callers that cannot
give the library a device workspace (for instance an operator called from
inside another runtime's execution callback, where the memory plan is fixed
and allocating at call time is not allowed, or a host program with no
scratch allocator of its own). It runs the same kernels on a static scratch
array kept inside the library.

Each call is compared with llmint8_matmul on a caller workspace bit for bit
(the kernels are deterministic: integer accumulation, fixed fp32 order), and
with the CPU oracle (int32 accumulators exact through the workspace path's
ci output, fp16 output within 2e-3 * (1 + |oracle|)), over consecutive calls
that share the library's scratch (decode-sized, prefill-sized, then
decode-sized again, so a call always starts from what the previous one left
behind). The scratch array's status word, read through
llmint8_noalloc_read_device_status, stays clear. This file is collected last
on purpose: if it fails, a run that stops at the first failure has already
run every other test.
"""
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


def test_noalloc_matches_workspace_entry_point_and_oracle_on_consecutive_calls():
    wl = workloads.get_workload("tiny")
    problems = [
        (workloads.make_x(wl)[0], workloads.make_w(wl)),   # s = 16: decode kernel
        _problem(300, 1024, 784, (3, 500, 1000), seed=11),  # prefill
        _problem(5, 512, 272, (0, 17), seed=12),            # decode
        _problem(200, 1040, 256, tuple(range(3, 1040, 61)), seed=13),  # |O| = 17
    ]
    prepared = []
    for X, W in problems:
        s, h = X.shape
        pw = binding.llmint8_prepare_weight(to_dev(W))
        Xd = to_dev(X)
        ws = binding.Workspace(s, h, pw.o)
        ci = torch.empty((s, pw.o), dtype=torch.int32, device="cuda")
        ref = binding.llmint8_matmul(Xd, pw, 6.0, workspace=ws, ci=ci)
        got = binding.llmint8_matmul_noalloc(Xd, pw, 6.0)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), (s, h, pw.o)
        Wq, aw = oracle.prepare_weight(W)
        orc, ci_orc = oracle.matmul(X, Wq, aw, 6.0, want_ci=True)
        assert np.array_equal(ci.cpu().numpy(), ci_orc)
        assert_close_fp16(got.cpu().numpy(), orc, "noalloc out vs oracle")
        assert binding.llmint8_read_device_status(ws) == 0
        assert binding.llmint8_noalloc_read_device_status() == 0
        prepared.append((Xd, pw, got.clone()))
    # and once more on each problem, after the others used the scratch
    for Xd, pw, first in prepared:
        again = binding.llmint8_matmul_noalloc(Xd, pw, 6.0)
        torch.cuda.synchronize()
        assert torch.equal(again.view(torch.int16), first.view(torch.int16))
    assert binding.llmint8_noalloc_read_device_status() == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    s, h, o = 16, 4096, 8192
    assert binding.llmint8_workspace_size(s, h, o) > binding.NOALLOC_MAX_SCRATCH_BYTES
    X = torch.zeros((s, h), dtype=torch.float16, device="cuda")
    W = torch.zeros((h, o), dtype=torch.float16, device="cuda")
    pw = binding.llmint8_prepare_weight(W)
    out = torch.zeros((s, o), dtype=torch.float16, device="cuda")
    with pytest.raises(binding.Llmint8Error) as e:
        binding.llmint8_matmul_noalloc(X, pw, 6.0, out=out)
    assert e.value.code == -9
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
