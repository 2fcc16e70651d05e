"""GPU test of llmint8_matmul_noalloc, the entry point for callers that cannot
give the library a device workspace (for instance an operator called from
inside another runtime's execution callback, where the memory plan is fixed
and allocating at call time is not allowed, or a host program with no
scratch allocator of its own). It runs the same kernels on a static scratch
array kept inside the library.

Each call is checked against llmint8_matmul with a caller workspace, within
the fp16 tolerance the parity tests use, over consecutive calls that share
the library's scratch (decode-sized, prefill-sized, then decode-sized again,
so a call always starts from what the previous one left behind). This file
is collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test.
"""
import numpy as np
import pytest
import torch

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
    return to_dev(X), binding.llmint8_prepare_weight(to_dev(W))


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    wl = workloads.get_workload("tiny")
    Xt, Wt = workloads.make_x(wl)[0], workloads.make_w(wl)
    problems = [
        (to_dev(Xt), binding.llmint8_prepare_weight(to_dev(Wt))),  # s = 16
        _problem(300, 1024, 784, (3, 500, 1000), seed=11),          # prefill
        _problem(5, 512, 272, (0, 17), seed=12),                    # decode
    ]
    for X, pw in problems:
        s, h = X.shape
        ws = binding.Workspace(s, h, pw.o)
        ref = binding.llmint8_matmul(X, pw, 6.0, workspace=ws)
        got = binding.llmint8_matmul_noalloc(X, pw, 6.0)
        torch.cuda.synchronize()
        assert_close_fp16(got.cpu().numpy(), ref.cpu().numpy(), "noalloc out")
    # and once more on the first problem, after the others used the scratch
    X, pw = problems[0]
    again = binding.llmint8_matmul_noalloc(X, pw, 6.0).cpu().numpy()
    first = binding.llmint8_matmul(X, pw, 6.0).cpu().numpy()
    assert_close_fp16(again, first, "noalloc out, repeated")


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
