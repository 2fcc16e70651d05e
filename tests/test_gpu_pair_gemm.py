"""The prefill GEMM with CTA pairs (tcgen05 cta_group::2, one 256 x 256 tile
per cluster of two CTAs) against the oracle, and bit for bit against the
one-CTA-per-tile GEMM on the same inputs ("The Full LLM.int8() Algorithm",
Steps 3-5: both compute the same int32 accumulators and the same fp32
epilogue, so every output bit agrees)."""
import numpy as np
import pytest
import torch

import oracle
from mixed_precision_int8_b200 import binding, build, workloads
from tests.parity_utils import (assert_close_fp16, gpu_matmul, gpu_prepare,
                                oracle_prepared, sample_cols, sample_rows, to_dev)

pytestmark = pytest.mark.gpu

PAIR, SINGLE = binding.PATH_PREFILL_PAIR, binding.PATH_PREFILL_SINGLE


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    binding.load_library()
    yield


def _inputs(case, seed):
    s, h, o, cols, alpha = case
    rng = np.random.default_rng(3000 + seed + s + h + o)
    X = workloads.random_x(rng, s, h, outlier_cols=cols, lo=6.0, hi=60.0)
    W = workloads.random_w(rng, h, o, sigma=0.02)
    return X, W, alpha


# (s, h, o, outlier columns, alpha): odd and even numbers of 128-row blocks
# (an odd one leaves the last pair's second CTA wholly past s), ragged
# columns, one and several tiles per pair, narrow and wide outlier sets
CASES = [
    (17, 256, 272, (100,), 6.0),
    (128, 512, 256, (5, 6, 7), 6.0),
    (300, 1024, 528, tuple(range(0, 1024, 64)), 6.0),       # |O| = 16
    (256, 1040, 784, tuple(range(3, 1040, 13)), 6.0),       # |O| = 80, wide
    (384, 512, 2048, (), 0.0),                              # every column out
    (300, 1040, 15376, tuple(range(3, 1040, 61)), 6.0),     # more tiles than pairs
    (1000, 2048, 4096, (11, 2000), 6.0),
]


@pytest.mark.parametrize("wo_build", [binding.WO_SHARED, binding.WO_EACH_CTA],
                         ids=["wo_shared", "wo_each_cta"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}a{c[4]}")
def test_pair_gemm_matches_the_oracle_and_the_single_cta_gemm(case, wo_build):
    X, W, alpha = _inputs(case, seed=1)
    pw, _ = gpu_prepare(W)
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    ref, ci_ref = oracle.matmul(X, Wq_ref, aw_ref, alpha, want_ci=True)
    out_p, ci_p, ws = gpu_matmul(X, pw, alpha, path=PAIR, want_ci=True, wo_build=wo_build)
    assert np.array_equal(ci_p, ci_ref), "int32 accumulators"
    assert_close_fp16(out_p, ref, "out")
    out_s, ci_s, _ = gpu_matmul(X, pw, alpha, path=SINGLE, want_ci=True, wo_build=wo_build)
    assert np.array_equal(ci_s, ci_p)
    assert np.array_equal(out_s.view(np.uint16), out_p.view(np.uint16))
    f_ref, idx_ref, n_ref = oracle.detect_outliers(X, alpha)
    n, XO, WO = binding.llmint8_read_outlier_tiles(ws)
    assert n == n_ref
    assert np.array_equal(WO.numpy().view(np.uint16),
                          oracle.outlier_weights(Wq_ref, aw_ref, idx_ref).view(np.uint16))


def test_pair_gemm_fp16_outlier_rows():
    X, W, alpha = _inputs((256, 1040, 784, tuple(range(3, 1040, 13)), 6.0), seed=2)
    pw, _ = gpu_prepare(W, keep_fp16=True)
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    ref, ci_ref = oracle.matmul(X, Wq_ref, aw_ref, alpha, want_ci=True, W16=W)
    out, ci, _ = gpu_matmul(X, pw, alpha, path=PAIR, want_ci=True)
    assert np.array_equal(ci, ci_ref)
    assert_close_fp16(out, ref, "out")


@pytest.mark.parametrize("name", ["opt6.7b_attn_prefill", "opt13b_ffn_up_prefill"])
def test_pair_gemm_on_the_workloads(name):
    """Full-size OPT shapes through the pair kernel: bit for bit against the
    one-CTA kernel everywhere, and against the oracle on sampled outputs."""
    wl, X, cols, W = workloads.make_inputs(name)
    Wd = torch.from_numpy(W).cuda()
    pw = binding.llmint8_prepare_weight(Wd)
    Xd = to_dev(X)
    ws = binding.Workspace(wl.s, wl.h, wl.o)
    outs = []
    for path in (PAIR, SINGLE):
        out = binding.llmint8_matmul(Xd, pw, wl.alpha, workspace=ws, path=path)
        torch.cuda.synchronize()
        assert binding.llmint8_read_device_status(ws) == 0
        outs.append(out.cpu().numpy())
    assert np.array_equal(outs[0].view(np.uint16), outs[1].view(np.uint16))
    rows = sample_rows(wl.s, 48)
    c = sample_cols(wl.o, 512)
    Wq_ref, aw_ref = oracle_prepared(W, c)
    ref = oracle.matmul(X, Wq_ref, aw_ref, wl.alpha, rows=rows)
    assert_close_fp16(outs[0][np.ix_(rows, c)], ref)
    del pw, ws, Xd
    torch.cuda.empty_cache()


def test_automatic_kernel_choice():
    """The decode kernel for s <= 16, else the one-CTA-per-tile GEMM (the
    pair kernel only when asked for)."""
    assert binding.llmint8_prefill_kernel(8, 12288, 49152) == binding.PATH_DECODE
    assert binding.llmint8_prefill_kernel(2048, 4096, 4096) == binding.PATH_PREFILL_SINGLE
    assert binding.llmint8_prefill_kernel(2048, 12288, 49152) == binding.PATH_PREFILL_SINGLE
    with pytest.raises(binding.Llmint8Error):
        binding.llmint8_prefill_kernel(-1, 16, 16)
