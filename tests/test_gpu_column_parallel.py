"""Column-parallel shards on one GPU: every rank's block of the layer, built
from llmint8_prepare_weight_cols on the full fp16 weight, equals the matching
columns of the unsharded CUDA output bit for bit (fp16 output, int32
accumulators, prepared codes and scales), for even and uneven splits, on
small shapes and on the OPT-6.7B and OPT-175B FFN shapes. Ranks are run one
after another in one process: the layer has no exchange step, so no rank
waits for another.
"""
import numpy as np
import pytest
import torch

from mixed_precision_int8_b200 import binding, build, workloads
from mixed_precision_int8_b200.column_parallel import ColumnParallelLinear, shard_columns
from tests.parity_utils import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    binding.load_library()
    yield


def _check_shards(X, Wd, alpha, world, ranks=None):
    s = X.shape[0]
    h, o = Wd.shape
    full_pw = binding.llmint8_prepare_weight(Wd)
    ci_full = torch.empty((s, o), dtype=torch.int32, device="cuda")
    full = binding.llmint8_matmul(X, full_pw, alpha, ci=ci_full)
    for r in (range(world) if ranks is None else ranks):
        layer = ColumnParallelLinear(Wd, world=world, rank=r)
        c0, w = shard_columns(o, world, r)
        assert (layer.col0, layer.width) == (c0, w)
        if w == 0:
            assert layer(X, alpha).shape == (s, 0)
            continue
        assert torch.equal(layer.pw.wq, full_pw.wq[c0:c0 + w])
        assert torch.equal(layer.pw.aw, full_pw.aw[c0:c0 + w])
        block = layer(X, alpha)
        ci = torch.empty((s, w), dtype=torch.int32, device="cuda")
        binding.llmint8_matmul(X, layer.pw, alpha, ci=ci)
        torch.cuda.synchronize()
        assert torch.equal(block.view(torch.int16), full[:, c0:c0 + w].view(torch.int16)), r
        assert torch.equal(ci, ci_full[:, c0:c0 + w]), r


@pytest.mark.parametrize("s,h,o,world", [(40, 512, 784, 3), (300, 1040, 4096, 4),
                                          (8, 512, 272, 4), (129, 256, 512, 8)])
def test_column_shards_equal_slices_of_the_full_output(s, h, o, world):
    rng = np.random.default_rng(s + h + o + world)
    X = to_dev(workloads.random_x(rng, s, h, outlier_cols=(1, h // 2, h - 1)))
    Wd = to_dev(workloads.random_w(rng, h, o))
    _check_shards(X, Wd, 6.0, world)


@pytest.mark.parametrize("name,world,ranks", [("opt6.7b_attn_prefill", 8, None),
                                              ("opt175b_ffn_up_prefill", 8, (0, 7))])
def test_column_shards_on_the_opt_shapes(name, world, ranks):
    wl, X, cols, W = workloads.make_inputs(name)
    _check_shards(to_dev(X), to_dev(W), wl.alpha, world, ranks)
    torch.cuda.empty_cache()
