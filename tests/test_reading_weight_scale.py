"""The one reading of the pages whose effect depends on the data: the weight
column scale.

"The Full LLM.int8() Algorithm", Step 4, takes each column's absmax over the
non-outlier rows of W; the same page prepares W once at load time, before any
input (and so any outlier set) exists. This build takes the column absmax
over all h rows, offline. The two agree except in columns whose largest |W|
lies in one of the input's outlier rows; there the offline scale is larger
and the column's codes coarser. With Gaussian W that happens to about
|O| * o / h columns. This test counts them on the seeded workloads, so the
size of the difference is stated, not assumed.
"""
import numpy as np
import pytest

import oracle
from mixed_precision_int8_b200 import workloads


@pytest.mark.parametrize("name,count,ratio", [("opt6.7b_attn_prefill", 3, 1.109),
                                              ("opt13b_ffn_up_prefill", 28, 1.484)])
def test_columns_whose_scale_depends_on_the_reading(name, count, ratio):
    wl, X, cols, W = workloads.make_inputs(name)
    _, idx, n = oracle.detect_outliers(X, wl.alpha)
    A = np.abs(W.astype(np.float32))
    all_rows = A.max(axis=0)
    regular = np.ones(wl.h, dtype=bool)
    regular[idx] = False
    regular_rows = A[regular].max(axis=0)
    differ = regular_rows < all_rows
    assert int(differ.sum()) == count
    # expected count for Gaussian W: the argmax row is uniform over h rows
    assert abs(count - wl.o * n / wl.h) <= 3 * np.sqrt(wl.o * n / wl.h)
    assert abs(float((all_rows / regular_rows).max()) - ratio) < 1e-3
    # the oracle's (and the GPU's) scale is the all-rows one
    _, aw = oracle.prepare_weight(np.ascontiguousarray(W[:, :256]))
    assert np.array_equal(aw, all_rows[:256])
