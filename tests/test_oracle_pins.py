"""Pins for the CPU oracle: checks against what the pages and the mathematics
fix, never against the oracle itself or the CUDA path.

Each test names the fact it pins. Together they are chosen so that a plausible
slip anywhere in the oracle (dropped term, wrong sign or index, transposed
operand, wrong scale, wrong tie rule, wrong threshold comparison) fails one.
"""
import math

import numpy as np
import pytest

import oracle
from mixed_precision_int8_b200 import workloads
from tests.conftest import load_golden

RNG = np.random.default_rng(12345)


# ----------------------------------------------------------------- binary16

def test_half_decode_every_bit_pattern_matches_numpy():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_half_encode_matches_numpy_rne_including_ties():
    # random magnitudes over the whole binary16 range, subnormals included
    mags = np.exp2(RNG.uniform(-27, 17, size=20000))
    vals = mags * RNG.choice([-1.0, 1.0], size=mags.size)
    # exact midpoints between neighbouring binary16 values (ties to even)
    fin = np.arange(0, 0x7bff, dtype=np.uint16).view(np.float16)
    lo = fin[:-1].astype(np.float64)
    hi = fin[1:].astype(np.float64)
    mids = (lo + hi) / 2.0
    pick = RNG.choice(mids.size, size=5000, replace=False)
    vals = np.concatenate([vals, mids[pick], -mids[pick],
                           [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9,
                            2.0 ** -25, 2.0 ** -24, 3 * 2.0 ** -26]])
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.double_to_half(float(v)) for v in vals],
                   dtype=np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------- pages' worked examples

def _row(key):
    g = load_golden(key)
    x = np.array([[float(v) for v in g["x"]]], dtype=np.float16)
    alpha = float(g["alpha"][0])
    return g, x, alpha


@pytest.mark.parametrize("fixture", ["absmax_worked_example.txt",
                                     "absmax_outlier_example.txt"])
def test_pages_worked_quantisation_examples(fixture):
    g, x, alpha = _row(fixture)
    flags, idx, n = oracle.detect_outliers(x, alpha)
    assert n == 0
    Xq, ax = oracle.quantize_rows(x, flags)
    assert ax[0] == float(g["absmax"][0])
    assert Xq[0].tolist() == [int(v) for v in g["codes"]]
    deq = Xq[0].astype(np.float64) * ax[0] / 127.0
    ref = np.array([float(v) for v in g["dequant_approx"]])
    assert np.max(np.abs(deq - ref)) <= float(g["dequant_abs_tol"][0])


def test_pages_outlier_row_with_decomposition():
    g, x, alpha = _row("absmax_outlier_decomposed.txt")
    flags, idx, n = oracle.detect_outliers(x, alpha)
    assert idx.tolist() == [int(v) for v in g["outliers"]]
    Xq, ax = oracle.quantize_rows(x, flags)
    assert ax[0] == float(g["absmax"][0])
    assert Xq[0].tolist() == [int(v) for v in g["codes"]]


def test_pages_range_arithmetic():
    g = load_golden("range_arithmetic.txt")
    amax = float(g["max_value"][0])
    r = float(g["small_range"][0])
    assert oracle.quantize_value(amax, amax) == 127
    assert oracle.quantize_value(-amax, amax) == -127
    assert oracle.quantize_value(r, amax) == int(g["small_code_max"][0])
    assert oracle.quantize_value(-r, amax) == -int(g["small_code_max"][0])
    assert abs(100.0 / 127.0 - float(g["step_for_100"][0])) < 1e-3


# ------------------------------------------------ quantiser, exact facts

def test_tie_rule_is_half_away_from_zero():
    # a = 127/16 is a binary16 value; 127*x/a = 16*x is an exact half for
    # x = (2k+1)/32, so the tie rule decides the code.
    a = np.float16(127.0 / 16.0)
    assert float(a) == 127.0 / 16.0
    for k in range(0, 40):
        x = np.float16((2 * k + 1) / 32.0)
        assert float(x) * 16.0 == k + 0.5
        assert oracle.quantize_value(float(x), float(a)) == k + 1
        assert oracle.quantize_value(-float(x), float(a)) == -(k + 1)


def _exact_codes(x16, a16):
    """round-half-away-from-zero of the exact rational 127*x/a, integers only.

    Every binary16 value is an integer multiple of 2^-24, so with X = x*2^24
    and A = a*2^24 (integers) the code is sign(X)*floor((254|X| + A)/(2A)).
    """
    X = (x16.astype(np.float64) * 2.0 ** 24).astype(np.int64)
    A = (a16.astype(np.float64) * 2.0 ** 24).astype(np.int64)
    q = (254 * np.abs(X) + A) // (2 * A)
    return np.sign(X) * q


def test_fp32_quantiser_equals_exact_rational_rounding():
    n = 200000
    a = np.exp2(RNG.uniform(-22, 15.9, size=n)).astype(np.float16)
    a = a[(a > 0) & np.isfinite(a)]
    u = RNG.uniform(-1.0, 1.0, size=a.size)
    x = (u * a.astype(np.float64)).astype(np.float16)
    keep = np.abs(x.astype(np.float64)) <= a.astype(np.float64)
    x, a = x[keep], a[keep]
    got = np.array([oracle.quantize_value(float(xi), float(ai))
                    for xi, ai in zip(x[:40000], a[:40000])])
    assert np.array_equal(got, _exact_codes(x[:40000], a[:40000]))
    # the same through the row quantiser (vectorised), one row per pair
    X = np.stack([x[40000:], a[40000:]], axis=1)
    flags = np.zeros(2, dtype=np.uint8)
    Xq, ax = oracle.quantize_rows(X, flags)
    assert np.array_equal(ax, np.maximum(np.abs(x[40000:]),
                                         a[40000:]).astype(np.float32))
    assert np.array_equal(Xq[:, 0], _exact_codes(x[40000:], a[40000:]))


def test_roundtrip_error_bound_absmax_over_254():
    # "tm_llm_int8", section "Absmax INT8 quantization from first
    # principles": per-element error at most absmax/254.
    X = workloads.random_x(RNG, 64, 512, outlier_cols=(3, 100), lo=6, hi=90)
    flags, idx, n = oracle.detect_outliers(X, 6.0)
    Xq, ax = oracle.quantize_rows(X, flags)
    keep = flags == 0
    x = X[:, keep].astype(np.float64)
    deq = Xq[:, keep].astype(np.float64) * ax[:, None].astype(np.float64) / 127
    bound = ax[:, None].astype(np.float64) / 254.0
    assert np.all(np.abs(x - deq) <= bound * (1 + 1e-12))
    assert np.all(Xq[:, ~keep] == 0)


def test_symmetric_range_and_absmax_maps_to_127():
    X = workloads.random_x(RNG, 128, 256, outlier_cols=(5,), scale=1.7)
    flags, idx, n = oracle.detect_outliers(X, 6.0)
    Xq, ax = oracle.quantize_rows(X, flags)
    assert Xq.min() >= -127 and Xq.max() <= 127
    assert np.all(np.abs(Xq).max(axis=1) == 127)
    W = workloads.random_w(RNG, 300, 48)
    Wq, aw = oracle.prepare_weight(W)
    assert Wq.min() >= -127
    assert np.all(np.abs(Wq).max(axis=1) == 127)


# ------------------------------------------------------ weight preparation

def test_prepare_weight_layout_scale_and_codes():
    W = workloads.random_w(RNG, 200, 72)
    W[:, 5] = 0  # a zero column: scale 0, codes 0
    Wq, aw = oracle.prepare_weight(W)
    assert Wq.shape == (72, 200)
    assert np.array_equal(aw, np.abs(W.astype(np.float32)).max(axis=0))
    assert aw[5] == 0 and np.all(Wq[5] == 0)
    j = np.arange(72) != 5
    exact = _exact_codes(W.T[j].ravel(),
                         np.repeat(aw[j].astype(np.float16), 200))
    assert np.array_equal(Wq[j].ravel().astype(np.int64), exact)


def test_tensor_wise_and_row_wise_codes_of_the_golden_rows():
    g = load_golden("tensorwise_example.txt")
    X = np.array([[float(v) for v in g["row1"]], [float(v) for v in g["row2"]]],
                 dtype=np.float16)
    flags = np.zeros(4, dtype=np.uint8)
    Xq, ax = oracle.quantize_rows(X, flags, tensor=True)
    assert ax.tolist() == [float(g["tensor_scale"][0])] * 2
    assert Xq[0].tolist() == [int(v) for v in g["tensor_codes1"]]
    assert Xq[1].tolist() == [int(v) for v in g["tensor_codes2"]]
    Xq, ax = oracle.quantize_rows(X, flags)
    assert ax.tolist() == [float(v) for v in g["row_scales"]]
    assert Xq[0].tolist() == [int(v) for v in g["tensor_codes1"]]
    assert Xq[1].tolist() == [int(v) for v in g["row_codes2"]]
    # one scale for all rows: any row subset sees the whole tensor's constant
    Xq, ax = oracle.quantize_rows(X, flags, rows=[1], tensor=True)
    assert ax.tolist() == [3.0] and Xq[0].tolist() == [int(v) for v in g["tensor_codes2"]]


def test_tensor_wise_equals_row_wise_when_every_row_shares_its_absmax():
    X = workloads.random_x(RNG, 12, 96, outlier_cols=(7,), row_frac=1.0)
    X[:, 3] = 4.5  # below alpha, above every N(0,1) draw here: every row's max
    flags, _, _ = oracle.detect_outliers(X, 6.0)
    a = oracle.quantize_rows(X, flags)
    b = oracle.quantize_rows(X, flags, tensor=True)
    assert np.all(a[1] == 4.5)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_tensor_wise_weight_uses_the_global_absmax():
    W = workloads.random_w(RNG, 150, 40)
    Wq, aw = oracle.prepare_weight(W, tensor=True)
    m = np.abs(W.astype(np.float32)).max()
    assert np.all(aw == m)
    exact = _exact_codes(W.T.ravel(), np.full(W.size, m, dtype=np.float16))
    assert np.array_equal(Wq.ravel().astype(np.int64), exact)


# ----------------------------------------------------------- detection

def test_detection_threshold_is_inclusive():
    x = np.zeros((3, 6), dtype=np.float16)
    x[0, 1] = 6.0                       # exactly alpha: outlier
    x[1, 2] = np.float16(5.9960938)     # largest binary16 below 6: not
    x[2, 4] = -6.0                      # magnitude counts, not sign
    x[1, 5] = np.inf
    flags, idx, n = oracle.detect_outliers(x, 6.0)
    assert idx.tolist() == [1, 4, 5]
    assert flags.tolist() == [0, 1, 0, 0, 1, 1]


def test_detection_finds_planted_columns_of_tiny_workload():
    wl = workloads.get_workload("tiny")
    x, cols = workloads.make_x(wl)
    flags, idx, n = oracle.detect_outliers(x, wl.alpha)
    assert idx.tolist() == [7, 200]
    # planted: exactly round(0.8*16) = 13 rows of each column are >= 8
    for c in (7, 200):
        assert int(np.sum(np.abs(x[:, c].astype(np.float32)) >= 8)) == 13


def test_detection_ignores_alpha_infinity_and_alpha_zero_flags_nonzero():
    x = workloads.random_x(RNG, 8, 32, outlier_cols=(2,))
    x[:, 9] = 0
    _, _, n = oracle.detect_outliers(x, math.inf)
    assert n == 0
    flags, idx, n = oracle.detect_outliers(x, 0.0)
    assert n == 32  # |x| >= 0 holds everywhere, zero columns included


# ------------------------------------------------------------ int8 product

def test_int8_product_matches_numpy_int64():
    Xq = RNG.integers(-127, 128, size=(33, 300), dtype=np.int8)
    Wq = RNG.integers(-127, 128, size=(45, 300), dtype=np.int8)
    got = oracle.int8_gemm(Xq, Wq)
    ref = Xq.astype(np.int64) @ Wq.astype(np.int64).T
    assert np.array_equal(got.astype(np.int64), ref)
    cols = [44, 0, 7]
    assert np.array_equal(oracle.int8_gemm(Xq, Wq, cols), ref[:, cols])


def test_int32_overflow_is_reported_one_past_the_limit():
    # 127*127*h fits int32 up to h = 133144 and not beyond.
    assert 127 * 127 * 133144 < 2 ** 31 <= 127 * 127 * 133145
    for h, ok in ((133144, True), (133145, False)):
        Xq = np.full((1, h), 127, dtype=np.int8)
        Wq = np.full((1, h), 127, dtype=np.int8)
        if ok:
            assert oracle.int8_gemm(Xq, Wq)[0, 0] == 127 * 127 * h
        else:
            with pytest.raises(OverflowError):
                oracle.int8_gemm(Xq, Wq)


# ------------------------------------------------- the whole decomposition

def _dyadic_case(rng, s, h, o, outlier_cols):
    """Inputs on which both quantisations are lossless, so the method's
    output must equal the exact product X.W rounded once to binary16."""
    n = rng.integers(-127, 128, size=(s, h))
    regular = np.setdiff1d(np.arange(h), outlier_cols)
    n[np.arange(s), rng.choice(regular, size=s)] = 127  # row absmax 127*2^-5
    X = (n * 2.0 ** -5)
    for c in outlier_cols:
        X[:, c] = rng.choice([6.0, -7.5, 10.25, 31.0, 0.5, 0.0], size=s)
        X[0, c] = 6.0  # guarantee the column is flagged
    m = rng.integers(-127, 128, size=(h, o))
    m[rng.integers(0, h, size=o), np.arange(o)] = -127  # col absmax
    W = m * 2.0 ** -10
    return X.astype(np.float16), W.astype(np.float16)


def test_lossless_case_equals_rounded_exact_product():
    rng = np.random.default_rng(7)
    s, h, o = 24, 96, 40
    X, W = _dyadic_case(rng, s, h, o, outlier_cols=(3, 50, 51))
    Wq, aw = oracle.prepare_weight(W)
    assert np.all(aw == np.float32(127 * 2.0 ** -10))
    out = oracle.matmul(X, Wq, aw, 6.0)
    exact = X.astype(np.float64) @ W.astype(np.float64)
    assert np.array_equal(out.view(np.uint16),
                          exact.astype(np.float16).view(np.uint16))


def test_alpha_zero_is_a_plain_fp16_product_of_the_outlier_rows():
    # alpha = 0 flags every column; the int8 part vanishes and the output is
    # X . WO rounded once, WO being the weight recovered from its int8 code.
    X = workloads.random_x(RNG, 10, 64, outlier_cols=(1,))
    W = workloads.random_w(RNG, 64, 24)
    Wq, aw = oracle.prepare_weight(W)
    flags, idx, n = oracle.detect_outliers(X, 0.0)
    assert n == 64
    WO = oracle.outlier_weights(Wq, aw, idx)
    # WO against an independent exact recomputation of the dequantised weight
    ref_wo = (Wq.T.astype(np.float64) * aw[None, :].astype(np.float64)
              / 127.0)
    assert np.all(np.abs(WO.astype(np.float64) - ref_wo)
                  <= np.abs(ref_wo) * 2.0 ** -11 * 1.0001 + 2.0 ** -25)
    out, Ci = oracle.matmul(X, Wq, aw, 0.0, want_ci=True)
    assert np.all(Ci == 0)
    ref = X.astype(np.float64) @ WO.astype(np.float64)
    assert np.array_equal(out.view(np.uint16),
                          ref.astype(np.float16).view(np.uint16))


def test_exact_fp16_outlier_rows_with_alpha_zero_give_the_fp16_product():
    # [P4] "Mixed-Precision Decomposition": the outlier part of W stays in
    # fp16. Given the caller's fp16 W and alpha = 0, every column is an
    # outlier column, the int8 part vanishes and the output is X . W itself
    # (a textbook product, rounded once). h != o catches a transposed read.
    X = workloads.random_x(RNG, 10, 64, outlier_cols=(1,))
    W = workloads.random_w(RNG, 64, 24)
    Wq, aw = oracle.prepare_weight(W)
    out, Ci = oracle.matmul(X, Wq, aw, 0.0, want_ci=True, W16=W)
    assert np.all(Ci == 0)
    ref = X.astype(np.float64) @ W.astype(np.float64)
    assert np.array_equal(out.view(np.uint16),
                          ref.astype(np.float16).view(np.uint16))


def test_exact_fp16_outlier_rows_change_nothing_without_outliers():
    # With no outlier column the fp16 weight is never read: the output equals
    # the recovered-rows output bit for bit; with outliers it differs.
    X = workloads.random_x(RNG, 16, 128, scale=1.0)
    W = workloads.random_w(RNG, 128, 40)
    Wq, aw = oracle.prepare_weight(W)
    a = oracle.matmul(X, Wq, aw, 6.0)
    b = oracle.matmul(X, Wq, aw, 6.0, W16=W)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))
    Xo = workloads.random_x(RNG, 16, 128, outlier_cols=(3, 70), lo=20.0, hi=60.0)
    a = oracle.matmul(Xo, Wq, aw, 6.0)
    b = oracle.matmul(Xo, Wq, aw, 6.0, W16=W)
    assert not np.array_equal(a.view(np.uint16), b.view(np.uint16))


def test_no_outlier_input_is_pure_vector_wise_int8():
    # With max |X| < alpha the outlier set is empty, so alpha has no further
    # effect: any alpha above max |X| gives the same output as alpha = +inf.
    X = workloads.random_x(RNG, 16, 128, scale=1.0)
    W = workloads.random_w(RNG, 128, 32)
    Wq, aw = oracle.prepare_weight(W)
    amax = float(np.abs(X.astype(np.float32)).max())
    a = oracle.matmul(X, Wq, aw, math.inf)
    b = oracle.matmul(X, Wq, aw, amax + 0.01)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))
    # and the int32 part equals the row-code x column-code product
    flags = np.zeros(128, dtype=np.uint8)
    Xq, ax = oracle.quantize_rows(X, flags)
    assert np.array_equal(
        oracle.matmul(X, Wq, aw, math.inf, want_ci=True)[1].astype(np.int64),
        Xq.astype(np.int64) @ Wq.astype(np.int64).T)


def test_error_against_fp64_product_within_closed_form_bound():
    for seed in range(4):
        rng = np.random.default_rng(100 + seed)
        s, h, o = 12, 64, 20
        X = workloads.random_x(rng, s, h, outlier_cols=(4, 33), lo=6, hi=50)
        W = workloads.random_w(rng, h, o, sigma=0.05)
        Wq, aw = oracle.prepare_weight(W)
        flags, idx, n = oracle.detect_outliers(X, 6.0)
        Xq, ax = oracle.quantize_rows(X, flags)
        out = oracle.matmul(X, Wq, aw, 6.0).astype(np.float64)
        x = X.astype(np.float64)
        w = W.astype(np.float64)
        exact = x @ w
        reg = flags == 0
        axd = ax.astype(np.float64)[:, None]
        awd = aw.astype(np.float64)[None, :]
        bound = (np.abs(x[:, reg]) @ np.ones((reg.sum(), o)) * awd / 254
                 + axd * (np.ones((s, reg.sum())) @ np.abs(w[reg])) / 254
                 + reg.sum() * 3 * axd * awd / 254 ** 2)
        bound += np.abs(x[:, ~reg]) @ (awd / 254
                                       + np.abs(w[~reg]) * 2.0 ** -10)
        bound += np.abs(exact) * 2.0 ** -10 + 2.0 ** -24
        assert np.all(np.abs(out - exact) <= bound)


def test_zero_row_and_zero_weight_column():
    X = workloads.random_x(RNG, 6, 48, outlier_cols=(10,), row_frac=1.0)
    X[2, :] = 0
    X[4, :] = 0
    X[4, 10] = 9.0  # row 4: only its outlier entry is nonzero -> ax = 0
    W = workloads.random_w(RNG, 48, 16)
    W[:, 3] = 0
    Wq, aw = oracle.prepare_weight(W)
    flags, idx, n = oracle.detect_outliers(X, 6.0)
    Xq, ax = oracle.quantize_rows(X, flags)
    assert ax[2] == 0 and ax[4] == 0 and np.all(Xq[[2, 4]] == 0)
    out = oracle.matmul(X, Wq, aw, 6.0).astype(np.float64)
    assert np.all(out[2] == 0)
    assert np.all(out[:, 3] == 0)
    WO = oracle.outlier_weights(Wq, aw, idx).astype(np.float64)
    ref = (9.0 * WO[0]).astype(np.float16).astype(np.float64)
    assert np.array_equal(out[4], ref)


def test_row_and_column_subsets_equal_slices_of_full_output():
    wl = workloads.get_workload("tiny")
    X, _ = workloads.make_x(wl)
    W = workloads.make_w(wl)
    Wq, aw = oracle.prepare_weight(W)
    full, ci = oracle.matmul(X, Wq, aw, 6.0, want_ci=True)
    rows = [15, 0, 7]
    cols = [255, 1, 128, 7]
    part, cp = oracle.matmul(X, Wq, aw, 6.0, rows=rows, cols=cols,
                             want_ci=True)
    assert np.array_equal(part.view(np.uint16),
                          full[np.ix_(rows, cols)].view(np.uint16))
    assert np.array_equal(cp, ci[np.ix_(rows, cols)])
