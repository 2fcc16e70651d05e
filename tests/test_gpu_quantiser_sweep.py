"""GPU sweep of the int8 quantisers over the whole binary16 range.

The row quantiser of the CUDA path decides each code without a division
(one reciprocal per row, two biased fmas and an exact residual where they
disagree); the weight quantiser divides. Both must equal the rule

    q = round_half_away_from_zero(fp32(127 x) / a)      ("tm_llm_int8",
    "Absmax INT8 quantization from first principles"; "LLM.int8(): 8-bit
    Matrix Multiplication for Transformers at Scale", "Quantization
    Primitives")

for every binary16 x with |x| <= a. Here the codes of a few hundred thousand
(x, a) pairs are compared bit for bit with the oracle and with the exact
rational rounding floor((254 |x| + a) / (2 a)) computed in integers. The
pairs cover:
  - absmax a from the smallest subnormal (2^-24) to 65504, log-uniform;
  - exact ties 127 x / a = n + 1/2 in every binade where they exist
    (a = 127 d, x = (2n + 1) d / 2 for d = m 2^k, m odd), and their
    neighbours one ulp away;
  - every kernel that writes row codes: the one-read activation pass, its
    fix-up (rows whose candidate scale sits in an outlier column are
    requantised), the two-pass kernels for rows longer than a shared-memory
    stage, and the prefill and decode matmul paths (read back through an
    identity weight, whose int32 accumulators are 127 times the codes).
"""
import numpy as np
import pytest
import torch

import oracle
from mixed_precision_int8_b200 import binding, build
from tests.parity_utils import to_dev

pytestmark = pytest.mark.gpu

INF = float("inf")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    binding.load_library()
    yield


def _f16(v):
    return np.asarray(v, dtype=np.float64).astype(np.float16)


def exact_codes(x16: np.ndarray, a16: np.ndarray) -> np.ndarray:
    """round-half-away-from-zero(127 x / a) in exact integer arithmetic
    (binary16 values are integer multiples of 2^-24); 0 where a == 0."""
    xi = np.rint(x16.astype(np.float64) * 2.0 ** 24).astype(np.int64)
    ai = np.rint(a16.astype(np.float64) * 2.0 ** 24).astype(np.int64)
    ai = np.broadcast_to(ai, xi.shape)
    safe = np.where(ai == 0, 1, ai)
    mag = (254 * np.abs(xi) + safe) // (2 * safe)
    q = np.where(xi < 0, -mag, mag)
    return np.where(ai == 0, 0, q).astype(np.int8)


def tie_pairs():
    """(a, x) with 127 x / a exactly n + 1/2, both binary16 values, over
    every binade where they exist, plus the neighbours of each x."""
    out = []
    for m in (1, 3, 5, 7, 9, 11, 13, 15):
        for k in range(-24, 16):
            d = m * 2.0 ** k
            a = 127.0 * d
            if a > 65504.0 or float(_f16(a)) != a:
                continue
            for n in range(127):
                x = (2 * n + 1) * d / 2.0
                if float(_f16(x)) != x:
                    continue
                out.append((a, x))
    pairs = np.array(out, dtype=np.float64)
    a16, x16 = _f16(pairs[:, 0]), _f16(pairs[:, 1])
    up = np.nextafter(x16, np.float16(np.inf))
    dn = np.nextafter(x16, np.float16(0))
    a_all = np.concatenate([a16, a16, a16])
    x_all = np.concatenate([x16, np.minimum(up, a16), dn])
    return a_all, x_all


def random_pairs(rng, n):
    """(a, x): a log-uniform over [2^-24, 65504], x = a u, u ~ U(-1, 1),
    both rounded to binary16 (|x| <= a since rounding is monotone)."""
    a = _f16(np.exp2(rng.uniform(-24.0, np.log2(65504.0), size=n)))
    a = np.where(a == 0, np.float16(2.0 ** -24), a)
    x = _f16(a.astype(np.float64) * rng.uniform(-1.0, 1.0, size=n))
    return a, x


def rows_from_pairs(a, x, h, rng):
    """Rows of width h: column 0 holds the row's absmax a (random sign),
    the other h - 1 columns hold x values quantised against it."""
    per = h - 1
    # every x of a row shares that row's a: group pairs by a, one a per row
    order = np.argsort(a, kind="stable")
    a_s, x_s = a[order], x[order]
    rows = []
    i = 0
    while i < len(a_s):
        j = i
        while j < len(a_s) and j - i < per and a_s[j] == a_s[i]:
            j += 1
        r = np.zeros(h, dtype=np.float16)
        r[0] = a_s[i] if rng.random() < 0.5 else -a_s[i]
        r[1:1 + (j - i)] = x_s[i:j]
        rows.append(r)
        i = j
    return np.stack(rows)


def sweep_rows(h, n_random, seed):
    rng = np.random.default_rng(seed)
    at, xt = tie_pairs()
    ar, xr = random_pairs(rng, n_random)
    # random pairs keep their own a: one row per a value, filled with fresh
    # multiples of it so rows stay full
    per = h - 1
    n_rows = max(1, n_random // per)
    a_rows = ar[:n_rows]
    u = rng.uniform(-1.0, 1.0, size=(n_rows, per))
    Xr = np.empty((n_rows, h), dtype=np.float16)
    Xr[:, 0] = np.where(rng.random(n_rows) < 0.5, a_rows, -a_rows)
    Xr[:, 1:] = _f16(a_rows.astype(np.float64)[:, None] * u)
    Xt = rows_from_pairs(at, xt, h, rng)
    X = np.concatenate([Xr, Xt])
    return X[rng.permutation(X.shape[0])]


def n_pairs(X):
    return X.shape[0] * (X.shape[1] - 1)


def check_rows_against_rules(X, Xq, ax, flags):
    """Codes and scales against the oracle and the exact rational rule."""
    Xq_ref, ax_ref = oracle.quantize_rows(X, flags)
    assert np.array_equal(ax, ax_ref), "row scales"
    bad = np.argwhere(Xq != Xq_ref)
    assert bad.size == 0, (f"{len(bad)} codes differ from the oracle; first "
                           f"row {bad[0][0]} col {bad[0][1]}: x={X[tuple(bad[0])]} "
                           f"a={ax_ref[bad[0][0]]} gpu={Xq[tuple(bad[0])]} "
                           f"oracle={Xq_ref[tuple(bad[0])]}")
    regular = flags == 0
    exact = exact_codes(X[:, regular], ax_ref.astype(np.float16)[:, None])
    assert np.array_equal(Xq[:, regular], exact), "exact rational rounding"


def test_row_quantiser_sweep_one_read_pass():
    X = sweep_rows(16, 200_000, seed=1)
    assert n_pairs(X) >= 200_000
    Xq, ax, flags, idx, n = binding.llmint8_quantize_rows(to_dev(X), INF)
    torch.cuda.synchronize()
    assert int(n.item()) == 0
    f = flags.cpu().numpy()
    assert not f.any()
    check_rows_against_rules(X, Xq.cpu().numpy(), ax.cpu().numpy(), f)
    # the row maxima span the binary16 range, subnormals included
    a = np.abs(X[:, 0].astype(np.float32))
    assert a.min() < 2.0 ** -14 and a.max() > 32768


def test_row_quantiser_sweep_wide_rows_and_ties():
    X = sweep_rows(1040, 60_000, seed=2)
    Xq, ax, flags, idx, n = binding.llmint8_quantize_rows(to_dev(X), INF)
    torch.cuda.synchronize()
    check_rows_against_rules(X, Xq.cpu().numpy(), ax.cpu().numpy(),
                             flags.cpu().numpy())


def test_row_quantiser_sweep_fixup_recomputes_rows():
    """alpha = 6: column 0 is an outlier column (one row holds 50 there); in
    every other row column 0 holds that row's largest |x| below 6, so the
    candidate scale sits in an outlier column and the fix-up requantises the
    row against the largest regular |x| instead."""
    rng = np.random.default_rng(3)
    h = 272
    X = sweep_rows(h, 40_000, seed=4)
    # keep every magnitude below alpha, spread over the subnormal..6 range
    scale = np.abs(X.astype(np.float64)).max(axis=1, keepdims=True)
    scale[scale == 0] = 1.0
    target = np.exp2(rng.uniform(-24.0, np.log2(5.99), size=(X.shape[0], 1)))
    X = _f16(X.astype(np.float64) / scale * target)
    X[:, 0] = _f16(np.abs(X.astype(np.float64)).max(axis=1) * 1.0)
    X[0, 0] = 50.0
    Xq, ax, flags, idx, n = binding.llmint8_quantize_rows(to_dev(X), 6.0)
    torch.cuda.synchronize()
    f = flags.cpu().numpy()
    f_ref, idx_ref, n_ref = oracle.detect_outliers(X, 6.0)
    assert np.array_equal(f, f_ref) and f[0] == 1
    check_rows_against_rules(X, Xq.cpu().numpy(), ax.cpu().numpy(), f)
    assert np.all(Xq.cpu().numpy()[:, 0] == 0)


LONG_H = 108544  # rows too long for a shared-memory stage: two-pass kernels


def test_row_quantiser_sweep_long_rows():
    rng = np.random.default_rng(5)
    at, xt = tie_pairs()
    n_rows = 24
    X = np.zeros((n_rows, LONG_H), dtype=np.float16)
    ks = np.linspace(-24, 15.9, n_rows)
    for r in range(n_rows):
        a = _f16(2.0 ** ks[r])
        if r % 3 == 0:
            # a tie family of this row's binade when one exists
            sel = np.nonzero(np.abs(np.log2(at.astype(np.float64)) - ks[r]) < 1.0)[0]
            if sel.size:
                a = at[sel[0]]
                same = sel[at[sel] == a]
                X[r, 1:1 + same.size] = xt[same]
        X[r, 0] = a
        fill = X[r, 1:] == 0
        X[r, 1:][fill] = _f16(float(a) * rng.uniform(-1.0, 1.0, size=int(fill.sum())))
    Xq, ax, flags, idx, n = binding.llmint8_quantize_rows(to_dev(X), INF)
    torch.cuda.synchronize()
    check_rows_against_rules(X, Xq.cpu().numpy(), ax.cpu().numpy(),
                             flags.cpu().numpy())


def _identity_weight(h):
    W = np.zeros((h, h), dtype=np.float16)
    np.fill_diagonal(W, 1.0)
    return binding.llmint8_prepare_weight(to_dev(W))


@pytest.mark.parametrize("path", [1, 2], ids=["prefill", "decode"])
def test_matmul_row_codes_sweep_through_identity_weight(path):
    """Both matmul paths: with W = I the weight codes are 127 I and every
    column scale is 1, so the exact int32 accumulators are 127 Xq."""
    h = 256
    X = sweep_rows(h, 200_000 if path == 1 else 40_000, seed=6 + path)
    pw = _identity_weight(h)
    assert np.array_equal(pw.aw.cpu().numpy(), np.ones(h, np.float32))
    rows_per_call = X.shape[0] if path == 1 else binding.llmint8_decode_max_rows()
    ws = binding.Workspace(rows_per_call, h, h)
    for r0 in range(0, X.shape[0], rows_per_call):
        Xc = np.ascontiguousarray(X[r0:r0 + rows_per_call])
        s = Xc.shape[0]
        ci = torch.full((s, h), 7, dtype=torch.int32, device="cuda")
        binding.llmint8_matmul(to_dev(Xc), pw, INF, workspace=ws, ci=ci, path=path)
        c = ci.cpu().numpy()
        assert np.all(c % 127 == 0)
        Xq_ref, _ = oracle.quantize_rows(Xc, np.zeros(h, np.uint8))
        assert np.array_equal((c // 127).astype(np.int8), Xq_ref), f"rows {r0}.."
    assert binding.llmint8_read_device_status(ws) == 0


def test_weight_quantiser_sweep():
    """Column scales across the binary16 range (each column one binade or a
    tie family), weight codes bit for bit against the oracle and the exact
    rational rule."""
    rng = np.random.default_rng(8)
    at, xt = tie_pairs()
    h, o = 256, 4096
    W = np.zeros((h, o), dtype=np.float16)
    uniq = np.unique(at)
    for j in range(o):
        if j % 2 == 0 and j // 2 < uniq.size:
            a = uniq[j // 2]
            vals = xt[at == a][: h - 1]
        else:
            a = _f16(2.0 ** rng.uniform(-24.0, np.log2(65504.0)))
            if a == 0:
                a = np.float16(2.0 ** -24)
            vals = np.zeros(0, np.float16)
        col = _f16(float(a) * rng.uniform(-1.0, 1.0, size=h))
        col[0] = a if rng.random() < 0.5 else -a
        col[1:1 + vals.size] = vals * np.where(rng.random(vals.size) < 0.5, 1, -1).astype(np.float16)
        W[:, j] = col
    pw = binding.llmint8_prepare_weight(to_dev(W))
    torch.cuda.synchronize()
    Wq_ref, aw_ref = oracle.prepare_weight(W)
    aw = pw.aw.cpu().numpy()
    wq = pw.wq.cpu().numpy()
    assert np.array_equal(aw, aw_ref)
    assert np.array_equal(wq, Wq_ref)
    exact = exact_codes(W.T, aw_ref.astype(np.float16)[:, None])
    assert np.array_equal(wq, exact)
    assert h * o >= 1_000_000
