"""The division-free rule the CUDA kernels use for the int8 row codes, checked
on the CPU in exact integer arithmetic (no GPU, no oracle).

The method's code is q = round_half_away_from_zero(127 x / a) for |x| <= a
("tm_llm_int8", "Absmax INT8 quantization from first principles";
"LLM.int8(): 8-bit Matrix Multiplication for Transformers at Scale",
"Quantization Primitives"). The kernels compute one fp32 reciprocal per row,
rounded up, R = RU(127 / a), and per element one fused multiply-add rounded
toward minus infinity,

    k = floor(2 |x| R + 1),   q = floor(k / 2),

which equals floor(|x| R + 1/2). Because R >= 127/a, the computed value is
never below the exact one, and it exceeds it by less than q 2^-23, less than
the distance from 127|x|/a + 1/2 to the next integer whenever that quantity
is not itself an integer (binary16 mantissas have 11 bits). So the result is
exactly the rounded quotient, ties included. This file checks that claim on
about two million (x, a) pairs, including every exact tie 127x/a = n + 1/2
that binary16 allows, against floor((254 |x| + a) / (2 a)).
"""
import numpy as np


def _all_magnitudes():
    """Every finite non-negative binary16 value as (bits, mantissa, shift):
    value = mantissa * 2^(shift - 24), mantissa < 2^11."""
    bits = np.arange(0, 0x7C00, dtype=np.int64)
    e = bits >> 10
    m = bits & 0x3FF
    mant = np.where(e == 0, m, m + 1024)
    shift = np.where(e == 0, 0, e - 1)
    return bits, mant, shift


def _ru_reciprocal(A: int):
    """R * 2^er = 127 / a rounded up to fp32 (a = A 2^-24, A > 0): R has 24
    bits, found with Python integers."""
    num = 127 << 24  # 127 / a = num / A
    # choose er so that 2^23 <= num / (A 2^er) < 2^24
    er = (num.bit_length() - A.bit_length()) - 24
    while True:
        if er >= 0:
            R = -(-num // (A << er))
        else:
            R = -(-(num << -er) // A)
        if R >= 1 << 24:
            er += 1
            continue
        if R < 1 << 23:
            er -= 1
            continue
        return R, er


def _gpu_rule(mx, px, R, er):
    """floor(floor(2 x R 2^er + 1) / 2) for x = mx 2^(px - 24), in int64:
    2 x R 2^er = mx R 2^(px + er - 23)."""
    prod = mx * R  # < 2^35
    sh = px + er - 23
    k = np.where(sh >= 0, prod << np.maximum(sh, 0), prod >> np.maximum(-sh, 0)) + 1
    return k >> 1


def _exact(X, A):
    return (254 * X + A) // (2 * A)


def test_division_free_row_code_equals_exact_rounding():
    bits, mant, shift = _all_magnitudes()
    X_all = mant << shift
    a_bits = [(e << 10) | m for e in range(31) for m in (0, 1, 0x0AB, 0x155, 0x2C1, 0x3FF)]
    checked = 0
    for ab in a_bits:
        A = int(X_all[ab])
        if A == 0:
            continue
        R, er = _ru_reciprocal(A)
        sel = X_all <= A
        mx, px, X = mant[sel], shift[sel], X_all[sel]
        got = _gpu_rule(mx, px, R, er)
        want = _exact(X, A)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, (f"a bits {ab:#06x}: {bad.size} codes differ, first x bits "
                               f"{int(bits[sel][bad[0]]):#06x}: {int(got[bad[0]])} != "
                               f"{int(want[bad[0]])}")
        assert want.max() == 127 and want.min() == 0
        checked += X.size
    assert checked > 1_500_000


def test_division_free_row_code_on_every_exact_tie():
    """a = 127 d and x = (2n + 1) d / 2 (d = m 2^k, m odd) make 127 x / a = n +
    1/2 exactly; each such binary16 pair rounds away from zero, to n + 1."""
    bits, mant, shift = _all_magnitudes()
    X_all = mant << shift
    value_of = {int(X): i for i, X in enumerate(X_all)}
    ties = 0
    for m in range(1, 16, 2):
        for k in range(-24, 16):
            # d = m 2^k; in units of 2^-24: D = m 2^(k + 24) (needs k + 24 >= 1
            # so that x = (2n+1) D / 2 is a multiple of 2^-24)
            if k + 24 < 1:
                continue
            D = m << (k + 24)
            A = 127 * D
            if A not in value_of:
                continue
            R, er = _ru_reciprocal(A)
            for n in range(127):
                X = (2 * n + 1) * D // 2
                if X not in value_of:
                    continue
                i = value_of[X]
                got = int(_gpu_rule(mant[i:i + 1], shift[i:i + 1], R, er)[0])
                assert got == n + 1 == int(_exact(np.int64(X), np.int64(A))), (m, k, n)
                ties += 1
    assert ties > 10_000


def test_division_free_row_code_on_the_half_of_every_scale():
    """x = a / 2 gives 127 x / a = 63.5 for every a: code 64, for each of the
    ~30k binary16 a whose half is representable (every mantissa pattern)."""
    bits, mant, shift = _all_magnitudes()
    X_all = mant << shift
    value_of = {int(X): i for i, X in enumerate(X_all)}
    n = 0
    for A in X_all[1:].tolist():
        if A % 2 or (A // 2) not in value_of:
            continue
        i = value_of[A // 2]
        R, er = _ru_reciprocal(A)
        assert int(_gpu_rule(mant[i:i + 1], shift[i:i + 1], R, er)[0]) == 64, A
        n += 1
    assert n > 29_000


def test_zero_scale_and_zero_value():
    # a == 0 is given the reciprocal 0: k = floor(0 + 1) = 1, q = 0
    assert int(_gpu_rule(np.int64(5), np.int64(3), 0, 0)) == 0
    R, er = _ru_reciprocal(1)  # a = 2^-24, the smallest binary16
    assert int(_gpu_rule(np.int64(0), np.int64(0), R, er)) == 0
    assert int(_gpu_rule(np.int64(1), np.int64(0), R, er)) == 127
