/*
 * CPU oracle for the LLM.int8() linear-layer hot path C = X.W.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call
 * this file: only the test-suite, the smoke check and the benchmark's CPU
 * baseline leg use it. It shares no code, header or table with the CUDA path.
 *
 * Plain, slow, obviously correct: one loop per step of the method, in the
 * order the pages give it. Integer stages use int64; float stages use fp64
 * except where a quantised code is decided, which is done in IEEE fp32 exactly
 * as the pages' formula reads (127*x is exact in fp32, one rounded fp32
 * division), followed by round-half-away-from-zero.
 *
 * Sources (page title, section):
 *   [P1] "LLM.int8() 完全拆解" (pinghaoyang.com.cn), sections on absmax
 *        quantisation, "第一件武器：向量级量化" and "第二件武器：混合精度分解".
 *   [P2] "tm_llm_int8" (aicassindra.com), sections "Absmax INT8 quantization
 *        from first principles", "Vector-wise: a scale per row and per column",
 *        "A worked quantization example", "The mixed-precision decomposition".
 *   [P4] "LLM.int8(): 8-bit Matrix Multiplication for Transformers at Scale"
 *        (paper-graph-ui summary), sections "Quantization Primitives",
 *        "Vector-wise Quantization", "Mixed-Precision Decomposition" and
 *        "The Full LLM.int8() Algorithm", Steps 1-5.
 *
 * Readings where the pages are silent or disagree (each also listed in the
 * design notes of the repository):
 *   - outlier test is |x| >= alpha ([P4] Step 1; [P1] says "greater than");
 *   - column index range is 0 <= j < h ([P1]/[P4] formal definitions print
 *     "0 <= i <= h", an off-by-one);
 *   - rounding is half away from zero (pages only say "nearest integer");
 *   - the weight column absmax runs over all h rows, computed once offline
 *     ([P4] Step 1 "identified once at model-load time" and the remark that
 *     the weight constants are precomputed at load time);
 *   - the fp16 outlier rows of W are dequantised from the int8 weight:
 *     WO[t][j] = fp16( fp32( fp32(Wq[j][O_t]) * aw[j] ) / 127 );
 *   - scales are kept as the absmax itself (an exact fp16 value held in an
 *     fp32), not as its rounded reciprocal 127/absmax;
 *   - a row whose non-outlier part is empty or all zero has ax = 0 and
 *     quantises to zeros; likewise a zero weight column has aw = 0.
 *
 * Half-precision values cross this interface as raw IEEE binary16 bit
 * patterns (uint16_t); the codec below is written from the IEEE 754
 * definition of binary16.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_OVERFLOW (-2)

/* ---------------------------------------------------------------- binary16 */

/* Value of a binary16 bit pattern: sign, 5-bit biased exponent (bias 15),
 * 10-bit fraction; exponent 0 holds subnormals m * 2^-24. */
double oracle_half_to_double(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int e = (bits >> 10) & 0x1f;
    int m = bits & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = (m != 0) ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

/* Round a non-negative double that is an exact multiple of 1/2 or finer to
 * the nearest integer, ties to even. */
static double round_half_even(double q)
{
    double r = floor(q);
    double d = q - r; /* exact: q and r share the binade up to 2^53 */
    if (d > 0.5)
        return r + 1.0;
    if (d < 0.5)
        return r;
    return (fmod(r, 2.0) == 0.0) ? r : r + 1.0;
}

/* binary16 bit pattern nearest to v (round to nearest, ties to even),
 * with overflow to infinity at and above 65520 = 65504 + half an ulp. */
uint16_t oracle_double_to_half(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v))
        return 0x7e00;
    if (a >= 65520.0)
        return sign | 0x7c00;
    if (a < ldexp(1.0, -14)) {
        /* subnormal grid: multiples of 2^-24; 1024 * 2^-24 is the smallest
         * normal and encodes as exponent 1, fraction 0, i.e. bits 0x400 */
        double q = round_half_even(ldexp(a, 24));
        return sign | (uint16_t)q;
    }
    int E;
    frexp(a, &E);                 /* a = f * 2^E, f in [0.5, 1) */
    int ub = E - 1;               /* a in [2^ub, 2^(ub+1)) */
    double q = round_half_even(ldexp(a, 10 - ub)); /* in [1024, 2048] */
    if (q >= 2048.0) {
        q = 1024.0;
        ub += 1;
    }
    if (ub + 15 >= 31)
        return sign | 0x7c00;
    return sign | (uint16_t)(((ub + 15) << 10) | ((int)q - 1024));
}

/* -------------------------------------------------------------- quantiser */

/* Round half away from zero of an fp32 value, evaluated in fp64 where
 * |v| + 0.5 is exact. */
static double round_half_away(float v)
{
    double d = (double)v;
    double r = floor(fabs(d) + 0.5);
    return (d < 0.0) ? -r : r;
}

/* Absmax code of x against scale a ([P2] "Absmax INT8 quantization from first
 * principles": Q(x) = round(127 * x / absmax); [P4] "Quantization
 * Primitives"): fp32 product 127*x (exact for binary16 x), one IEEE fp32
 * division, then round half away from zero. a == 0 gives 0. */
int oracle_quantize_value(float x, float a)
{
    if (a == 0.0f)
        return 0;
    float prod = 127.0f * x;
    float v = prod / a;
    return (int)round_half_away(v);
}

/* ------------------------------------------------------- weight, offline */

/* [P4] Step 1 / Step 4 bullet 2, read as an offline per-column pass over all
 * h rows: aw[j] = max_k |W[k][j]|; Wq[j][k] = Q(W[k][j], aw[j]).
 * W is [h][o] row-major binary16; Wq is stored transposed, [o][h]
 * (the reduction dimension k contiguous); aw is [o] fp32. */
/* With `tensor` set, the baseline of [P4] "Quantization Primitives" (absmax
 * over the whole tensor, the Table 1 "Int8 absmax" / row-wise weight side):
 * one constant, the largest |W| of all, for every column. */
int oracle_prepare_weight_mode(const uint16_t *W, int64_t h, int64_t o,
                               int tensor, int8_t *Wq, float *aw)
{
    if (!W || !Wq || !aw || h < 0 || o < 0)
        return ORACLE_ERR_ARG;
    for (int64_t j = 0; j < o; ++j) {
        double m = 0.0;
        for (int64_t k = 0; k < h; ++k) {
            double w = fabs(oracle_half_to_double(W[k * o + j]));
            if (w > m)
                m = w;
        }
        aw[j] = (float)m; /* a binary16 value: exact in fp32 */
    }
    if (tensor) {
        float m = 0.0f;
        for (int64_t j = 0; j < o; ++j)
            if (aw[j] > m)
                m = aw[j];
        for (int64_t j = 0; j < o; ++j)
            aw[j] = m;
    }
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < o; ++j) {
        for (int64_t k = 0; k < h; ++k) {
            float w = (float)oracle_half_to_double(W[k * o + j]);
            Wq[j * h + k] = (int8_t)oracle_quantize_value(w, aw[j]);
        }
    }
    return ORACLE_OK;
}

int oracle_prepare_weight(const uint16_t *W, int64_t h, int64_t o,
                          int8_t *Wq, float *aw)
{
    return oracle_prepare_weight_mode(W, h, o, 0, Wq, aw);
}

/* ------------------------------------------------------ Step 1: detection */

/* [P4] Step 1: column j is an outlier feature when some row holds
 * |X[i][j]| >= alpha. flags[j] in {0,1}; idx lists the outlier columns in
 * ascending order; *n_out is their number. */
int oracle_detect_outliers(const uint16_t *X, int64_t s, int64_t h,
                           float alpha, uint8_t *flags, int32_t *idx,
                           int32_t *n_out)
{
    if ((!X && s * h > 0) || !flags || !n_out || s < 0 || h < 0)
        return ORACLE_ERR_ARG;
    double a = (double)alpha;
    int32_t n = 0;
    for (int64_t j = 0; j < h; ++j) {
        int hit = 0;
        for (int64_t i = 0; i < s; ++i) {
            if (fabs(oracle_half_to_double(X[i * h + j])) >= a) {
                hit = 1;
                break;
            }
        }
        flags[j] = (uint8_t)hit;
        if (hit) {
            if (idx)
                idx[n] = (int32_t)j;
            ++n;
        }
    }
    *n_out = n;
    return ORACLE_OK;
}

/* ----------------------------------------- Step 4: row scales, row codes */

/* [P4] Step 4 bullets 1 and 3: ax[i] = max over non-outlier columns of
 * |X[i][j]| (0 when there is none), Xq[i][j] = Q(X[i][j], ax[i]) on
 * non-outlier columns and 0 on outlier columns. Rows are taken from `rows`
 * (nrows of them; all rows when rows == NULL); output row r is rows[r]. */
/* Largest |X[i][j]| over the non-outlier columns of row i. */
static double regular_absmax(const uint16_t *X, int64_t h, const uint8_t *flags, int64_t i)
{
    double m = 0.0;
    for (int64_t j = 0; j < h; ++j) {
        if (flags[j])
            continue;
        double v = fabs(oracle_half_to_double(X[i * h + j]));
        if (v > m)
            m = v;
    }
    return m;
}

/* With `tensor` set, the tensor-wise baseline of [P4] "Quantization
 * Primitives" on the activation side: one constant for all of X (the
 * largest regular |X| of every row), so ax[r] is that constant for every
 * row. */
int oracle_quantize_rows_mode(const uint16_t *X, int64_t s, int64_t h,
                              const uint8_t *flags, const int64_t *rows,
                              int64_t nrows, int tensor, int8_t *Xq, float *ax)
{
    if ((!X && s * h > 0) || !flags || !ax || s < 0 || h < 0)
        return ORACLE_ERR_ARG;
    if (!rows)
        nrows = s;
    double all = 0.0;
    if (tensor)
        for (int64_t i = 0; i < s; ++i) {
            double m = regular_absmax(X, h, flags, i);
            if (m > all)
                all = m;
        }
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        ax[r] = (float)(tensor ? all : regular_absmax(X, h, flags, i));
        if (Xq) {
            for (int64_t j = 0; j < h; ++j) {
                float x = (float)oracle_half_to_double(X[i * h + j]);
                Xq[r * h + j] =
                    flags[j] ? 0 : (int8_t)oracle_quantize_value(x, ax[r]);
            }
        }
    }
    return ORACLE_OK;
}

int oracle_quantize_rows(const uint16_t *X, int64_t s, int64_t h,
                         const uint8_t *flags, const int64_t *rows,
                         int64_t nrows, int8_t *Xq, float *ax)
{
    return oracle_quantize_rows_mode(X, s, h, flags, rows, nrows, 0, Xq, ax);
}

/* ------------------------------------------------ Step 4: int8 x int8 sum */

/* Ci[r][c] = sum_k Xq[r][k] * Wq[cols[c]][k], exact in int64, then checked
 * to fit int32 (the accumulator width the pages name). Xq holds nrows rows
 * of h codes; Wq is [o][h]. cols == NULL means all o columns. */
int oracle_int8_gemm(const int8_t *Xq, int64_t nrows, int64_t h,
                     const int8_t *Wq, int64_t o, const int64_t *cols,
                     int64_t ncols, int32_t *Ci)
{
    if (!Xq || !Wq || !Ci || nrows < 0 || h < 0 || o < 0)
        return ORACLE_ERR_ARG;
    if (!cols)
        ncols = o;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t r = 0; r < nrows; ++r) {
        for (int64_t c = 0; c < ncols; ++c) {
            int64_t j = cols ? cols[c] : c;
            int64_t acc = 0;
            for (int64_t k = 0; k < h; ++k)
                acc += (int64_t)Xq[r * h + k] * (int64_t)Wq[j * h + k];
            if (acc > INT32_MAX || acc < INT32_MIN)
                bad = 1;
            Ci[r * ncols + c] = (int32_t)acc;
        }
    }
    return bad ? ORACLE_ERR_OVERFLOW : ORACLE_OK;
}

/* ------------------------------------------- Step 2: fp16 outlier weights */

/* The rows of W that belong to the outlier columns of X ([P4] Step 2),
 * recovered from the int8 weight: WO[t][j] = fp16(fp32(fp32(Wq[j][O_t]) *
 * aw[j]) / 127). The product of a 7-bit code and a binary16 scale is exact in
 * fp32; the division is one IEEE fp32 rounding; the result is rounded once
 * more to binary16. */
int oracle_outlier_weights(const int8_t *Wq, const float *aw, int64_t h,
                           int64_t o, const int32_t *idx, int32_t n,
                           uint16_t *WO)
{
    if ((n > 0 && (!Wq || !aw || !idx || !WO)) || n < 0)
        return ORACLE_ERR_ARG;
    for (int32_t t = 0; t < n; ++t) {
        int64_t k = idx[t];
        if (k < 0 || k >= h)
            return ORACLE_ERR_ARG;
        for (int64_t j = 0; j < o; ++j) {
            float prod = (float)Wq[j * h + k] * aw[j];
            float v = prod / 127.0f;
            WO[t * o + j] = oracle_double_to_half((double)v);
        }
    }
    return ORACLE_OK;
}

/* ----------------------------------------------------- Steps 1-5 together */

/* The full procedure ([P4] "The Full LLM.int8() Algorithm", Steps 1-5;
 * [P1]/[P2] mixed-precision decomposition) for the output rows `rows` and
 * columns `cols` (NULL = all), given the prepared weight (Wq [o][h], aw [o]).
 *
 *   1. O from all s rows of X (|x| >= alpha).
 *   2. XO = X[:, O]; WO from Wq as in oracle_outlier_weights, or, when the
 *      caller's fp16 weight W16 ([h][o], nullable) is given, the outlier rows
 *      of W themselves, WO[t][j] = W16[O_t][j] ([P4] "Mixed-Precision
 *      Decomposition": the outlier part of W stays in fp16).
 *   3. E[i][j] = sum_t XO[i][t] * WO[t][j]                 (fp64)
 *   4. ax, Xq as in oracle_quantize_rows; Ci exact;
 *      D[i][j] = Ci[i][j] * ax[i] * aw[j] / (127 * 127)     (fp64)
 *   5. out[i][j] = fp16(D[i][j] + E[i][j])                  (one rounding)
 *
 * With x_tensor, step 4 uses one constant for all of X (the tensor-wise
 * baseline, see oracle_quantize_rows_mode); a tensor-wise W is a prepared
 * weight from oracle_prepare_weight_mode.
 *
 * out is [nrows][ncols] binary16; Ci_out (nullable) receives the int32
 * accumulators of the same outputs. */
int oracle_matmul(const uint16_t *X, int64_t s, int64_t h, const int8_t *Wq,
                  const float *aw, int64_t o, const uint16_t *W16, float alpha,
                  int x_tensor, const int64_t *rows, int64_t nrows,
                  const int64_t *cols, int64_t ncols, uint16_t *out, int32_t *Ci_out)
{
    if (s < 0 || h < 0 || o < 0 || !out || (!X && s * h > 0) ||
        (!Wq && h * o > 0) || (!aw && o > 0))
        return ORACLE_ERR_ARG;
    if (!rows)
        nrows = s;
    if (!cols)
        ncols = o;
    int rc = ORACLE_OK;

    uint8_t *flags = (uint8_t *)calloc((size_t)(h > 0 ? h : 1), 1);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)(h > 0 ? h : 1));
    int8_t *Xq = (int8_t *)malloc((size_t)(nrows * h > 0 ? nrows * h : 1));
    float *ax = (float *)malloc(sizeof(float) * (size_t)(nrows > 0 ? nrows : 1));
    int32_t *Ci = (int32_t *)malloc(sizeof(int32_t) *
                                    (size_t)(nrows * ncols > 0 ? nrows * ncols : 1));
    int32_t n = 0;
    uint16_t *WO = NULL;
    if (!flags || !idx || !Xq || !ax || !Ci) {
        rc = ORACLE_ERR_ARG;
        goto done;
    }
    /* Step 1 */
    rc = oracle_detect_outliers(X, s, h, alpha, flags, idx, &n);
    if (rc)
        goto done;
    /* Step 2 (weight side) */
    WO = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(n * o > 0 ? n * o : 1));
    if (!WO) {
        rc = ORACLE_ERR_ARG;
        goto done;
    }
    if (W16) {
        for (int32_t t = 0; t < n; ++t)
            for (int64_t j = 0; j < o; ++j)
                WO[t * o + j] = W16[(int64_t)idx[t] * o + j];
    } else {
        rc = oracle_outlier_weights(Wq, aw, h, o, idx, n, WO);
        if (rc)
            goto done;
    }
    /* Step 4: codes and exact integer product */
    rc = oracle_quantize_rows_mode(X, s, h, flags, rows, nrows, x_tensor, Xq, ax);
    if (rc)
        goto done;
    rc = oracle_int8_gemm(Xq, nrows, h, Wq, o, cols, ncols, Ci);
    if (rc)
        goto done;
    /* Steps 3, 4 (dequantisation) and 5 */
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        for (int64_t c = 0; c < ncols; ++c) {
            int64_t j = cols ? cols[c] : c;
            double e = 0.0;
            for (int32_t t = 0; t < n; ++t)
                e += oracle_half_to_double(X[i * h + idx[t]]) *
                     oracle_half_to_double(WO[t * o + j]);
            double d = (double)Ci[r * ncols + c] * (double)ax[r] *
                       (double)aw[j] / (127.0 * 127.0);
            out[r * ncols + c] = oracle_double_to_half(d + e);
        }
    }
    if (Ci_out)
        memcpy(Ci_out, Ci, sizeof(int32_t) * (size_t)(nrows * ncols));
done:
    free(flags);
    free(idx);
    free(Xq);
    free(ax);
    free(Ci);
    free(WO);
    return rc;
}

/* Threads the OpenMP loops above use. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
