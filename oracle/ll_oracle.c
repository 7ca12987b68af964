/*
 * ll_oracle.c -- plain, slow CPU reference of the LiteLinear forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library under rank_fp8_residual_b200/) shares no code with it.
 *
 * What it computes (LiteLinear README, introduction, the display formula):
 *
 *     W ~= A*B + Q_fp8,
 *     y  = (x B^T) A^T + scale * (x Q_fp8^T) + bias
 *
 * with the storage formats of the README's "Features" list: A and B bf16,
 * Q_fp8 e4m3fn, bf16 activations.  Shapes as in the sibling SVDLinearLayer
 * (tt_compressor page, class SVDLinearLayer: A is (out, r), B is (r, in)),
 * Q shaped like nn.Linear.weight, [out, in]:
 *
 *     x [M][K], B [r][K], A [N][r], Q [N][K], scale [N] or [1], bias [N].
 *
 * Every product of two decoded inputs is exact in binary64 (bf16 x bf16 and
 * bf16 x e4m3 products need at most 16 significand bits), and every sum is
 * carried in binary64, so for the sizes used here the result is the exact
 * real value up to binary64 rounding of the running sums.
 *
 * Modes:
 *   LLO_EXACT  (0): t = x B^T is kept unrounded (the graded reference).
 *   LLO_MIRROR (1): t is rounded to bf16 (round to nearest, ties to even)
 *                   before the up-projection, the reading in which the
 *                   low-rank intermediate is held in the activation dtype
 *                   (README "Features": the PyTorch fallback mirrors the
 *                   fused kernel cast-for-cast; modegpt page,
 *                   MoDeGPTLowRankLinear.forward applies F.linear(x, V) in
 *                   the activation dtype).  Diagnostic only.
 *   LLO_FP8ACT (2): the FP8-activation reading.  The residual product
 *                   x Q^T uses x quantised per token to e4m3fn,
 *                   x ~= 2^e_m * q_m, where 2^e_m is the smallest power of
 *                   two with max_k |x[m][k]| <= 448 * 2^e_m and q_m is the
 *                   round-to-nearest-even e4m3fn code of x / 2^e_m (README
 *                   "Features": e4m3fn is the FP8 format of the layer; its
 *                   benchmark's fused "Accel" kernel; the per-token power of
 *                   two is the plainest scale that keeps every product
 *                   exact).  t = x B^T keeps the unquantised x.
 *   LLO_FP8SPLIT (3): x in the residual product is the two-term e4m3fn
 *                   expansion 2^e_m * (hi + lo), hi as in LLO_FP8ACT and
 *                   lo the e4m3fn rounding of x / 2^e_m - hi.  Diagnostic
 *                   mirror of the two-term kernel (graded against
 *                   LLO_EXACT).
 *
 * Parity status: every function here is pinned by the tests under
 * tests/test_oracle_*.py (exhaustive decoder checks against torch's
 * float8_e4m3fn and bfloat16, exact rational brute force on tiny shapes,
 * closed forms, and the r=0 / Q=0 / dense-weight invariants).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define LLO_EXACT 0
#define LLO_MIRROR 1
#define LLO_FP8ACT 2
#define LLO_FP8SPLIT 3
#define LLO_SCALE_PER_TENSOR 0
#define LLO_SCALE_PER_ROW 1

/* e4m3fn (OCP 8-bit float, the "fn" variant named in the README's
 * "Features" list): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
 * bits, no infinities, and S.1111.111 is NaN.
 *   exponent field 0  -> subnormal  (-1)^s * (m / 8) * 2^(1-7)
 *   otherwise         -> normal     (-1)^s * (1 + m / 8) * 2^(e-7)
 */
double llo_dec_e4m3(uint8_t c)
{
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 15;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, 1 - 7);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double llo_dec_bf16(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a binary64 value to the nearest bfloat16 (ties to even) and
 * return its bits.  Written from the format definition: 8 significant
 * bits, exponent range of binary32, gradual underflow below 2^-126. */
uint16_t llo_enc_bf16_rne(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (isnan(v))
        return 0x7FC0u;
    if (isinf(v))
        return sign | 0x7F80u;
    if (a == 0.0)
        return sign;
    int e;
    (void)frexp(a, &e);           /* a = f * 2^e, f in [0.5, 1) */
    int q = e - 8;                /* quantum exponent for 8 significant bits */
    if (q < -133)                 /* subnormal range: fixed quantum 2^-133 */
        q = -133;
    double n = ldexp(a, -q);      /* exact: a / 2^q */
    double fl = floor(n);
    double fr = n - fl;
    double rn;
    if (fr > 0.5)
        rn = fl + 1.0;
    else if (fr < 0.5)
        rn = fl;
    else
        rn = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    double r = ldexp(rn, q);
    /* largest finite bf16 is (2 - 2^-7) * 2^127 */
    if (r > ldexp(2.0 - ldexp(1.0, -7), 127))
        return sign | 0x7F80u;
    float f = (float)r;           /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)((u >> 16) & 0x7FFFu);
}

/* Round a binary64 value to e4m3fn, nearest with ties to the even code,
 * and return the code.  Magnitudes above 448 give 448 (the largest finite
 * code; e4m3fn has no infinity), NaN gives 0x7F.  Written as a search
 * over the 127 finite non-negative codes, whose values are given in
 * `pos` (pos[c] = llo_dec_e4m3(c), c = 0x00 .. 0x7E): the nearest value
 * wins, and of two equally near ones (always adjacent codes) the even
 * code. */
static uint8_t enc_e4m3_search(double v, const double *pos)
{
    if (isnan(v))
        return 0x7Fu;
    uint8_t sign = signbit(v) ? 0x80u : 0u;
    double a = fabs(v);
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(pos[c] - a);
        if (d < bd || (d == bd && (c & 1) == 0)) {
            best = c;
            bd = d;
        }
    }
    return sign | (uint8_t)best;
}

static void e4m3_positive_values(double *pos)
{
    for (int c = 0; c <= 0x7E; ++c)
        pos[c] = llo_dec_e4m3((uint8_t)c);
}

uint8_t llo_enc_e4m3_rne(double v)
{
    double pos[0x7F];
    e4m3_positive_values(pos);
    return enc_e4m3_search(v, pos);
}

/* Per-token exponent of the FP8-activation readings: the smallest integer
 * e with amax <= 448 * 2^e, limited to [-126, 126] (so that 2^e and 2^-e
 * are normal binary32 numbers); 0 for amax == 0. */
int llo_token_exp(double amax)
{
    if (!(amax > 0.0))
        return 0;
    int e = -126;
    while (e < 126 && amax > ldexp(448.0, e))
        ++e;
    return e;
}

/* Quantise one token row: returns e_m and writes the codes hi[k] (and
 * lo[k] when terms == 2) of u = x[k] / 2^e_m:  hi = e4m3(u),
 * lo = e4m3(u - hi).  `pos` as for enc_e4m3_search. */
static int quant_row(const uint16_t *xr, int K, int terms, const double *pos, uint8_t *hi, uint8_t *lo)
{
    double amax = 0.0;
    for (int k = 0; k < K; ++k) {
        double a = fabs(llo_dec_bf16(xr[k]));
        if (a > amax)
            amax = a;
    }
    int e = llo_token_exp(amax);
    for (int k = 0; k < K; ++k) {
        double u = ldexp(llo_dec_bf16(xr[k]), -e);
        uint8_t h = enc_e4m3_search(u, pos);
        hi[k] = h;
        if (terms == 2)
            lo[k] = enc_e4m3_search(u - llo_dec_e4m3(h), pos);
    }
    return e;
}

/* The per-token quantisation of x [M][K] used by the FP8-activation
 * readings: e_out [M], hi [M][K] and, for terms == 2, lo [M][K].
 * Returns 0, or -1 on bad arguments. */
int llo_quant_x(int M, int K, const uint16_t *x, int terms, int *e_out, uint8_t *hi, uint8_t *lo)
{
    if (M < 0 || K < 0 || (terms != 1 && terms != 2) || (M > 0 && (!x || !e_out || !hi)) ||
        (M > 0 && terms == 2 && !lo))
        return -1;
    double pos[0x7F];
    e4m3_positive_values(pos);
    for (int m = 0; m < M; ++m)
        e_out[m] = quant_row(x + (size_t)m * (size_t)K, K, terms, pos, hi + (size_t)m * (size_t)K,
                             terms == 2 ? lo + (size_t)m * (size_t)K : NULL);
    return 0;
}

/*
 * The residual quantisation of the decomposition step (LiteLinear README,
 * "Usage": LiteLinear.from_dense, an SVD-based decomposition; the MoDeGPT
 * compressor's _decompose_single keeps U_r S_r and V_r^T as the two
 * factors).  Given W [N][K] and the bf16 factors A [N][r], B [r][K]:
 *
 *   R[n][k]  = W[n][k] - sum_j A[n][j] * B[j][k]      (binary64, j in order)
 *   amax     = max_k |R[n][k]|  (per row)  or  max over all of R (per tensor)
 *   scale    = amax / 448, rounded to binary32 (0 when amax == 0)
 *   Q[n][k]  = e4m3fn code nearest to (binary32)(R[n][k] / scale), ties to
 *              even, saturating at 448; 0 where scale == 0
 *
 * The pages do not state how the residual's scale is chosen; the plainest
 * reading maps each row's largest magnitude to the largest e4m3fn value.
 * The rounding steps are fixed so that the decision of every code is taken
 * in the same precision wherever it is computed.  Writes Q [N][K] and
 * scale [N] (per row) or [1] (per tensor).  Returns 0, or -1 on bad
 * arguments.
 */
int llo_residual_quant(int N, int K, int r, const uint16_t *W, const uint16_t *A, const uint16_t *B,
                       int scale_mode, uint8_t *Q, float *scale)
{
    if (N < 0 || K < 0 || r < 0 || (N > 0 && K > 0 && (!W || !Q)) || !scale ||
        (r > 0 && N > 0 && K > 0 && (!A || !B)))
        return -1;
    if (scale_mode != LLO_SCALE_PER_TENSOR && scale_mode != LLO_SCALE_PER_ROW)
        return -1;
    double pos[0x7F];
    e4m3_positive_values(pos);
    double *R = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1) * (size_t)(K > 0 ? K : 1));
    if (!R)
        return -1;
    double gmax = 0.0;
    for (int n = 0; n < N; ++n) {
        for (int k = 0; k < K; ++k) {
            double acc = 0.0;
            for (int j = 0; j < r; ++j)
                acc = acc + llo_dec_bf16(A[(size_t)n * r + j]) * llo_dec_bf16(B[(size_t)j * K + k]);
            double v = llo_dec_bf16(W[(size_t)n * K + k]) - acc;
            R[(size_t)n * K + k] = v;
            if (fabs(v) > gmax)
                gmax = fabs(v);
        }
    }
    if (scale_mode == LLO_SCALE_PER_TENSOR)
        scale[0] = (float)(gmax / 448.0);
    for (int n = 0; n < N; ++n) {
        float s;
        if (scale_mode == LLO_SCALE_PER_ROW) {
            double amax = 0.0;
            for (int k = 0; k < K; ++k)
                if (fabs(R[(size_t)n * K + k]) > amax)
                    amax = fabs(R[(size_t)n * K + k]);
            s = (float)(amax / 448.0);
            scale[n] = s;
        } else {
            s = scale[0];
        }
        for (int k = 0; k < K; ++k) {
            uint8_t c = 0;
            if (s != 0.0f) {
                float u = (float)(R[(size_t)n * K + k] / (double)s);
                c = enc_e4m3_search((double)u, pos);
            }
            Q[(size_t)n * K + k] = c;
        }
    }
    free(R);
    return 0;
}

/*
 * The forward pass for the rows listed in `rows` (or all M rows when
 * rows == NULL), written out as the definition:
 *
 *   t[j]    = sum_k x[m][k] * B[j][k]                      (j < r)
 *   yq[n]   = sum_k x[m][k] * Q[n][k]                      (decoded e4m3)
 *   ylr[n]  = sum_j t[j] * A[n][j]
 *   y[i][n] = s_n * yq[n] + ylr[n] + bias[n]
 *
 * In the FP8 modes yq uses the quantised row (see the mode list above).
 *
 * s_n = scale[n] (per row) or scale[0] (per tensor); bias may be NULL.
 * Output y is [nrows][N] binary64, where nrows = M when rows == NULL.
 * Returns 0 on success, -1 on bad arguments or allocation failure.
 */
int llo_forward(int M, int K, int N, int r,
                const uint16_t *x, const uint16_t *B, const uint16_t *A,
                const uint8_t *Q, const float *scale, int scale_mode,
                const uint16_t *bias, int mode,
                const int *rows, int nrows, double *y)
{
    if (M < 0 || K < 0 || N < 0 || r < 0 || !y)
        return -1;
    if (mode != LLO_EXACT && mode != LLO_MIRROR && mode != LLO_FP8ACT && mode != LLO_FP8SPLIT)
        return -1;
    if (scale_mode != LLO_SCALE_PER_TENSOR && scale_mode != LLO_SCALE_PER_ROW)
        return -1;
    if ((M > 0 && K > 0 && !x) || (N > 0 && K > 0 && !Q) || (N > 0 && !scale))
        return -1;
    if (r > 0 && ((K > 0 && !B) || (N > 0 && !A)))
        return -1;
    if (!rows)
        nrows = M;
    if (nrows < 0)
        return -1;
    for (int i = 0; rows && i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= M)
            return -1;

    /* Decode tables and decoded factors (binary64). */
    double dq[256];
    for (int c = 0; c < 256; ++c)
        dq[c] = llo_dec_e4m3((uint8_t)c);
    double pos[0x7F];
    e4m3_positive_values(pos);
    double *Bd = NULL, *Ad = NULL;
    if (r > 0) {
        Bd = (double *)malloc(sizeof(double) * (size_t)r * (size_t)(K > 0 ? K : 1));
        Ad = (double *)malloc(sizeof(double) * (size_t)N * (size_t)r + 8);
        if (!Bd || !Ad) {
            free(Bd);
            free(Ad);
            return -1;
        }
        for (size_t i = 0; i < (size_t)r * (size_t)K; ++i)
            Bd[i] = llo_dec_bf16(B[i]);
        for (size_t i = 0; i < (size_t)N * (size_t)r; ++i)
            Ad[i] = llo_dec_bf16(A[i]);
    }
    int fail = 0;

#pragma omp parallel
    {
        double *xd = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
        double *xq = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
        uint8_t *qh = (uint8_t *)malloc((size_t)(K > 0 ? K : 1));
        uint8_t *ql = (uint8_t *)malloc((size_t)(K > 0 ? K : 1));
        double *t = (double *)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
        if (!xd || !xq || !qh || !ql || !t) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int i = 0; i < nrows; ++i) {
                int m = rows ? rows[i] : i;
                const uint16_t *xr = x + (size_t)m * (size_t)K;
                for (int k = 0; k < K; ++k)
                    xd[k] = llo_dec_bf16(xr[k]);
                /* the row that enters x Q^T */
                const double *xr_q = xd;
                if (mode == LLO_FP8ACT || mode == LLO_FP8SPLIT) {
                    int terms = mode == LLO_FP8ACT ? 1 : 2;
                    int e = quant_row(xr, K, terms, pos, qh, ql);
                    for (int k = 0; k < K; ++k) {
                        double v = llo_dec_e4m3(qh[k]);
                        if (terms == 2)
                            v += llo_dec_e4m3(ql[k]);
                        xq[k] = ldexp(v, e);
                    }
                    xr_q = xq;
                }
                /* t = x B^T */
                for (int j = 0; j < r; ++j) {
                    const double *bj = Bd + (size_t)j * (size_t)K;
                    double acc = 0.0;
                    for (int k = 0; k < K; ++k)
                        acc += xd[k] * bj[k];
                    t[j] = (mode == LLO_MIRROR) ? llo_dec_bf16(llo_enc_bf16_rne(acc)) : acc;
                }
                double *yr = y + (size_t)i * (size_t)N;
                for (int n = 0; n < N; ++n) {
                    const uint8_t *qn = Q + (size_t)n * (size_t)K;
                    double yq = 0.0;
                    for (int k = 0; k < K; ++k)
                        yq += xr_q[k] * dq[qn[k]];
                    double ylr = 0.0;
                    const double *an = Ad ? Ad + (size_t)n * (size_t)r : NULL;
                    for (int j = 0; j < r; ++j)
                        ylr += t[j] * an[j];
                    double s = (double)scale[scale_mode == LLO_SCALE_PER_ROW ? n : 0];
                    double b = bias ? llo_dec_bf16(bias[n]) : 0.0;
                    yr[n] = s * yq + ylr + b;
                }
            }
        }
        free(xd);
        free(xq);
        free(qh);
        free(ql);
        free(t);
    }
    free(Bd);
    free(Ad);
    return fail ? -1 : 0;
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int llo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
