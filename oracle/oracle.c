/*
 * oracle.c -- plain fp64 CPU oracle for the fused tensor-core GEMM
 *
 *     C = epilogue(A . B),   epilogue(x)[i,j] = GELU(x[i,j] + bias[j])  or  identity
 *     (or bias only, GELU only, and the tanh form of GELU with or without bias)
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check of the build
 * entry point and the CPU-baseline leg of the benchmark may load this file.
 * The product path never calls it, never links it, and shares no code with it.
 *
 * What it follows:
 *   - "Designing High-Performance GPU Kernels with TileLang" (blog retelling),
 *     Step 4 "Tensor-Core GEMM": A_shared is (block_M, block_K), B_shared is
 *     (block_K, block_N), so A is M x K and B is K x N, both row-major; the
 *     accumulator fragment is float32.  Here the accumulation is done in fp64,
 *     an exact stand-in: every product of two fp16 (or two bf16) values is
 *     exact in fp64, so the only error left is the fp64 summation.
 *   - TileLang GPU kernel design article, paragraph 5 (fused GEMM epilogue):
 *     bias add, then GELU, applied to the accumulator before the one write
 *     of the output.  Read as: per-column bias (length N), added
 *     first; GELU in its exact form 0.5 x (1 + erf(x / sqrt 2)).  The bias-only
 *     and GELU-only epilogues are the same steps with one of them left out.
 *
 * Plain definition, no blocking, no reordering: for each output element the
 * sum over k runs k = 0 .. K-1 in order, in double.  The result is kept in
 * fp64 and is NOT rounded to the input dtype.
 *
 * Inputs are raw 16-bit patterns (IEEE binary16 or bfloat16), decoded here
 * from the format definitions.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#ifndef M_PI
#define M_PI 3.14159265358979323846
#endif

#define ORACLE_F16 0
#define ORACLE_BF16 1
#define ORACLE_EPI_NONE 0
#define ORACLE_EPI_BIAS_GELU 1
#define ORACLE_EPI_BIAS 2
#define ORACLE_EPI_GELU 3
#define ORACLE_EPI_BIAS_GELU_TANH 4
#define ORACLE_EPI_GELU_TANH 5

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * Normal: (1024 + f) * 2^(e - 25).  Subnormal (e = 0): f * 2^-24.          */
static double decode_f16(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f + 1024), e - 25);
    return s ? -v : v;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits.
 * Normal: (128 + f) * 2^(e - 134).  Subnormal (e = 0): f * 2^-133.         */
static double decode_bf16(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 7) & 0xff;
    int f = h & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133);
    else if (e == 255)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f + 128), e - 134);
    return s ? -v : v;
}

static double decode(uint16_t h, int dtype)
{
    return dtype == ORACLE_BF16 ? decode_bf16(h) : decode_f16(h);
}

/* Exact (erf) GELU: x * Phi(x) with Phi the standard normal CDF,
 * Phi(x) = (1 + erf(x / sqrt 2)) / 2 = erfc(-x / sqrt 2) / 2.
 * The erfc form is the same function; for negative x the erf form subtracts
 * two numbers close to 1 and keeps only a few correct digits of Phi.        */
double oracle_gelu(double x)
{
    return 0.5 * x * erfc(-x / sqrt(2.0));
}

/* Tanh form of GELU (Hendrycks and Gimpel, "Gaussian Error Linear Units",
 * the approximation of Phi by the logistic-tanh curve):
 *     g(x) = 0.5 x (1 + tanh(u)),   u = sqrt(2 / pi) (x + 0.044715 x^3).
 * Computed through the identity 0.5 (1 + tanh u) = 1 / (1 + exp(-2u))
 * = exp(2u) / (1 + exp(2u)), the same function, taking the form whose
 * exponential is at most 1: for negative x the 1 + tanh form subtracts two
 * numbers close to 1 (in fp64 it is already 0 at x = -7, where g is about
 * -1e-19), and exp(-2u) alone overflows before g leaves the subnormals.     */
double oracle_gelu_tanh(double x)
{
    const double u = sqrt(2.0 / M_PI) * (x + 0.044715 * x * x * x);
    const double e = exp(-2.0 * fabs(u));
    return u >= 0.0 ? x / (1.0 + e) : x * e / (1.0 + e);
}

void oracle_gelu_tanh_array(const double *x, double *y, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        y[i] = oracle_gelu_tanh(x[i]);
}

static int epi_has_bias(int epi)
{
    return epi == ORACLE_EPI_BIAS_GELU || epi == ORACLE_EPI_BIAS || epi == ORACLE_EPI_BIAS_GELU_TANH;
}

/* The epilogue on one accumulated value s of column j: bias first, then the
 * activation (article, paragraph 5: bias add, then GELU). */
static double epilogue(double s, const uint16_t *bias, int64_t j, int dtype, int epi)
{
    if (epi_has_bias(epi))
        s = s + decode(bias[j], dtype);
    if (epi == ORACLE_EPI_BIAS_GELU || epi == ORACLE_EPI_GELU)
        s = oracle_gelu(s);
    else if (epi == ORACLE_EPI_BIAS_GELU_TANH || epi == ORACLE_EPI_GELU_TANH)
        s = oracle_gelu_tanh(s);
    return s;
}

void oracle_gelu_array(const double *x, double *y, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        y[i] = oracle_gelu(x[i]);
}

void oracle_decode_array(const uint16_t *bits, int dtype, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = decode(bits[i], dtype);
}

/* Rows `rows[0..nrows)` of C, written densely to out[r * N + j].
 * Returns 0 on success, -1 if a row index is out of range or memory runs out. */
int oracle_gemm_rows(int64_t M, int64_t N, int64_t K,
                     const uint16_t *A, const uint16_t *B, const uint16_t *bias,
                     int dtype, int epi,
                     const int64_t *rows, int64_t nrows, double *out)
{
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= M)
            return -1;
    if (epi < ORACLE_EPI_NONE || epi > ORACLE_EPI_GELU_TANH || (epi_has_bias(epi) && bias == NULL))
        return -1;

    /* B decoded once; every row reads all of it. */
    double *Bd = (double *)malloc((size_t)(K * N > 0 ? K * N : 1) * sizeof(double));
    if (!Bd)
        return -1;
    oracle_decode_array(B, dtype, Bd, K * N);

    int64_t r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nrows; ++r) {
        const int64_t i = rows[r];
        double *c = out + r * N;
        for (int64_t j = 0; j < N; ++j)
            c[j] = 0.0;
        /* c[j] = sum_{k=0}^{K-1} A[i,k] * B[k,j], k in increasing order */
        for (int64_t k = 0; k < K; ++k) {
            const double a = decode(A[i * K + k], dtype);
            const double *b = Bd + k * N;
            for (int64_t j = 0; j < N; ++j)
                c[j] += a * b[j];
        }
        for (int64_t j = 0; j < N; ++j)
            c[j] = epilogue(c[j], bias, j, dtype, epi);
    }
    free(Bd);
    return 0;
}

/* Whole C (M x N, row-major, fp64). */
int oracle_gemm(int64_t M, int64_t N, int64_t K,
                const uint16_t *A, const uint16_t *B, const uint16_t *bias,
                int dtype, int epi, double *C)
{
    int64_t *rows = (int64_t *)malloc((size_t)(M > 0 ? M : 1) * sizeof(int64_t));
    if (!rows)
        return -1;
    for (int64_t i = 0; i < M; ++i)
        rows[i] = i;
    int rc = oracle_gemm_rows(M, N, K, A, B, bias, dtype, epi, rows, M, C);
    free(rows);
    return rc;
}

/* Single elements C[ii[p], jj[p]] for p < npts: the same sum, same k order. */
int oracle_gemm_points(int64_t M, int64_t N, int64_t K,
                       const uint16_t *A, const uint16_t *B, const uint16_t *bias,
                       int dtype, int epi,
                       const int64_t *ii, const int64_t *jj, int64_t npts, double *out)
{
    for (int64_t p = 0; p < npts; ++p)
        if (ii[p] < 0 || ii[p] >= M || jj[p] < 0 || jj[p] >= N)
            return -1;
    if (epi < ORACLE_EPI_NONE || epi > ORACLE_EPI_GELU_TANH || (epi_has_bias(epi) && bias == NULL))
        return -1;
    int64_t p;
#pragma omp parallel for schedule(static)
    for (p = 0; p < npts; ++p) {
        const int64_t i = ii[p], j = jj[p];
        double s = 0.0;
        for (int64_t k = 0; k < K; ++k)
            s += decode(A[i * K + k], dtype) * decode(B[k * N + j], dtype);
        out[p] = epilogue(s, bias, j, dtype, epi);
    }
    return 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------
 * Attention forward, the plain definition (fp64):
 *
 *     O = softmax(scale * Q K^T  [causal: keys j > query i removed]) V
 *     lse_i = log sum_j exp(scale * q_i . k_j)      (over the kept keys)
 *
 * It follows the TileLang GPU kernel design article, paragraph 6 (attention
 * over query, key and value tiles with online softmax: running maximum,
 * normaliser and rescaling -- an evaluation order of this same definition),
 * checked there against PyTorch's scaled dot-product attention, whose
 * causal mask keeps key j <= query i.  Here the scores are summed in d
 * order, the maximum is subtracted before exponentiating (the same value),
 * and the normaliser is applied once at the end.
 *
 * Layout: Q is [BH][Sq][D], K and V are [BH][Sk][D], row-major 16-bit
 * patterns.  Row p of the output is (bh_idx[p], q_idx[p]): O[p][0..D),
 * lse[p] (natural log).  Returns 0, or -1 for an index out of range.
 * ------------------------------------------------------------------------ */
int oracle_attention_rows(int64_t BH, int64_t Sq, int64_t Sk, int64_t D,
                          const uint16_t *Q, const uint16_t *K, const uint16_t *V, int dtype,
                          int causal, double scale,
                          const int64_t *bh_idx, const int64_t *q_idx, int64_t nrows,
                          double *O, double *lse)
{
    for (int64_t p = 0; p < nrows; ++p)
        if (bh_idx[p] < 0 || bh_idx[p] >= BH || q_idx[p] < 0 || q_idx[p] >= Sq)
            return -1;
    if (Sk < 1 || D < 1)
        return -1;
    int64_t p;
#pragma omp parallel for schedule(dynamic, 4)
    for (p = 0; p < nrows; ++p) {
        const int64_t bh = bh_idx[p], i = q_idx[p];
        const uint16_t *q = Q + (bh * Sq + i) * D;
        const int64_t nkeys = causal ? (i + 1 < Sk ? i + 1 : Sk) : Sk;
        double *s = (double *)malloc((size_t)nkeys * sizeof(double));
        double *o = O + p * D;
        if (!s) {
            for (int64_t d = 0; d < D; ++d)
                o[d] = NAN;
            lse[p] = NAN;
            continue;
        }
        double m = -INFINITY;
        for (int64_t j = 0; j < nkeys; ++j) {
            const uint16_t *k = K + (bh * Sk + j) * D;
            double acc = 0.0;
            for (int64_t d = 0; d < D; ++d)
                acc += decode(q[d], dtype) * decode(k[d], dtype);
            s[j] = scale * acc;
            if (s[j] > m)
                m = s[j];
        }
        double l = 0.0;
        for (int64_t d = 0; d < D; ++d)
            o[d] = 0.0;
        for (int64_t j = 0; j < nkeys; ++j) {
            const double w = exp(s[j] - m);
            const uint16_t *v = V + (bh * Sk + j) * D;
            l += w;
            for (int64_t d = 0; d < D; ++d)
                o[d] += w * decode(v[d], dtype);
        }
        for (int64_t d = 0; d < D; ++d)
            o[d] /= l;
        lse[p] = m + log(l);
        free(s);
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Row softmax (TileLang GPU kernel design article, paragraph 5: a row-wise
 * softmax with max and sum reductions): for each row x of a rows x cols
 * matrix, y_j = exp(x_j - max x) / sum_k exp(x_k - max x), in fp64 from the
 * 16-bit inputs.  Returns 0, or -1 for bad sizes.
 * ------------------------------------------------------------------------ */
int oracle_softmax_rows(int64_t rows, int64_t cols, const uint16_t *X, int dtype, double *Y)
{
    if (rows < 0 || cols < 1)
        return -1;
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; ++r) {
        const uint16_t *x = X + r * cols;
        double *y = Y + r * cols;
        double m = -INFINITY;
        for (int64_t j = 0; j < cols; ++j) {
            y[j] = decode(x[j], dtype);
            if (y[j] > m)
                m = y[j];
        }
        double s = 0.0;
        for (int64_t j = 0; j < cols; ++j) {
            y[j] = exp(y[j] - m);
            s += y[j];
        }
        for (int64_t j = 0; j < cols; ++j)
            y[j] /= s;
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Vector add (TileLang GPU kernel design article, paragraph 3; blog retelling,
 * Step 3): C[i] = A[i] + B[i] in float32.  The sum of two floats is exact in
 * double, so rounding it once to float gives the IEEE float32 sum.
 * ------------------------------------------------------------------------ */
void oracle_vector_add(int64_t n, const float *A, const float *B, float *C)
{
    for (int64_t i = 0; i < n; ++i)
        C[i] = (float)((double)A[i] + (double)B[i]);
}
