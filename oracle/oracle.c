/*
 * oracle.c -- plain, slow, FP64 CPU oracle for the LM-head loss path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this file:
 * only tests/, the smoke check in __graft_entry__.py and the cpu_baseline /
 * reference arm of bench.py load it.  It shares no code, header or constant
 * with the CUDA library (lm_head_fp32_b200/csrc), and it never includes a
 * CUDA header.
 *
 * Sources (page title, then section):
 *   [P1]  Megatron-LM PR #6252 "Add mixed-precision (FP32) LM output logits",
 *         "What does this PR do?", "Tests", "Integer bitwise exactness
 *         results", "Method".
 *   [P2]  TransformerEngine #2325 "[Pytorch] change fused cross entropy
 *         backward grad to fp32 and reduce one read", "Description",
 *         "Changes" and the review discussion (saved target and m_d_X_y).
 *
 * Every quantity is the plain mathematical definition evaluated in FP64 with
 * the sums taken in index order; results are rounded once, by the caller,
 * to the dtype under test.  No blocking, fusion or reordering of any sum.
 *
 * Pins: every function here is checked in tests/test_oracle.py against
 * something other than itself (exact integer arithmetic, closed forms,
 * library routines in float64, finite differences, invariants).  No function
 * is left "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats.                                                          */
/* ------------------------------------------------------------------------ */

/* bfloat16 is, by definition, the upper 16 bits of an IEEE binary32 word,
 * so widening is a shift; float -> double is exact. */
double oracle_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round an FP64 value to bfloat16 with round-to-nearest-even, in ONE step
 * (no detour through binary32, which could round twice).  bfloat16 keeps 8
 * significant bits and binary32's exponent range: for |v| in [2^(e-1), 2^e)
 * the spacing is 2^(e-8); below 2^-126 the spacing is the subnormal step
 * 2^-133.  v / q is exact (q is a power of two), rint() rounds half to even
 * in the default rounding mode, and a result of 2^128 or more overflows to
 * infinity. */
uint16_t oracle_f64_to_bf16(double v)
{
    if (isnan(v))
        return (uint16_t)0x7FC0u;
    uint16_t sign = signbit(v) ? (uint16_t)0x8000u : (uint16_t)0u;
    double a = fabs(v);
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e);                 /* a = f * 2^e, 0.5 <= f < 1 */
    int qexp = e - 8;
    if (qexp < -133)
        qexp = -133;
    double q = ldexp(1.0, qexp);
    double r = rint(a / q) * q;
    if (r >= ldexp(1.0, 128))
        return (uint16_t)(sign | 0x7F80u);
    float rf = (float)r;          /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &rf, sizeof u);
    return (uint16_t)(sign | (uint16_t)(u >> 16));
}

/* ------------------------------------------------------------------------ */
/* a1: logits = X . W^T  ([P1] "What does this PR do?": the FP32 GEMM output  */
/* keeps the accumulator instead of rounding each logit to BF16).           */
/* ------------------------------------------------------------------------ */

/* out[r*V + v] = sum_{k=0}^{K-1} X[i,k] * W[v,k], i = rows[r] (or r when
 * rows == NULL, n_rows == M).  X is [M,K], W is [V,K], both bf16, row-major.
 * Each bf16 x bf16 product is exact in FP64 (16 significant bits). */
void oracle_logits(const uint16_t *X, const uint16_t *W, int64_t M, int64_t K,
                   int64_t V, const int64_t *rows, int64_t n_rows, double *out)
{
    (void)M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t i = rows ? rows[r] : r;
        const uint16_t *x = X + i * K;
        for (int64_t v = 0; v < V; ++v) {
            const uint16_t *w = W + v * K;
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k)
                s += oracle_bf16_to_f64(x[k]) * oracle_bf16_to_f64(w[k]);
            out[r * V + v] = s;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* a2: cross-entropy forward statistics per row ([P2] discussion: the        */
/* forward saves the target and m_d_X_y, n_rows x 4).                       */
/* ------------------------------------------------------------------------ */

/* Row status codes returned by oracle_ce_row. */
#define ORACLE_ROW_VALID 0
#define ORACLE_ROW_IGNORED 1
#define ORACLE_ROW_BAD_TARGET 2

/* For one row x[0..V) with target y:
 *   m   = max_j x_j
 *   s   = sum_{j != y} exp(x_j - m)        (the other columns' share)
 *   d   = s + exp(x_y - m)                 (= sum_j exp(x_j - m))
 *   x_y = x_y
 *   loss = -log softmax(x)_y = log(d / exp(x_y - m)) = log1p(s * exp(m - x_y))
 * The loss is the same value as m + log(d) - x_y, written through s: when the
 * target holds nearly all of the row's mass, d = 1 + s rounds most of s away
 * (even in FP64 for s below ~1e-12), and log(d) would lose it.
 * y == ignore_index: the row is ignored (loss 0, stats 0, x not read).
 * y outside [0,V) and not ignore_index: reported as a bad target and
 * treated like an ignored row.  *s_out (may be NULL) receives s. */
static int oracle_ce_row(const float *x, int64_t V, int64_t y,
                         int64_t ignore_index, double st[4], double *s_out)
{
    st[0] = st[1] = st[2] = st[3] = 0.0;
    if (s_out)
        *s_out = 0.0;
    if (y == ignore_index)
        return ORACLE_ROW_IGNORED;
    if (y < 0 || y >= V)
        return ORACLE_ROW_BAD_TARGET;
    double m = -INFINITY;
    for (int64_t j = 0; j < V; ++j)
        if ((double)x[j] > m)
            m = (double)x[j];
    double s = 0.0;
    for (int64_t j = 0; j < V; ++j)
        if (j != y)
            s += exp((double)x[j] - m);
    double xy = (double)x[y];
    st[0] = m;
    st[1] = s + exp(xy - m);
    st[2] = xy;
    st[3] = log1p(s * exp(m - xy));
    if (s_out)
        *s_out = s;
    return ORACLE_ROW_VALID;
}

/* stats[r*4 + {0,1,2,3}] = {m, d, x_y, loss} of row rows[r] (or r).
 * row_code[r] (may be NULL) receives ORACLE_ROW_*. */
void oracle_ce_fwd(const float *logits, const int64_t *target, int64_t M,
                   int64_t V, int64_t ignore_index, const int64_t *rows,
                   int64_t n_rows, double *stats, int32_t *row_code)
{
    (void)M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t i = rows ? rows[r] : r;
        int c = oracle_ce_row(logits + i * V, V, target[i], ignore_index,
                              stats + r * 4, NULL);
        if (row_code)
            row_code[r] = c;
    }
}

/* ------------------------------------------------------------------------ */
/* a3: cross-entropy backward in FP64 ([P2] "Description"/"Changes": the     */
/* gradient is computed in FP32 rather than BF16; [P1] "What does this PR   */
/* do?": the cast down to BF16 happens after it).                           */
/* ------------------------------------------------------------------------ */

/* d loss_i / d x_ij = softmax(x_i)_j - [j == y_i], scaled by the upstream
 * gradient g_i = grad_loss[i * grad_stride] (stride 0: one scalar).
 * softmax_j = exp(x_j - m) / d with m, d recomputed here from the logits; at
 * the target, softmax_y - 1 = -s / d (s: the other columns' share, as in
 * oracle_ce_row), the same value without the cancellation of 1 - 1.
 * Ignored and bad-target rows have gradient exactly 0. */
void oracle_ce_bwd(const float *logits, const int64_t *target,
                   const float *grad_loss, int64_t grad_stride, int64_t M,
                   int64_t V, int64_t ignore_index, const int64_t *rows,
                   int64_t n_rows, double *dlogits)
{
    (void)M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t i = rows ? rows[r] : r;
        const float *x = logits + i * V;
        double *out = dlogits + r * V;
        double st[4], s;
        int c = oracle_ce_row(x, V, target[i], ignore_index, st, &s);
        if (c != ORACLE_ROW_VALID) {
            for (int64_t j = 0; j < V; ++j)
                out[j] = 0.0;
            continue;
        }
        double g = (double)grad_loss[i * grad_stride];
        int64_t y = target[i];
        for (int64_t j = 0; j < V; ++j)
            out[j] = (j == y ? -s / st[1] : exp((double)x[j] - st[0]) / st[1]) * g;
    }
}

/* ------------------------------------------------------------------------ */
/* a4/a5: the two gradient GEMMs of logits = X . W^T ([P1] "What does this   */
/* PR do?": the backward follows the GEMM contract with BF16 gradients).    */
/* ------------------------------------------------------------------------ */

/* dX[r,k] = sum_{v=0}^{V-1} dl[i,v] * W[v,k], i = rows[r] (or r).
 * The loop over k is innermost so that W is read row by row; every output
 * is still one sum taken in ascending v. */
void oracle_dx(const uint16_t *dl, const uint16_t *W, int64_t M, int64_t K,
               int64_t V, const int64_t *rows, int64_t n_rows, double *dX)
{
    (void)M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t i = rows ? rows[r] : r;
        double *acc = dX + r * K;
        for (int64_t k = 0; k < K; ++k)
            acc[k] = 0.0;
        for (int64_t v = 0; v < V; ++v) {
            double a = oracle_bf16_to_f64(dl[i * V + v]);
            const uint16_t *w = W + v * K;
            for (int64_t k = 0; k < K; ++k)
                acc[k] += a * oracle_bf16_to_f64(w[k]);
        }
    }
}

/* dW[r,k] = sum_{i=0}^{M-1} dl[i,v] * X[i,k], v = vrows[r] (or r).
 * k innermost as above; every output is one sum taken in ascending i. */
void oracle_dw(const uint16_t *dl, const uint16_t *X, int64_t M, int64_t K,
               int64_t V, const int64_t *vrows, int64_t n_rows, double *dW)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t v = vrows ? vrows[r] : r;
        double *acc = dW + r * K;
        for (int64_t k = 0; k < K; ++k)
            acc[k] = 0.0;
        for (int64_t i = 0; i < M; ++i) {
            double a = oracle_bf16_to_f64(dl[i * V + v]);
            const uint16_t *x = X + i * K;
            for (int64_t k = 0; k < K; ++k)
                acc[k] += a * oracle_bf16_to_f64(x[k]);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Rounding of whole arrays, for the comparisons.                           */
/* ------------------------------------------------------------------------ */

void oracle_round_f32(const double *in, int64_t n, float *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = (float)in[j];
}

void oracle_round_bf16(const double *in, int64_t n, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = oracle_f64_to_bf16(in[j]);
}

int oracle_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
