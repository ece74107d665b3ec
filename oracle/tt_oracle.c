/*
 * tt_oracle.c -- plain fp64 CPU reference for Tensor-Train embedding gather.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code with the CUDA path.
 *
 * What it computes (FlowTT: Exploiting Computation Flow Reuse in Irregular
 * Tensor-Train Embedding, Abstract and section 2.4 "Problem Definition"; TT-Rec
 * abstract for TT-compressed embedding tables):
 *
 *   A table of N rows and D = d_1*...*d_k columns is held as k cores G_j of
 *   shape [r_{j-1}][n_j][d_j][r_j] (row-major, r_0 = r_k = 1).  Row i is split
 *   into mixed-radix digits (i_1..i_k) over (n_1..n_k), i_1 the most
 *   significant digit, and the row is the chained contraction of the slices
 *   G_1[:, i_1], G_2[:, i_2], ..., G_k[:, i_k] taken left to right (the
 *   "C = A.B, then E = C.D" order of section 3.2).  Column c of the row is the
 *   multi-index (a_1..a_k) flattened row-major.  Rows are sum-pooled into bags.
 *
 *   The backward pass is the textbook TT gradient: for the loss
 *   L = sum_b <g_b, out_b>, each lookup adds to dG_j[:, i_j, a_j, :] the
 *   product  Left_j^T * g(a_j) * Right_j^T, where Left_j is the product of the
 *   slices before j, Right_j the product of the slices after j, and g(a_j) is
 *   the bag's upstream gradient viewed as a (prefix columns) x (suffix
 *   columns) matrix at fixed a_j.
 *
 * Every lookup is contracted on its own: no sorting, no deduplication, no
 * prefix sharing.  Arithmetic is fp64 throughout.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define TTO_MAX_K 8

enum { TTO_OK = 0, TTO_ERR_ARG = 1, TTO_ERR_INDEX = 2, TTO_ERR_OFFSETS = 3, TTO_ERR_NOMEM = 4 };

typedef struct {
    int32_t k;
    const int64_t* n;      /* [k] factors of this table */
    const int32_t* d;      /* [k] */
    const int32_t* r;      /* [k+1] */
    const double* const* G;/* [k] cores, G[j] = [r_j][n_j][d_j][r_{j+1}] (0-based j) */
} tto_table;

/* Mixed-radix digits of row i: i_1 (digit[0]) is the most significant. */
static void tto_digits(const tto_table* tb, int64_t i, int64_t* digit)
{
    for (int j = tb->k - 1; j >= 0; --j) {
        digit[j] = i % tb->n[j];
        i /= tb->n[j];
    }
}

/* Element G_j[rho, i_j, a, sigma] of core j (0-based j). */
static inline double tto_core(const tto_table* tb, int j, int64_t rho, int64_t ij, int64_t a,
                              int64_t sigma)
{
    const int64_t nj = tb->n[j], dj = tb->d[j], rj1 = tb->r[j + 1];
    return tb->G[j][((rho * nj + ij) * dj + a) * rj1 + sigma];
}

/*
 * Left partials.  left[j] is the product of slices 0..j-1 as a matrix of
 * (d_0*...*d_{j-1}) rows and r_j columns; left[0] is the 1x1 identity.
 * left[j+1][(alpha, a), sigma] = sum_rho left[j][alpha, rho] * G_j[rho, i_j, a, sigma].
 */
static void tto_left_partials(const tto_table* tb, const int64_t* digit, double** left)
{
    left[0][0] = 1.0;
    int64_t rows = 1;
    for (int j = 0; j < tb->k; ++j) {
        const int64_t rj = tb->r[j], dj = tb->d[j], rj1 = tb->r[j + 1];
        for (int64_t alpha = 0; alpha < rows; ++alpha)
            for (int64_t a = 0; a < dj; ++a)
                for (int64_t sigma = 0; sigma < rj1; ++sigma) {
                    double acc = 0.0;
                    for (int64_t rho = 0; rho < rj; ++rho)
                        acc += left[j][alpha * rj + rho] * tto_core(tb, j, rho, digit[j], a, sigma);
                    left[j + 1][(alpha * dj + a) * rj1 + sigma] = acc;
                }
        rows *= dj;
    }
}

/*
 * Right partials.  right[j] is the product of slices j..k-1 as a matrix of
 * r_j rows and (d_j*...*d_{k-1}) columns; right[k] is the 1x1 identity.
 * right[j][rho, (a, beta)] = sum_sigma G_j[rho, i_j, a, sigma] * right[j+1][sigma, beta].
 */
static void tto_right_partials(const tto_table* tb, const int64_t* digit, double** right)
{
    right[tb->k][0] = 1.0;
    int64_t cols = 1;
    for (int j = tb->k - 1; j >= 0; --j) {
        const int64_t rj = tb->r[j], dj = tb->d[j], rj1 = tb->r[j + 1];
        for (int64_t rho = 0; rho < rj; ++rho)
            for (int64_t a = 0; a < dj; ++a)
                for (int64_t beta = 0; beta < cols; ++beta) {
                    double acc = 0.0;
                    for (int64_t sigma = 0; sigma < rj1; ++sigma)
                        acc += tto_core(tb, j, rho, digit[j], a, sigma) * right[j + 1][sigma * cols + beta];
                    right[j][rho * (dj * cols) + a * cols + beta] = acc;
                }
        cols *= dj;
    }
}

static int64_t tto_dim(const tto_table* tb)
{
    int64_t D = 1;
    for (int j = 0; j < tb->k; ++j) D *= tb->d[j];
    return D;
}

/* Largest left/right partial, in doubles. */
static int64_t tto_partial_size(const tto_table* tb)
{
    int64_t best = 1, rows = 1, cols = 1;
    for (int j = 0; j < tb->k; ++j) {
        rows *= tb->d[j];
        if (rows * tb->r[j + 1] > best) best = rows * tb->r[j + 1];
    }
    for (int j = tb->k - 1; j >= 0; --j) {
        cols *= tb->d[j];
        if (cols * tb->r[j] > best) best = cols * tb->r[j];
    }
    return best;
}

static int tto_check_shapes(int32_t T, int32_t k, const int32_t* d, const int32_t* r)
{
    if (T < 1 || k < 1 || k > TTO_MAX_K) return TTO_ERR_ARG;
    if (r[0] != 1 || r[k] != 1) return TTO_ERR_ARG;
    for (int j = 0; j < k; ++j)
        if (d[j] < 1 || r[j] < 1) return TTO_ERR_ARG;
    return TTO_OK;
}

static int tto_check_inputs(int32_t T, int32_t k, const int64_t* n, const int64_t* n_rows,
                            const int64_t* indices, const int64_t* offsets, int64_t B)
{
    if (offsets[0] != 0) return TTO_ERR_OFFSETS;
    for (int64_t g = 0; g < (int64_t)T * B; ++g)
        if (offsets[g + 1] < offsets[g]) return TTO_ERR_OFFSETS;
    for (int32_t t = 0; t < T; ++t) {
        int64_t prod = 1;
        for (int j = 0; j < k; ++j) prod *= n[t * k + j];
        if (n_rows[t] < 1 || n_rows[t] > prod) return TTO_ERR_ARG;
        for (int64_t l = offsets[(int64_t)t * B]; l < offsets[(int64_t)(t + 1) * B]; ++l)
            if (indices[l] < 0 || indices[l] >= n_rows[t]) return TTO_ERR_INDEX;
    }
    return TTO_OK;
}

/*
 * Forward: out[b][t*D + c] = sum over the lookups i of bag (t, b) of row_t(i)[c].
 *   n       [T*k]   factors n_j of each table
 *   n_rows  [T]     valid rows of each table (indices must be < n_rows[t])
 *   d, r    [k], [k+1]  shared column factors and ranks
 *   cores   [T*k]   fp64 cores, table-major
 *   indices [L], offsets [T*B+1]  table-major bags
 *   out     [B][T*D]  overwritten
 * Returns TTO_OK or an error code; bags are independent (OpenMP over bags).
 */
int tto_forward(int32_t T, int32_t k, const int64_t* n, const int64_t* n_rows, const int32_t* d,
                const int32_t* r, const double* const* cores, const int64_t* indices,
                const int64_t* offsets, int64_t B, double* out, int32_t nthreads)
{
    int rc = tto_check_shapes(T, k, d, r);
    if (rc) return rc;
    rc = tto_check_inputs(T, k, n, n_rows, indices, offsets, B);
    if (rc) return rc;
    int64_t D = 1;
    for (int j = 0; j < k; ++j) D *= d[j];
    if (nthreads < 1) nthreads = 1;
    int failed = 0;

#pragma omp parallel num_threads(nthreads)
    {
        int64_t cap = 1;
        for (int32_t t = 0; t < T; ++t) {
            tto_table tb = {k, n + (int64_t)t * k, d, r, cores + (int64_t)t * k};
            int64_t s = tto_partial_size(&tb);
            if (s > cap) cap = s;
        }
        double* store = (double*)malloc(sizeof(double) * (size_t)cap * (size_t)(k + 1));
        double* left[TTO_MAX_K + 1];
        if (!store) {
#pragma omp atomic write
            failed = 1;
        } else {
            for (int j = 0; j <= k; ++j) left[j] = store + (size_t)j * (size_t)cap;
        }
#pragma omp for schedule(dynamic, 64)
        for (int64_t g = 0; g < (int64_t)T * B; ++g) {
            if (!store) continue;
            const int32_t t = (int32_t)(g / B);
            const int64_t b = g % B;
            tto_table tb = {k, n + (int64_t)t * k, d, r, cores + (int64_t)t * k};
            double* o = out + b * (int64_t)T * D + (int64_t)t * D;
            for (int64_t c = 0; c < D; ++c) o[c] = 0.0;
            for (int64_t l = offsets[g]; l < offsets[g + 1]; ++l) {
                int64_t digit[TTO_MAX_K] = {0};
                tto_digits(&tb, indices[l], digit);
                tto_left_partials(&tb, digit, left);
                /* left[k] is D x r_k = D x 1: the row. */
                for (int64_t c = 0; c < D; ++c) o[c] += left[k][c];
            }
        }
        free(store);
    }
    return failed ? TTO_ERR_NOMEM : TTO_OK;
}

/*
 * Backward: grads[t*k + j] (same shapes as the cores, fp64) are OVERWRITTEN
 * with dL/dG_j for L = sum_b <grad_out[b][t*D:(t+1)*D], out[b][t*D:(t+1)*D]>.
 * For one lookup of row i in bag (t, b), with g = grad_out[b][t*D:(t+1)*D]
 * viewed as [alpha][a_j][beta] (alpha: the d's before j, beta: the d's after):
 *   dG_j[rho, i_j, a_j, sigma] += sum_{alpha, beta}
 *       left[j][alpha, rho] * g[alpha, a_j, beta] * right[j+1][sigma, beta]
 * evaluated as M = left[j]^T g(a_j), then M * right[j+1]^T.
 * Tables are independent (OpenMP over tables); lookups of a table run in order.
 */
int tto_backward(int32_t T, int32_t k, const int64_t* n, const int64_t* n_rows, const int32_t* d,
                 const int32_t* r, const double* const* cores, const int64_t* indices,
                 const int64_t* offsets, int64_t B, const double* grad_out, double* const* grads,
                 int32_t nthreads)
{
    int rc = tto_check_shapes(T, k, d, r);
    if (rc) return rc;
    rc = tto_check_inputs(T, k, n, n_rows, indices, offsets, B);
    if (rc) return rc;
    int64_t D = 1;
    for (int j = 0; j < k; ++j) D *= d[j];
    if (nthreads < 1) nthreads = 1;
    int failed = 0;

#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
    for (int32_t t = 0; t < T; ++t) {
        tto_table tb = {k, n + (int64_t)t * k, d, r, cores + (int64_t)t * k};
        for (int j = 0; j < k; ++j) {
            int64_t sz = (int64_t)r[j] * tb.n[j] * d[j] * r[j + 1];
            memset(grads[(int64_t)t * k + j], 0, sizeof(double) * (size_t)sz);
        }
        int64_t cap = tto_partial_size(&tb);
        int64_t mcap = 1;
        for (int j = 0; j < k; ++j) {
            int64_t s = (int64_t)r[j] * D; /* rho x a_j x beta <= r_j * D */
            if (s > mcap) mcap = s;
        }
        double* store = (double*)malloc(sizeof(double) * ((size_t)cap * (size_t)(2 * k + 2) + (size_t)mcap));
        if (!store) {
#pragma omp atomic write
            failed = 1;
            continue;
        }
        double* left[TTO_MAX_K + 1];
        double* right[TTO_MAX_K + 1];
        for (int j = 0; j <= k; ++j) {
            left[j] = store + (size_t)j * (size_t)cap;
            right[j] = store + (size_t)(k + 1 + j) * (size_t)cap;
        }
        double* M = store + (size_t)cap * (size_t)(2 * k + 2);

        for (int64_t b = 0; b < B; ++b) {
            const int64_t g = (int64_t)t * B + b;
            const double* gb = grad_out + b * (int64_t)T * D + (int64_t)t * D;
            for (int64_t l = offsets[g]; l < offsets[g + 1]; ++l) {
                int64_t digit[TTO_MAX_K] = {0};
                tto_digits(&tb, indices[l], digit);
                tto_left_partials(&tb, digit, left);
                tto_right_partials(&tb, digit, right);
                int64_t arows = 1; /* d_0 * ... * d_{j-1} */
                for (int j = 0; j < k; ++j) {
                    const int64_t rj = r[j], dj = d[j], rj1 = r[j + 1];
                    const int64_t bcols = D / (arows * dj); /* d_{j+1} * ... * d_{k-1} */
                    /* M[rho][a][beta] = sum_alpha left[j][alpha, rho] * g[alpha, a, beta] */
                    for (int64_t rho = 0; rho < rj; ++rho)
                        for (int64_t a = 0; a < dj; ++a)
                            for (int64_t beta = 0; beta < bcols; ++beta) {
                                double acc = 0.0;
                                for (int64_t alpha = 0; alpha < arows; ++alpha)
                                    acc += left[j][alpha * rj + rho] * gb[(alpha * dj + a) * bcols + beta];
                                M[(rho * dj + a) * bcols + beta] = acc;
                            }
                    /* dG_j[rho, i_j, a, sigma] += sum_beta M[rho][a][beta] * right[j+1][sigma, beta] */
                    double* Gj = grads[(int64_t)t * k + j];
                    for (int64_t rho = 0; rho < rj; ++rho)
                        for (int64_t a = 0; a < dj; ++a)
                            for (int64_t sigma = 0; sigma < rj1; ++sigma) {
                                double acc = 0.0;
                                for (int64_t beta = 0; beta < bcols; ++beta)
                                    acc += M[(rho * dj + a) * bcols + beta] * right[j + 1][sigma * bcols + beta];
                                Gj[((rho * tb.n[j] + digit[j]) * dj + a) * rj1 + sigma] += acc;
                            }
                    arows *= dj;
                }
            }
        }
        free(store);
    }
    return failed ? TTO_ERR_NOMEM : TTO_OK;
}

/* Mixed-radix digits of each row (i_1 first), for the pins. */
int tto_digits_batch(int32_t k, const int64_t* n, const int64_t* rows, int64_t count, int64_t* digits)
{
    if (k < 1 || k > TTO_MAX_K) return TTO_ERR_ARG;
    tto_table tb = {k, n, NULL, NULL, NULL};
    for (int64_t q = 0; q < count; ++q) tto_digits(&tb, rows[q], digits + q * k);
    return TTO_OK;
}

/* One row of the virtual table (for the pins), fp64. */
int tto_row(int32_t k, const int64_t* n, const int32_t* d, const int32_t* r,
            const double* const* cores, int64_t row, double* out)
{
    int rc = tto_check_shapes(1, k, d, r);
    if (rc) return rc;
    tto_table tb = {k, n, d, r, cores};
    int64_t cap = tto_partial_size(&tb);
    double* store = (double*)malloc(sizeof(double) * (size_t)cap * (size_t)(k + 1));
    if (!store) return TTO_ERR_NOMEM;
    double* left[TTO_MAX_K + 1];
    for (int j = 0; j <= k; ++j) left[j] = store + (size_t)j * (size_t)cap;
    int64_t digit[TTO_MAX_K] = {0};
    tto_digits(&tb, row, digit);
    tto_left_partials(&tb, digit, left);
    int64_t D = tto_dim(&tb);
    for (int64_t c = 0; c < D; ++c) out[c] = left[k][c];
    free(store);
    return TTO_OK;
}
