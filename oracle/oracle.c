/*
 * Oracle for the fused linear cross-entropy forward: plain, slow, fp64, CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this file; only the test suite, the smoke check and the CPU-baseline leg
 * of the benchmark use it.  It shares no code, header or constant with the CUDA
 * library.
 *
 * Source: D. Ineshin, "Een gefuseerde forward-kernel voor lineaire
 * cross-entropy op Apple-GPU's" (2026), section 1 ("De loss streamen zonder
 * volledige logits"):
 *   - the logits are Z = H W^T, with H an (N, D) matrix of hidden states and
 *     W the (V, D) output projection;
 *   - the per-token loss is loss_i = logsumexp(Z_i) - Z_{i, y_i};
 *   - the loss needs just two statistics of each row: its log-sum-exp and
 *     its target logit.
 * The method reaches this plain definition exactly (up to rounding order), so
 * the oracle is that definition written out: it materialises one full logits
 * row in fp64 and does a two-pass log-sum-exp (max pass, then sum of exp).
 * It deliberately does NOT stream vocab tiles or use the online (m, s)
 * recurrence; that is the thing under test.
 *
 * Readings of points the page leaves open:
 *   - log is the natural logarithm;
 *   - inputs are converted exactly to fp64 from their stored type (bf16 bit
 *     patterns or fp32), and every dot product is a sequential fp64 sum over
 *     k = 0..D-1;
 *   - a target outside [0, V) is invalid input: the call fails with
 *     ORACLE_ERR_TARGET and writes nothing for that row;
 *   - the mean loss is the plain sum of the per-token losses divided by N,
 *     summed sequentially in fp64.
 *
 * The backward (oracle_backward) differentiates that definition; see its
 * comment.
 *
 * Parity is pinned for every function here (closed forms, invariants, a
 * library cross-entropy and autograd on fp64 logits, finite differences and
 * exact brute force; see the tests).
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
#define ORACLE_ERR_TARGET (-2)
#define ORACLE_ERR_NOMEM (-3)

/* dtype codes for the stored element type of H and W */
#define ORACLE_BF16 0
#define ORACLE_FP32 1
#define ORACLE_FP64 2   /* only for the oracle's own finite-difference pins */

/* Exact conversion of one stored element to double.  A bf16 value is the
 * upper 16 bits of the fp32 with the same sign, exponent and leading mantissa
 * bits, so widening the bit pattern by 16 zero bits gives the fp32 exactly. */
static double load_elem(const void *base, int dtype, int64_t idx) {
    if (dtype == ORACLE_BF16) {
        uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    if (dtype == ORACLE_FP64) return ((const double *)base)[idx];
    return (double)((const float *)base)[idx];
}

/* One logit z_{ij} = sum_k H_ik W_jk in fp64, k in order (definition Z = H W^T). */
static double logit(const void *H, const void *W, int dtype, int64_t i,
                    int64_t j, int64_t D) {
    double acc = 0.0;
    for (int64_t k = 0; k < D; ++k)
        acc += load_elem(H, dtype, i * D + k) * load_elem(W, dtype, j * D + k);
    return acc;
}

/* Full logits row i into z[0..V). */
int oracle_logits_row(const void *H, const void *W, int dtype, int64_t i,
                      int64_t V, int64_t D, double *z) {
    if (!H || !W || !z || V < 1 || D < 1 || i < 0) return ORACLE_ERR_ARG;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_FP32 && dtype != ORACLE_FP64) return ORACLE_ERR_ARG;
    for (int64_t j = 0; j < V; ++j) z[j] = logit(H, W, dtype, i, j, D);
    return ORACLE_OK;
}

/*
 * Per-token outputs for a subset of rows.
 *   rows[t] (t < nrows) is the row index into H / y; rows == NULL means all N
 *   rows in order (nrows must then equal N).
 *   out_*[t] receive loss, lse, target logit and the row maximum max_j z_ij.
 *   Any out_* pointer may be NULL.
 * Returns ORACLE_OK, ORACLE_ERR_ARG, ORACLE_ERR_TARGET (some selected row has
 * y outside [0, V)) or ORACLE_ERR_NOMEM.
 */
int oracle_forward_rows(const void *H, const void *W, int dtype,
                        const int64_t *y, int64_t N, int64_t V, int64_t D,
                        const int64_t *rows, int64_t nrows, double *out_loss,
                        double *out_lse, double *out_target, double *out_max,
                        int nthreads) {
    if (!H || !W || !y || N < 0 || V < 1 || D < 1 || nrows < 0)
        return ORACLE_ERR_ARG;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_FP32 && dtype != ORACLE_FP64) return ORACLE_ERR_ARG;
    if (!rows && nrows != N) return ORACLE_ERR_ARG;
    for (int64_t t = 0; t < nrows; ++t) {
        int64_t i = rows ? rows[t] : t;
        if (i < 0 || i >= N) return ORACLE_ERR_ARG;
        if (y[i] < 0 || y[i] >= V) return ORACLE_ERR_TARGET;
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int status = ORACLE_OK;
#pragma omp parallel
    {
        double *z = (double *)malloc((size_t)V * sizeof(double));
        if (!z) {
#pragma omp atomic write
            status = ORACLE_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < nrows; ++t) {
            if (!z) continue;
            int64_t i = rows ? rows[t] : t;
            /* Z_i: the full logits row, materialised */
            for (int64_t j = 0; j < V; ++j) z[j] = logit(H, W, dtype, i, j, D);
            /* pass 1: M = max_j z_ij */
            double M = z[0];
            for (int64_t j = 1; j < V; ++j)
                if (z[j] > M) M = z[j];
            /* pass 2: S = sum_j exp(z_ij - M); logsumexp = M + log S */
            double S = 0.0;
            for (int64_t j = 0; j < V; ++j) S += exp(z[j] - M);
            double lse = M + log(S);
            double tgt = z[y[i]];
            if (out_loss) out_loss[t] = lse - tgt;
            if (out_lse) out_lse[t] = lse;
            if (out_target) out_target[t] = tgt;
            if (out_max) out_max[t] = M;
        }
        free(z);
    }
    return status;
}

/*
 * Backward of the weighted loss sum_i g_i loss_i (g_i = dL/dloss_i; g_i = 1/N
 * for the mean loss).  Differentiating loss_i = logsumexp(Z_i) - Z_{i,y_i}
 * (the page, section 1) gives
 *     dL/dZ_ij = g_i (softmax(Z_i)_j - [j == y_i]),  softmax(Z_i)_j = exp(z_ij - lse_i),
 * and through Z = H W^T
 *     dH = (dL/dZ) W        (N x D),     dW = (dL/dZ)^T H      (V x D).
 * Written out directly: pass 1 computes each row's logits and lse and its dH
 * row; pass 2 forms each dW row by recomputing the logits column it needs.
 * Optionally also returns the elementwise magnitudes
 *     bH_ik = sum_j |dZ_ij| |W_jk|,   bW_jk = sum_i |dZ_ij| |H_ik|
 * (the scale that rounding dZ to a narrower type multiplies), for tests.
 * Any of dH, dW, bH, bW may be NULL.  y must lie in [0, V).
 */
int oracle_backward(const void *H, const void *W, int dtype, const int64_t *y,
                    const double *g, int64_t N, int64_t V, int64_t D,
                    double *dH, double *dW, double *bH, double *bW, int nthreads) {
    if (!H || !W || !y || !g || N < 1 || V < 1 || D < 1) return ORACLE_ERR_ARG;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_FP32 && dtype != ORACLE_FP64) return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < N; ++i)
        if (y[i] < 0 || y[i] >= V) return ORACLE_ERR_TARGET;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    double *lse = (double *)malloc((size_t)N * sizeof(double));
    if (!lse) return ORACLE_ERR_NOMEM;
    int status = ORACLE_OK;
    /* pass 1: per row, logits, lse, and the dH row */
#pragma omp parallel
    {
        double *z = (double *)malloc((size_t)V * sizeof(double));
        if (!z) {
#pragma omp atomic write
            status = ORACLE_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < N; ++i) {
            if (!z) continue;
            for (int64_t j = 0; j < V; ++j) z[j] = logit(H, W, dtype, i, j, D);
            double M = z[0];
            for (int64_t j = 1; j < V; ++j)
                if (z[j] > M) M = z[j];
            double S = 0.0;
            for (int64_t j = 0; j < V; ++j) S += exp(z[j] - M);
            lse[i] = M + log(S);
            for (int64_t j = 0; j < V; ++j)  /* z[j] becomes dL/dZ_ij */
                z[j] = g[i] * (exp(z[j] - lse[i]) - (j == y[i] ? 1.0 : 0.0));
            for (int64_t k = 0; k < D; ++k) {
                double acc = 0.0, mag = 0.0;
                for (int64_t j = 0; j < V; ++j) {
                    double w = load_elem(W, dtype, j * D + k);
                    acc += z[j] * w;
                    mag += fabs(z[j]) * fabs(w);
                }
                if (dH) dH[i * D + k] = acc;
                if (bH) bH[i * D + k] = mag;
            }
        }
        free(z);
    }
    if (status != ORACLE_OK) {
        free(lse);
        return status;
    }
    /* pass 2: per vocab row, the dW row (the logits column recomputed) */
    if (dW || bW) {
#pragma omp parallel
        {
            double *dz = (double *)malloc((size_t)N * sizeof(double));
            if (!dz) {
#pragma omp atomic write
                status = ORACLE_ERR_NOMEM;
            }
#pragma omp for schedule(dynamic, 1)
            for (int64_t j = 0; j < V; ++j) {
                if (!dz) continue;
                for (int64_t i = 0; i < N; ++i)
                    dz[i] = g[i] * (exp(logit(H, W, dtype, i, j, D) - lse[i]) -
                                    (j == y[i] ? 1.0 : 0.0));
                for (int64_t k = 0; k < D; ++k) {
                    double acc = 0.0, mag = 0.0;
                    for (int64_t i = 0; i < N; ++i) {
                        double h = load_elem(H, dtype, i * D + k);
                        acc += dz[i] * h;
                        mag += fabs(dz[i]) * fabs(h);
                    }
                    if (dW) dW[j * D + k] = acc;
                    if (bW) bW[j * D + k] = mag;
                }
            }
            free(dz);
        }
    }
    free(lse);
    return status;
}

/* dH rows only (rows[t], t < nrows), with their magnitudes bH: row i of dH
 * depends on row i of the logits alone, so this is cheap for a row sample.
 * Same arithmetic as pass 1 of oracle_backward.  g is indexed by token. */
int oracle_grad_hidden_rows(const void *H, const void *W, int dtype, const int64_t *y,
                            const double *g, int64_t N, int64_t V, int64_t D, const int64_t *rows,
                            int64_t nrows, double *dH, double *bH, int nthreads) {
    if (!H || !W || !y || !g || !rows || !dH || N < 1 || V < 1 || D < 1 || nrows < 0)
        return ORACLE_ERR_ARG;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_FP32 && dtype != ORACLE_FP64) return ORACLE_ERR_ARG;
    for (int64_t t = 0; t < nrows; ++t) {
        if (rows[t] < 0 || rows[t] >= N) return ORACLE_ERR_ARG;
        if (y[rows[t]] < 0 || y[rows[t]] >= V) return ORACLE_ERR_TARGET;
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int status = ORACLE_OK;
#pragma omp parallel
    {
        double *z = (double *)malloc((size_t)V * sizeof(double));
        if (!z) {
#pragma omp atomic write
            status = ORACLE_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < nrows; ++t) {
            if (!z) continue;
            const int64_t i = rows[t];
            for (int64_t j = 0; j < V; ++j) z[j] = logit(H, W, dtype, i, j, D);
            double M = z[0];
            for (int64_t j = 1; j < V; ++j)
                if (z[j] > M) M = z[j];
            double S = 0.0;
            for (int64_t j = 0; j < V; ++j) S += exp(z[j] - M);
            const double lse = M + log(S);
            for (int64_t j = 0; j < V; ++j)
                z[j] = g[i] * (exp(z[j] - lse) - (j == y[i] ? 1.0 : 0.0));
            for (int64_t k = 0; k < D; ++k) {
                double acc = 0.0, mag = 0.0;
                for (int64_t j = 0; j < V; ++j) {
                    double w = load_elem(W, dtype, j * D + k);
                    acc += z[j] * w;
                    mag += fabs(z[j]) * fabs(w);
                }
                dH[t * D + k] = acc;
                if (bH) bH[t * D + k] = mag;
            }
        }
        free(z);
    }
    return status;
}

/* dL/dZ for one row i (V values), given upstream gradient g_i: the vector the
 * backward contracts with W and H.  For tests of the gradient definition. */
int oracle_grad_logits_row(const void *H, const void *W, int dtype, const int64_t *y, double g_i,
                           int64_t i, int64_t V, int64_t D, double *dz) {
    if (!H || !W || !y || !dz || V < 1 || D < 1 || i < 0) return ORACLE_ERR_ARG;
    if (y[i] < 0 || y[i] >= V) return ORACLE_ERR_TARGET;
    int rc = oracle_logits_row(H, W, dtype, i, V, D, dz);
    if (rc != ORACLE_OK) return rc;
    double M = dz[0];
    for (int64_t j = 1; j < V; ++j)
        if (dz[j] > M) M = dz[j];
    double S = 0.0;
    for (int64_t j = 0; j < V; ++j) S += exp(dz[j] - M);
    double lse = M + log(S);
    for (int64_t j = 0; j < V; ++j) dz[j] = g_i * (exp(dz[j] - lse) - (j == y[i] ? 1.0 : 0.0));
    return ORACLE_OK;
}

/* Mean loss: (sum_i loss_i) / n, summed sequentially in fp64.  n == 0 gives NaN. */
double oracle_mean(const double *loss, int64_t n) {
    if (!loss || n <= 0) return NAN;
    double acc = 0.0;
    for (int64_t i = 0; i < n; ++i) acc += loss[i];
    return acc / (double)n;
}

/* Threads the OpenMP runtime would use (for reporting the CPU baseline). */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
