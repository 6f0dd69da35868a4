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

/* dW rows only (vocabulary rows vrows[t], t < nvrows), with their magnitudes
 * bW, and optionally every token's lse.  Row j of dW is
 *     dW_j = sum_i dZ_ij H_i,   dZ_ij = g_i (exp(z_ij - lse_i) - [j == y_i]),
 * which needs the log-sum-exp of EVERY token (the whole logits of each row),
 * but only column j of the logits.  So: pass 1 computes lse_i for all N rows
 * (two passes over a materialised row, as oracle_forward_rows), pass 2 forms
 * each selected dW row from its recomputed logits column (as pass 2 of
 * oracle_backward).  g is indexed by token; lse_out may be NULL. */
int oracle_grad_weight_rows(const void *H, const void *W, int dtype, const int64_t *y,
                            const double *g, int64_t N, int64_t V, int64_t D,
                            const int64_t *vrows, int64_t nvrows, double *dW, double *bW,
                            double *lse_out, int nthreads) {
    if (!H || !W || !y || !g || !vrows || !dW || N < 1 || V < 1 || D < 1 || nvrows < 0)
        return ORACLE_ERR_ARG;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_FP32 && dtype != ORACLE_FP64) return ORACLE_ERR_ARG;
    for (int64_t t = 0; t < nvrows; ++t)
        if (vrows[t] < 0 || vrows[t] >= V) return ORACLE_ERR_ARG;
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
    /* pass 1: every token's log-sum-exp */
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
        }
        free(z);
    }
    /* pass 2: the selected dW rows */
    if (status == ORACLE_OK) {
#pragma omp parallel
        {
            double *dz = (double *)malloc((size_t)N * sizeof(double));
            if (!dz) {
#pragma omp atomic write
                status = ORACLE_ERR_NOMEM;
            }
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < nvrows; ++t) {
                if (!dz) continue;
                const int64_t j = vrows[t];
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
                    dW[t * D + k] = acc;
                    if (bW) bW[t * D + k] = mag;
                }
            }
            free(dz);
        }
    }
    if (status == ORACLE_OK && lse_out)
        for (int64_t i = 0; i < N; ++i) lse_out[i] = lse[i];
    free(lse);
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

/*
 * Quantised output head.
 *
 * Source: the same page, section 2: the first (pure MLX) prototype supported
 * "dense and quantised output heads"; section 9 leaves the quantised variants
 * out of the measured scope.  The page does not define the format.  Reading:
 * the affine group quantisation of MLX, the library that prototype is built
 * on.  Each row j of W is cut into groups of G consecutive elements along D;
 * group g of row j has a scale s_jg and a bias b_jg (bf16 bit patterns), and
 * element k holds an unsigned `bits`-bit code q_jk, so that
 *     W_jk = s_{j, floor(k/G)} * q_jk + b_{j, floor(k/G)}.
 * The codes of one row are packed 32/bits to a uint32 word, lowest bits
 * first: element k sits in word floor(k / (32/bits)) of the row at bit offset
 * bits * (k mod (32/bits)); a row takes D * bits / 32 words.
 * Supported here: bits in {2, 4, 8}, G in {32, 64, 128}, D a multiple of G.
 * The loss is the section-1 definition applied to that W, in fp64: every W_jk
 * is formed exactly (s q is exact in fp64 and so is the sum with b for bf16
 * operands of any practical range) and each logit is a sequential sum over k.
 */
static double bf16_bits_value(uint16_t b) {
    uint32_t bits = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static int quant_args_ok(int bits, int64_t G, int64_t D) {
    if (bits != 2 && bits != 4 && bits != 8) return 0;
    if (G != 32 && G != 64 && G != 128) return 0;
    return D >= G && D % G == 0;
}

/* The code q_jk, unpacked from its word. */
static uint32_t quant_code(const uint32_t *wq, int bits, int64_t D, int64_t j, int64_t k) {
    const int64_t per_word = 32 / bits;
    const uint32_t word = wq[j * (D / per_word) + k / per_word];
    return (word >> (bits * (int)(k % per_word))) & ((1u << bits) - 1u);
}

/* W_jk = s_jg q_jk + b_jg with g = floor(k / G). */
static double dequant_elem(const uint32_t *wq, const uint16_t *scales, const uint16_t *biases,
                           int bits, int64_t G, int64_t D, int64_t j, int64_t k) {
    const int64_t g = j * (D / G) + k / G;
    return bf16_bits_value(scales[g]) * (double)quant_code(wq, bits, D, j, k) +
           bf16_bits_value(biases[g]);
}

/* The whole dequantised W (V x D doubles), for small cases. */
int oracle_dequantize(const uint32_t *wq, const uint16_t *scales, const uint16_t *biases,
                      int bits, int64_t G, int64_t V, int64_t D, double *W) {
    if (!wq || !scales || !biases || !W || V < 1 || !quant_args_ok(bits, G, D))
        return ORACLE_ERR_ARG;
    for (int64_t j = 0; j < V; ++j)
        for (int64_t k = 0; k < D; ++k)
            W[j * D + k] = dequant_elem(wq, scales, biases, bits, G, D, j, k);
    return ORACLE_OK;
}

/*
 * Per-token outputs for a subset of rows with a quantised head: H is (N, D)
 * bf16 bit patterns; wq, scales and biases hold W as described above.  Same
 * row selection, outputs and errors as oracle_forward_rows.  Each logit is
 * z_ij = sum_k H_ik W_jk with W_jk formed on the fly (the full W is never
 * held), then the same two-pass log-sum-exp.
 */
int oracle_forward_quantized_rows(const uint16_t *H, const uint32_t *wq, const uint16_t *scales,
                                  const uint16_t *biases, int bits, int64_t G,
                                  const int64_t *y, int64_t N, int64_t V, int64_t D,
                                  const int64_t *rows, int64_t nrows, double *out_loss,
                                  double *out_lse, double *out_target, double *out_max,
                                  int nthreads) {
    if (!H || !wq || !scales || !biases || !y || N < 0 || V < 1 || nrows < 0 ||
        !quant_args_ok(bits, G, D))
        return ORACLE_ERR_ARG;
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
        double *h = (double *)malloc((size_t)D * sizeof(double));
        if (!z || !h) {
#pragma omp atomic write
            status = ORACLE_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < nrows; ++t) {
            if (!z || !h) continue;
            int64_t i = rows ? rows[t] : t;
            for (int64_t k = 0; k < D; ++k) h[k] = bf16_bits_value(H[i * D + k]);
            /* Z_i with the dequantised W */
            for (int64_t j = 0; j < V; ++j) {
                double acc = 0.0;
                for (int64_t k = 0; k < D; ++k)
                    acc += h[k] * dequant_elem(wq, scales, biases, bits, G, D, j, k);
                z[j] = acc;
            }
            double M = z[0];
            for (int64_t j = 1; j < V; ++j)
                if (z[j] > M) M = z[j];
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
        free(h);
    }
    return status;
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
