/*
 * gptq_oracle.c -- plain float64 CPU checker for the per-layer GPTQ path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header or table with the CUDA library.
 *
 * Every routine follows the GPTQ overview page (robocikowo.com/technologie-ai/gptq):
 *   - "Jak działa" and "Komponenty": H = 2 X X^T from the layer inputs; columns
 *     quantized one by one in a fixed order; after each column the remaining
 *     weights are corrected by the Optimal Brain Surgeon rule using the inverse
 *     Hessian; a Cholesky form of the inverse Hessian; one scale per group.
 *   - "Hiperparametry": bit width, weights per scale (group size), activation
 *     order, value added to the Hessian diagonal (damping).
 *   - "Ewolucja": GPTQ extends Optimal Brain Quantization (OBQ); the OBQ
 *     inverse-Hessian update after removing one coordinate is what
 *     orc_obs_upper() below performs.
 * and the AutoGPTQ integration page ("The Quantization Algorithm"): weights
 * quantized one at a time, remaining ones updated to compensate.
 *
 * Arithmetic is binary64 except the quantizer's grid choice and rounding
 * decision (scale, zero, code), which are taken in binary32 on binary32-rounded
 * operands -- the precision the CUDA kernels decide in -- so that an integer
 * code is decided the same way on both sides.  Build with -ffp-contract=off so
 * that no multiply-add is fused.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_NOT_PD 2

static double bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* H[i][j] += 2 * sum_t X[t][i] * X[t][j] for all i, j (full matrix).
 * X: bf16 bit patterns [n][d] row-major, widened exactly to binary64.
 * Page: "Jak działa", H = 2 X X^T (X there is d x N; here tokens are rows). */
int orc_hessian_accumulate(double *H, const uint16_t *X, int64_t n, int64_t d)
{
    if (!H || !X || n < 0 || d <= 0) return ORC_ERR_ARG;
    const int64_t T = 128;
    double *xc = (double *)malloc((size_t)(T * d) * sizeof(double));
    if (!xc) return ORC_ERR_ARG;
    for (int64_t t0 = 0; t0 < n; t0 += T) {
        int64_t tn = (n - t0 < T) ? n - t0 : T;
        for (int64_t k = 0; k < tn * d; k++) xc[k] = bf16_to_f64(X[t0 * d + k]);
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < d; i++) {
            double *Hi = H + i * d;
            for (int64_t t = 0; t < tn; t++) {
                const double *xt = xc + t * d;
                double a = 2.0 * xt[i];
                if (a == 0.0) continue;
                for (int64_t j = 0; j < d; j++) Hi[j] += a * xt[j];
            }
        }
    }
    free(xc);
    return ORC_OK;
}

/* out[a][b] = 2 * sum_t X[t][I[a]] * X[t][J[b]]: a block of entries of the
 * same H, computed one by one (for sampled checks at full size). */
int orc_hessian_block(double *out, const uint16_t *X, int64_t n, int64_t d,
                      const int64_t *I, int64_t ni, const int64_t *J, int64_t nj)
{
    if (!out || !X || !I || !J || n < 0 || d <= 0) return ORC_ERR_ARG;
    for (int64_t a = 0; a < ni; a++)
        if (I[a] < 0 || I[a] >= d) return ORC_ERR_ARG;
    for (int64_t b = 0; b < nj; b++)
        if (J[b] < 0 || J[b] >= d) return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t a = 0; a < ni; a++) {
        for (int64_t b = 0; b < nj; b++) {
            double s = 0.0;
            for (int64_t t = 0; t < n; t++)
                s += bf16_to_f64(X[t * d + I[a]]) * bf16_to_f64(X[t * d + J[b]]);
            out[a * nj + b] = 2.0 * s;
        }
    }
    return ORC_OK;
}

/* In-place inverse of a d x d matrix by Gauss-Jordan elimination with partial
 * pivoting on the augmented matrix [A | I].  Returns ORC_ERR_NOT_PD when a
 * pivot is exactly zero or not finite (singular for our purposes). */
int orc_inverse_gauss_jordan(double *A, int64_t d)
{
    if (!A || d <= 0) return ORC_ERR_ARG;
    int64_t w = 2 * d;
    double *M = (double *)calloc((size_t)(d * w), sizeof(double));
    if (!M) return ORC_ERR_ARG;
    for (int64_t i = 0; i < d; i++) {
        memcpy(M + i * w, A + i * d, (size_t)d * sizeof(double));
        M[i * w + d + i] = 1.0;
    }
    int status = ORC_OK;
    for (int64_t c = 0; c < d; c++) {
        int64_t p = c;
        double best = fabs(M[c * w + c]);
        for (int64_t r = c + 1; r < d; r++) {
            double v = fabs(M[r * w + c]);
            if (v > best) { best = v; p = r; }
        }
        if (!(best > 0.0) || !isfinite(best)) { status = ORC_ERR_NOT_PD; break; }
        if (p != c) {
            for (int64_t k = 0; k < w; k++) {
                double t = M[c * w + k];
                M[c * w + k] = M[p * w + k];
                M[p * w + k] = t;
            }
        }
        double piv = M[c * w + c];
        for (int64_t k = 0; k < w; k++) M[c * w + k] /= piv;
        const double *rc = M + c * w;
#pragma omp parallel for schedule(static)
        for (int64_t r = 0; r < d; r++) {
            if (r == c) continue;
            double f = M[r * w + c];
            if (f == 0.0) continue;
            double *rr = M + r * w;
            for (int64_t k = 0; k < w; k++) rr[k] -= f * rc[k];
        }
    }
    if (status == ORC_OK)
        for (int64_t i = 0; i < d; i++)
            memcpy(A + i * d, M + i * w + d, (size_t)d * sizeof(double));
    free(M);
    return status;
}

/* U (upper triangular, d x d) from Hinv = H_d^{-1} by successive OBS/OBQ
 * eliminations: for c = 0..d-1 the row U[c][c:] = Hinv[c][c:] / sqrt(Hinv[c][c]),
 * then coordinate c is removed from the inverse Hessian,
 *   Hinv <- Hinv - Hinv[:,c] Hinv[c,:] / Hinv[c][c].
 * The rows so produced satisfy U^T U = Hinv (the Cholesky form of the inverse
 * Hessian, page "Komponenty").  Entries below the diagonal are set to 0.
 * Returns ORC_ERR_NOT_PD if a pivot is not positive and finite. */
int orc_obs_upper(const double *Hinv, int64_t d, double *U)
{
    if (!Hinv || !U || d <= 0) return ORC_ERR_ARG;
    double *M = (double *)malloc((size_t)(d * d) * sizeof(double));
    if (!M) return ORC_ERR_ARG;
    memcpy(M, Hinv, (size_t)(d * d) * sizeof(double));
    memset(U, 0, (size_t)(d * d) * sizeof(double));
    int status = ORC_OK;
    for (int64_t c = 0; c < d; c++) {
        double p = M[c * d + c];
        if (!(p > 0.0) || !isfinite(p)) { status = ORC_ERR_NOT_PD; break; }
        double r = sqrt(p);
        for (int64_t j = c; j < d; j++) U[c * d + j] = M[c * d + j] / r;
#pragma omp parallel for schedule(static)
        for (int64_t i = c + 1; i < d; i++) {
            double f = M[i * d + c] / p;
            if (f == 0.0) continue;
            for (int64_t j = c + 1; j < d; j++) M[i * d + j] -= f * M[c * d + j];
        }
    }
    free(M);
    return status;
}

/* Grid of the asymmetric min/max quantizer on the values v[0..n): the range
 * always contains 0; an all-zero range becomes [-1, 1].  Decided in binary32. */
static void qgrid(const double *v, int64_t n, int maxq, float *s_out, float *z_out, float *zraw)
{
    float xmin = 0.0f, xmax = 0.0f;
    for (int64_t k = 0; k < n; k++) {
        float f = (float)v[k];
        if (f < xmin) xmin = f;
        if (f > xmax) xmax = f;
    }
    if (xmin == xmax) { xmin = -1.0f; xmax = 1.0f; }
    float s = (xmax - xmin) / (float)maxq;
    float zr = -xmin / s;
    float z = rintf(zr);
    *s_out = s;
    *z_out = z;
    if (zraw) *zraw = zr;
}

static int qcode(double w, float s, float z, int maxq, float *qraw)
{
    float r = (float)w / s;
    if (qraw) *qraw = r;
    float q = rintf(r) + z;
    if (q < 0.0f) q = 0.0f;
    if (q > (float)maxq) q = (float)maxq;
    return (int)q;
}

/* The column loop of GPTQ for every row of W, in processing order.
 *
 * W     [d_out][d_in]  in: weights (processing order); out: dequantized W^.
 * U     [d_in][d_in]   upper factor with U^T U = H_d^{-1} (same order).
 * block <= 0           unblocked: after column c the whole remainder of the
 *                      row is corrected at once, w[c+1:] -= e * U[c][c+1:].
 * block  > 0           lazy batch: the correction is applied inside the
 *                      current block immediately and to the columns after it
 *                      once, at the end of the block, as w -= E_blk U_blk.
 * group_size > 0       a new (scale, zero) at every group_size-th column, from
 *                      the row's current values of that group's columns;
 * group_size < 0       one (scale, zero) per row from the original row.
 * Per column: q = clamp(rint(w/s) + z, 0, maxq); w^ = s (q - z);
 *             e = (w - w^) / U[c][c].
 * Outputs: codes [d_out][d_in], scales/zeros [d_out][n_groups],
 *          E [d_out][d_in] (optional, the scaled errors e).
 * Optional diagnostics (NULL to skip): qraw [d_out][d_in] = w / s before
 * rounding, zraw [d_out][n_groups] = -min / s before rounding; they tell how
 * close each integer decision was to a rounding tie. */
int orc_gptq_rows(double *W, const double *U, int64_t d_out, int64_t d_in, int bits,
                  int64_t group_size, int64_t block, uint8_t *codes, float *scales,
                  float *zeros, double *E, float *qraw, float *zraw)
{
    if (!W || !U || !codes || !scales || !zeros || d_out < 0 || d_in <= 0 || bits < 1 ||
        bits > 8 || group_size == 0)
        return ORC_ERR_ARG;
    const int maxq = (1 << bits) - 1;
    const int64_t n_groups = group_size > 0 ? (d_in + group_size - 1) / group_size : 1;
    int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < d_out; r++) {
        double *w = W + r * d_in;
        double *e_row = (double *)malloc((size_t)d_in * sizeof(double));
        if (!e_row) { status = ORC_ERR_ARG; continue; }
        float s = 0.0f, z = 0.0f;
        if (group_size < 0) {
            qgrid(w, d_in, maxq, &s, &z, zraw ? zraw + r : NULL);
            scales[r] = s;
            zeros[r] = z;
        }
        for (int64_t c = 0; c < d_in; c++) {
            if (group_size > 0 && c % group_size == 0) {
                int64_t len = (d_in - c < group_size) ? d_in - c : group_size;
                qgrid(w + c, len, maxq, &s, &z,
                      zraw ? zraw + r * n_groups + c / group_size : NULL);
                scales[r * n_groups + c / group_size] = s;
                zeros[r * n_groups + c / group_size] = z;
            }
            int q = qcode(w[c], s, z, maxq, qraw ? qraw + r * d_in + c : NULL);
            double what = (double)s * ((double)q - (double)z);
            double e = (w[c] - what) / U[c * d_in + c];
            codes[r * d_in + c] = (uint8_t)q;
            w[c] = what;
            e_row[c] = e;
            if (block <= 0) {
                for (int64_t k = c + 1; k < d_in; k++) w[k] -= e * U[c * d_in + k];
            } else {
                int64_t b0 = (c / block) * block;
                int64_t b1 = (b0 + block < d_in) ? b0 + block : d_in;
                for (int64_t k = c + 1; k < b1; k++) w[k] -= e * U[c * d_in + k];
                if (c == b1 - 1) {
                    for (int64_t k = b1; k < d_in; k++) {
                        double acc = 0.0;
                        for (int64_t i = b0; i < b1; i++) acc += e_row[i] * U[i * d_in + k];
                        w[k] -= acc;
                    }
                }
            }
        }
        if (E) memcpy(E + r * d_in, e_row, (size_t)d_in * sizeof(double));
        free(e_row);
    }
    return status;
}

/* ---- GPTQ onto the two-level Q4_K grid ---------------------------------
 *
 * The gguf Q4_K layout as the torchao pull request "Add gguf q4_k
 * quantization" describes it: w = q * block_scale + block_min with 4-bit q,
 * a 6-bit scale and a 6-bit min per block, and a second level (super-block
 * scales) that quantizes those.  Blocks of 32 columns, super-blocks of 8
 * blocks (256 columns), in processing order:
 *     w^ = d sc q - dmin m,   q in 0..15,  sc in 1..63,  m in 0..63.
 * Parameter choice (the simple min/max choice of the pull request), decided
 * in binary32 like the one-level grid:
 *   - range of a block: [min(0, min v), max(0, max v)], an all-zero block
 *     taking [-1, 1]; raw scale = (max - min) / 15, raw offset = -min >= 0;
 *   - at a super-block's first column, from the row's current values of its
 *     256 columns: d = max raw scale / 63, dmin = max raw offset / 63;
 *   - at a block's first column, from the row's current values of its 32
 *     columns: sc = clamp(rint(scale / d), 1, 63), m = rint(offset / dmin)
 *     clamped to 0..63 (0 when dmin = 0).
 * Both levels use the values as updated by every earlier column, as the
 * one-level grid does at its group starts.  Per column:
 *     q = clamp(rint((w + dmin m) / (d sc)), 0, 15), w^ = d sc q - dmin m,
 *     e = (w - w^) / U[c][c], compensation as in orc_gptq_rows.
 * d_in must be a multiple of 256.  Outputs: codes [d_out][d_in]; sc6, m6
 * [d_out][d_in / 32]; dsup, dmin [d_out][d_in / 256]; E (optional).
 * Optional diagnostics (NULL to skip), the decision values before rounding:
 * qraw [d_out][d_in] = (w + o) / s, scraw and mraw [d_out][d_in / 32] =
 * scale / d and offset / dmin (0 when dmin = 0); they tell how close each
 * integer decision was to a rounding tie. */
static void q4k_block_range(const double *v, int64_t n, float *scale, float *offset)
{
    float xmin = 0.0f, xmax = 0.0f;
    for (int64_t k = 0; k < n; k++) {
        float f = (float)v[k];
        if (f < xmin) xmin = f;
        if (f > xmax) xmax = f;
    }
    if (xmin == xmax) { xmin = -1.0f; xmax = 1.0f; }
    *scale = (xmax - xmin) / 15.0f;
    *offset = -xmin;
}

int orc_gptq_rows_q4k(double *W, const double *U, int64_t d_out, int64_t d_in, int64_t block,
                      uint8_t *codes, uint8_t *sc6, uint8_t *m6, float *dsup, float *dmin,
                      double *E, float *qraw, float *scraw, float *mraw)
{
    if (!W || !U || !codes || !sc6 || !m6 || !dsup || !dmin || d_out < 0 || d_in <= 0 ||
        d_in % 256 != 0)
        return ORC_ERR_ARG;
    const int64_t nb = d_in / 32, ns = d_in / 256;
    int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < d_out; r++) {
        double *w = W + r * d_in;
        double *e_row = (double *)malloc((size_t)d_in * sizeof(double));
        if (!e_row) { status = ORC_ERR_ARG; continue; }
        float d = 1.0f, dm = 0.0f, s = 1.0f, o = 0.0f;
        for (int64_t c = 0; c < d_in; c++) {
            if (c % 256 == 0) {
                float smax = 0.0f, omax = 0.0f;
                for (int b = 0; b < 8; b++) {
                    float sc, of;
                    q4k_block_range(w + c + 32 * b, 32, &sc, &of);
                    if (sc > smax) smax = sc;
                    if (of > omax) omax = of;
                }
                d = smax / 63.0f;
                dm = omax / 63.0f;
                dsup[r * ns + c / 256] = d;
                dmin[r * ns + c / 256] = dm;
            }
            if (c % 32 == 0) {
                float sc, of;
                q4k_block_range(w + c, 32, &sc, &of);
                float scr = sc / d;
                float mr = dm > 0.0f ? of / dm : 0.0f;
                if (scraw) scraw[r * nb + c / 32] = scr;
                if (mraw) mraw[r * nb + c / 32] = mr;
                float qs = rintf(scr);
                if (qs < 1.0f) qs = 1.0f;
                if (qs > 63.0f) qs = 63.0f;
                float qm = rintf(mr);
                if (qm < 0.0f) qm = 0.0f;
                if (qm > 63.0f) qm = 63.0f;
                sc6[r * nb + c / 32] = (uint8_t)qs;
                m6[r * nb + c / 32] = (uint8_t)qm;
                s = d * qs;
                o = dm * qm;
            }
            float qr = ((float)w[c] + o) / s;
            if (qraw) qraw[r * d_in + c] = qr;
            float q = rintf(qr);
            if (q < 0.0f) q = 0.0f;
            if (q > 15.0f) q = 15.0f;
            double what = (double)s * (double)q - (double)o;
            double e = (w[c] - what) / U[c * d_in + c];
            codes[r * d_in + c] = (uint8_t)q;
            w[c] = what;
            e_row[c] = e;
            if (block <= 0) {
                for (int64_t k = c + 1; k < d_in; k++) w[k] -= e * U[c * d_in + k];
            } else {
                int64_t b0 = (c / block) * block;
                int64_t b1 = (b0 + block < d_in) ? b0 + block : d_in;
                for (int64_t k = c + 1; k < b1; k++) w[k] -= e * U[c * d_in + k];
                if (c == b1 - 1) {
                    for (int64_t k = b1; k < d_in; k++) {
                        double acc = 0.0;
                        for (int64_t i = b0; i < b1; i++) acc += e_row[i] * U[i * d_in + k];
                        w[k] -= acc;
                    }
                }
            }
        }
        if (E) memcpy(E + r * d_in, e_row, (size_t)d_in * sizeof(double));
        free(e_row);
    }
    return status;
}
